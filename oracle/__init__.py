"""fp64 CPU oracle for FiX attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the library.  It shares no
code with the CUDA path; both sides are fed from ``synth`` (random draws only).
"""
from .fix_ref import (backward, dq_rows, forward, forward_rows, suffix_backward,  # noqa: F401
                      to64, unit_backward, unit_forward)
from .brute import brute_forward, brute_loss  # noqa: F401
