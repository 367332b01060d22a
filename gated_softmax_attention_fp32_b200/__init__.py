"""FiX attention for NVIDIA B200 (sm_100a): C-ABI CUDA library plus a thin binding."""
from . import fixattn  # noqa: F401
from .fixattn import fix_attn, fix_attn_bwd, fix_attn_fwd  # noqa: F401
