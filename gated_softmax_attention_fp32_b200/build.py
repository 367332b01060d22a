"""Build libfixattn.so (sm_100a) in-tree with nvcc.

    python -m gated_softmax_attention_fp32_b200.build [--force] [--jobs N]

Each ``csrc/*.cu`` file is compiled to an object under ``_build/`` and the
objects are linked into ``gated_softmax_attention_fp32_b200/libfixattn.so``.
A second link, ``libfixattn_test.so``, is built from the same sources with
``-DFIX_TEST_HOOKS``: it adds the hooks the failure-detection tests use (a
forward whose waits expire on purpose) and is never loaded by the product
path.  A file is recompiled only when it or any header under
``csrc/``/``include/`` changed (content hash).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libfixattn.so")
TEST_LIB = os.path.join(PKG, "libfixattn_test.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
         "--expt-relaxed-constexpr", "-Xptxas", "-v"] + ARCH


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the FiX CUDA library cannot be built")


def _headers_digest() -> str:
    h = hashlib.sha256()
    for d in (CSRC, INCLUDE):
        for name in sorted(os.listdir(d)):
            if name.endswith((".h", ".cuh", ".hpp")):
                with open(os.path.join(d, name), "rb") as f:
                    h.update(name.encode()); h.update(f.read())
    return h.hexdigest()


def _compile(src: str, hdr: str, force: bool, variant: str = "") -> tuple:
    base = os.path.splitext(os.path.basename(src))[0]
    outdir = os.path.join(BUILD, variant) if variant else BUILD
    obj = os.path.join(outdir, base + ".o")
    stamp = obj + ".hash"
    extra = ["-DFIX_TEST_HOOKS"] if variant == "test" else []
    with open(src, "rb") as f:
        digest = hashlib.sha256(f.read() + hdr.encode() + " ".join(FLAGS + extra).encode()).hexdigest()
    if not force and os.path.exists(obj) and os.path.exists(stamp) and open(stamp).read() == digest:
        return obj, "", False
    cmd = [nvcc(), *FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    with open(stamp, "w") as f:
        f.write(digest)
    return obj, r.stderr, True


def _link(objs, out, rebuilt, force):
    if rebuilt or force or not os.path.exists(out):
        tmp = out + ".tmp"
        cmd = [nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, out)


def build(force: bool = False, jobs: int = 0, verbose: bool = False) -> str:
    os.makedirs(os.path.join(BUILD, "test"), exist_ok=True)
    srcs = sorted(os.path.join(CSRC, n) for n in os.listdir(CSRC) if n.endswith(".cu"))
    hdr = _headers_digest()
    jobs = jobs or min(2 * len(srcs), os.cpu_count() or 1)
    work = [(s_, "") for s_ in srcs] + [(s_, "test") for s_ in srcs]
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        results = list(ex.map(lambda a: _compile(a[0], hdr, force, a[1]), work))
    if verbose:
        for r in results:
            if r[1]:
                sys.stderr.write(r[1])
    prod, test = results[:len(srcs)], results[len(srcs):]
    _link([r[0] for r in prod], LIB, any(r[2] for r in prod), force)
    _link([r[0] for r in test], TEST_LIB, any(r[2] for r in test), force)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=0)
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args()
    print(build(a.force, a.jobs, a.verbose))
