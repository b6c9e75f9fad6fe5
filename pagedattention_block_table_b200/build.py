"""Build ``libpagedattn.so`` (the CUDA kernels and their C ABI) in-tree with nvcc for sm_100a.

The whole library is one translation unit (``csrc/api.cu`` includes every kernel header).
Run ``python -m pagedattention_block_table_b200.build`` or call :func:`build`.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpagedattn.so")
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(CSRC, "*.cpp")) + [os.path.join(ROOT, "include", "pagedattn.h")])


def _code_only(text: str) -> str:
    """Source text without comments and blank lines (what the compiler sees, for the digest)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def source_digest(names=None) -> str:
    """sha256 of CUDA sources, comments left out: identifies which kernels a profile was taken on.
    `names` lists the csrc files a kernel depends on (for example its header, pa_common.cuh and api.cu,
    which holds its launch code); None takes every csrc/*.cu and *.cuh.  Host-only C++ (the block
    manager) never enters it."""
    import hashlib
    h = hashlib.sha256()
    if names is None:
        files = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")))
    else:
        files = [os.path.join(CSRC, n) for n in sorted(names)]
    for src in files:
        with open(src, encoding="utf-8") as f:
            h.update(os.path.basename(src).encode() + b"\0" + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, out: str = LIB, extra=()) -> str:
    """Compile if any source is newer than the library (or ``force``).  Returns the .so path."""
    if not force and os.path.exists(out):
        t = os.path.getmtime(out)
        if all(os.path.getmtime(s) <= t for s in _sources()) and not extra:
            return out
    # the CUDA side is one translation unit (api.cu includes every kernel header); the host-only
    # block manager is a separate C++ file
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-o", out + ".tmp", os.path.join(CSRC, "api.cu"),
           os.path.join(CSRC, "block_manager.cpp")]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
