"""Build the CUDA library ``libattn.so`` in-tree for sm_100a.

    python -m tiled_attention_blackwell_b200.build [--force]

nvcc cross-compiles without a GPU.  The CUDA runtime is linked statically, so
the library needs only the NVIDIA driver at run time.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libattn.so")
# The rescale-statistics build: the same kernels compiled with
# -DATTN_COUNT_RESCALES (per-row counters reduced into a device buffer set
# through attn_count_set_buffer); never the library the product loads.
COUNT_LIB = os.path.join(PKG, "libattn_count.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared",
]


def _sources():
    deps = glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
    deps.append(os.path.join(ROOT, "include", "attn.h"))
    return deps


def _build_one(out: str, defines, force: bool, verbose: bool) -> str:
    newest = max(os.path.getmtime(p) for p in _sources())
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [NVCC, *NVCC_FLAGS, *[f"-D{d}" for d in defines], "-o", tmp,
           os.path.join(CSRC, "attn_api.cu")]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile csrc/attn_api.cu (and the kernels it includes) into libattn.so."""
    return _build_one(LIB, (), force, verbose)


def build_count(force: bool = False, verbose: bool = False) -> str:
    """The rescale-statistics build, libattn_count.so."""
    return _build_one(COUNT_LIB, ("ATTN_COUNT_RESCALES",), force, verbose)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
    if "--count" in sys.argv:
        print(build_count(force="--force" in sys.argv, verbose=True))
