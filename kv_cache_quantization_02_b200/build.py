"""Build libkvq.so in-tree with nvcc for sm_100a.

    python -m kv_cache_quantization_02_b200.build

The library links the CUDA runtime dynamically (libcudart.so.12), so that a
process that already loaded it (e.g. through torch) shares one runtime, and
with it the current device, with this library.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SOURCES = [os.path.join(PKG, "csrc", n) for n in ("kvq.cu", "kvq_attn.cu", "kvq_ex.cu")]
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libkvq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--fmad=false",                     # no multiply-add contraction anywhere
    "-Xcompiler", "-fPIC,-O2",
    "-shared", "-cudart", "shared",
    "-Xlinker", "-rpath,/usr/local/cuda/lib64",
]


def build(verbose: bool = False, extra: list[str] | None = None) -> str:
    cmd = [NVCC, *FLAGS, *(extra or []), "-I", INCLUDE, *SOURCES, "-o", LIBRARY]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    return LIBRARY


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
