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
SOURCES = [os.path.join(PKG, "csrc", n) for n in ("kvq.cu", "kvq_attn.cu", "kvq_attn_d64.cu", "kvq_attn_d128.cu",
                                                        "kvq_attn_d256.cu", "kvq_ex.cu", "kvq_srft_d64.cu",
                                                        "kvq_srft_d96.cu", "kvq_srft_d128.cu", "kvq_srft_d256.cu")]
# Per-unit flags.  The codec units keep --fmad=false: their results are
# defined bit for bit, and a contracted multiply-add rounds once where the
# codec's definition rounds twice.  The decode attention is checked against
# the oracle to a derived tolerance, not bit for bit, so its multiply-add
# pairs may contract (one rounding instead of two only shrinks the error).
UNIT_FLAGS = {n: ["--fmad=true"] for n in ("kvq_attn_d64.cu", "kvq_attn_d128.cu", "kvq_attn_d256.cu")}
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
    """Compile every translation unit to an object in parallel, then link."""
    import concurrent.futures
    import tempfile

    compile_flags = [f for f in FLAGS if f not in ("-shared", "-cudart", "shared")
                     and not f.startswith("-rpath")]
    compile_flags = [f for f in compile_flags if f != "-Xlinker"]
    with tempfile.TemporaryDirectory() as td:
        objs = [os.path.join(td, os.path.basename(src) + ".o") for src in SOURCES]

        def one(src, obj):
            unit = UNIT_FLAGS.get(os.path.basename(src), [])
            flags = [f for f in compile_flags if not (unit and f.startswith("--fmad="))] + unit
            cmd = [NVCC, *flags, *(extra or []), "-I", INCLUDE, "-c", src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
            return subprocess.run(cmd, capture_output=True, text=True)

        with concurrent.futures.ThreadPoolExecutor(len(SOURCES)) as ex:
            results = list(ex.map(one, SOURCES, objs))
        for res in results:
            if res.returncode != 0:
                raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
            if verbose:
                sys.stderr.write(res.stderr)
        link = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "shared",
                "-Xlinker", "-rpath,/usr/local/cuda/lib64", *objs, "-o", LIBRARY]
        res = subprocess.run(link, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("nvcc link failed:\n" + res.stdout + res.stderr)
    return LIBRARY


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
