"""Build the C-ABI library ``libsage_attn.so`` in-tree with nvcc for sm_100a.

    python -m quantized_attention_02_b200.build [--force] [--verbose]

Each .cu file is compiled separately (``-gencode arch=compute_100a,code=sm_100a
-lineinfo -O3``) and linked with the static CUDA runtime, so the library only
needs the GPU driver at run time (and nothing to load on a machine without one).
The quantization kernels are compiled with ``--fmad=false`` on top of using
explicitly rounded intrinsics, so no multiply-add contraction can change their
bit-exact results.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libsage_attn.so")

SOURCES = {
    "capi.cu": [],
    "prep_kernels.cu": ["--fmad=false"],
    "attn_kernels.cu": [],
    "noalloc.cu": [],
    "host_pipeline.cu": [],
    "mma_rate.cu": [],
    "sparse_kernels.cu": [],
}
HEADERS = ["sm100_ptx.cuh", "attn_kernels.cuh", "attn_v3.cuh", "prep_kernels.cuh", "workspace.cuh",
           "sparse_kernels.cuh", "fp4_codes.cuh", "attn_fp4.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    headers = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "sage_attn.h")]
    objs = []
    for src, extra in SOURCES.items():
        s = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, [s, __file__] + headers):
            cmd = [nvcc(), *ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                   "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC, *extra, "-c", s, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
                print(" ".join(cmd), flush=True)
            subprocess.run(cmd, check=True)
    if force or _stale(LIB, objs):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose))
    return 0


if __name__ == "__main__":
    sys.exit(main())
