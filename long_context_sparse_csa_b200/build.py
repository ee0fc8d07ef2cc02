"""Build libcsa.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: python -m long_context_sparse_csa_b200.build [--force] [--trace]

--trace builds libcsa_trace.so instead: the same kernels with CSA_TRACE defined, so they record
per-CTA %globaltimer stamps into device arrays that the csa_trace_read* symbols of that library copy
out (a diagnostic build; the product library never has them).
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libcsa.so")
TRACE_LIB = os.path.join(HERE, "libcsa_trace.so")

SOURCES = ["compress.cu", "index_score.cu", "topk.cu", "attend.cu", "api.cu", "static_scratch.cu", "debug.cu", "index_decode.cu", "index_prep.cu", "shard.cu", "attend_prefill.cu"]
HEADERS = ["common.cuh", "sm100.cuh", "kernels.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
]


def _nvcc():
    for cand in [os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"]:
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, trace: bool = False) -> str:
    build_dir = os.path.join(BUILD, "trace") if trace else BUILD
    lib = TRACE_LIB if trace else LIB
    flags = NVCC_FLAGS + (["-DCSA_TRACE"] if trace else [])
    os.makedirs(build_dir, exist_ok=True)
    nvcc = _nvcc()
    headers = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "csa.h")]
    objs = []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(build_dir, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s] + headers):
            cmd = [nvcc, *flags, "-I", INCLUDE, "-c", s, "-o", o]
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.run(cmd, check=True)
    if force or _stale(lib, objs):
        cmd = [nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", lib,
               "-lcudart_static", "-ldl", "-lpthread", "-lrt"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, trace="--trace" in sys.argv))
