"""Build the CUDA library libwq.so in-tree for sm_100a (B200).

    python weight_only_quantized_02_b200/build.py [--force] [--verbose]

Each .cu file under csrc/ is compiled with nvcc for
``-gencode arch=compute_100a,code=sm_100a`` and linked into one shared
library with the CUDA runtime linked statically (the process may also hold
torch's own runtime).  Objects go to ``_build/`` next to this file.
"""
from __future__ import annotations

import concurrent.futures
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libwq.so")

SOURCES = ["wq_api.cu", "wq_pack.cu", "wq_gemv.cu", "wq_gemv_sk.cu", "wq_gemv_i8.cu", "wq_gemm.cu", "wq_gemm_sk.cu",
           "wq_gemm_i8.cu", "wq_gemm_i4.cu", "wq_gemm_w4.cu", "wq_topk.cu", "wq_sk_debug.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libwq.so")


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "wq.h"))
    files.append(os.path.abspath(__file__))  # the source list and flags
    return files


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(f) for f in _deps())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    os.makedirs(BUILD, exist_ok=True)
    cc = nvcc()
    common = ARCH + [
        "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
        "--expt-relaxed-constexpr",
    ]
    if verbose:
        common += ["-Xptxas", "-v"]
    objs = [os.path.join(BUILD, src.replace(".cu", ".o")) for src in SOURCES]

    def compile_one(i):
        cmd = [cc] + common + ["-c", os.path.join(CSRC, SOURCES[i]), "-o", objs[i]]
        return subprocess.run(cmd, capture_output=True, text=True)

    # the translation units are independent: compile them side by side
    jobs = max(1, min(len(SOURCES), os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(jobs) as ex:
        results = list(ex.map(compile_one, range(len(SOURCES))))
    for src, r in zip(SOURCES, results):
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("nvcc failed on " + src)
        if verbose:
            sys.stderr.write(r.stdout + r.stderr)
    tmp = LIB + ".tmp"
    cmd = [cc] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs + ["-lpthread", "-ldl", "-lrt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("link of libwq.so failed")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
