"""Build libkv2.so in-tree for sm_100a (nvcc, no JIT cache).

    python -m bit_kv_cache_centroid_b200.build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJDIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libkv2.so")
SOURCES = ["api.cu", "quantize.cu", "decode.cu", "decode_groups.cu", "decode_noalloc.cu", "fit.cu", "chunk.cu", "fit_centroids.cu", "top1.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]


def _newer(src_paths, target):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(p) > t for p in src_paths)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(OBJDIR, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    headers.append(os.path.join(INCLUDE, "kv2.h"))
    objs, jobs = [], []
    for src in SOURCES:
        sp = os.path.join(CSRC, src)
        obj = os.path.join(OBJDIR, src.replace(".cu", ".o"))
        objs.append(obj)
        if force or _newer([sp] + headers, obj):
            cmd = [NVCC, "-c", sp, "-o", obj + ".tmp"] + FLAGS
            if verbose:
                cmd += ["-Xptxas", "-v"]
                print(" ".join(cmd), flush=True)
            jobs.append((cmd, obj))

    def compile_one(job):
        cmd, obj = job
        subprocess.run(cmd, check=True)
        os.replace(obj + ".tmp", obj)

    # the translation units are independent: compile them side by side
    with ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as pool:
        for f in [pool.submit(compile_one, j) for j in jobs]:
            f.result()
    if force or _newer(objs, LIB):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run([NVCC, "-shared", "-o", tmp] + objs +
                       ["-gencode", "arch=compute_100a,code=sm_100a"], check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
