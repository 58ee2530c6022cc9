"""Build libkv4.so in-tree with nvcc for sm_100a.

Usage: python int4_kv_cache_paged_b200/build.py [--verbose-ptxas] [--force]
(runs as a script: the package itself needs the built library to import)
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCES = ["kv4_api.cu", "kv4_append.cu", "kv4_attention.cu", "kv4_attention_grouped.cu", "kv4_noalloc.cu"]
LIB = os.path.join(HERE, "libkv4.so")
OBJDIR = os.path.join(ROOT, "_build")


def nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def flags(verbose_ptxas=False):
    f = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"), "-I", os.path.join(HERE, "csrc")]
    if verbose_ptxas:
        f += ["-Xptxas", "-v"]
    if os.environ.get("KV4_DEBUG_CHECKS") == "1":
        f += ["-DKV4_DEBUG_CHECKS"]   # self-checking kernels: bad accesses are recorded and skipped
    return f


def build(verbose_ptxas=False, force=False):
    """Compile every source to an object in _build/ and link libkv4.so next to this file."""
    os.makedirs(OBJDIR, exist_ok=True)
    objs = []
    # every header a source can include: an edit to any of them rebuilds every object
    headers = [os.path.join(HERE, "csrc", h) for h in sorted(os.listdir(os.path.join(HERE, "csrc")))
               if h.endswith((".cuh", ".h"))] + \
        [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include")))
         if h.endswith(".h")]
    newest_header = max(os.path.getmtime(h) for h in headers)
    for src in SOURCES:
        path = os.path.join(HERE, "csrc", src)
        obj = os.path.join(OBJDIR, src.replace(".cu", ".o"))
        objs.append(obj)
        if (not force and os.environ.get("KV4_DEBUG_CHECKS") != "1" and os.path.exists(obj) and os.path.getmtime(obj) >= os.path.getmtime(path)
                and os.path.getmtime(obj) >= newest_header and not verbose_ptxas):
            continue
        cmd = [nvcc()] + flags(verbose_ptxas) + ["-c", path, "-o", obj]
        subprocess.run(cmd, check=True)
    cmd = [nvcc(), "-shared", "-cudart", "static", "-gencode", "arch=compute_100a,code=sm_100a", "-o", LIB] + objs
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose_ptxas="--verbose-ptxas" in sys.argv, force="--force" in sys.argv)
    print(LIB)
