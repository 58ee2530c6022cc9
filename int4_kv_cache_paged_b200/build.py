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


def up_to_date(obj, deps, same_flags):
    """An object can be reused when it was compiled with the current flags after its last dependency changed."""
    return same_flags and os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(d) for d in deps)


def build(verbose_ptxas=False, force=False):
    """Compile every source to an object in _build/ and link libkv4.so next to this file."""
    os.makedirs(OBJDIR, exist_ok=True)
    objs = []
    # every header a source can include: an edit to any of them rebuilds every object
    headers = [os.path.join(HERE, "csrc", h) for h in sorted(os.listdir(os.path.join(HERE, "csrc")))
               if h.endswith((".cuh", ".h"))] + \
        [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include")))
         if h.endswith(".h")]
    # the flags the objects were compiled with (a self-checking build and a normal one share _build/)
    stamp = os.path.join(OBJDIR, "flags")
    f = flags()
    want = " ".join(x for i, x in enumerate(f) if x != "-I" and (i == 0 or f[i - 1] != "-I"))   # paths aside
    try:
        with open(stamp) as f:
            same_flags = f.read() == want
    except OSError:
        same_flags = False
    if not same_flags and os.path.exists(stamp):
        os.remove(stamp)
    for src in SOURCES:
        path = os.path.join(HERE, "csrc", src)
        obj = os.path.join(OBJDIR, src.replace(".cu", ".o"))
        objs.append(obj)
        if not force and not verbose_ptxas and up_to_date(obj, [path] + headers, same_flags):
            continue
        cmd = [nvcc()] + flags(verbose_ptxas) + ["-c", path, "-o", obj]
        subprocess.run(cmd, check=True)
    with open(stamp, "w") as f:
        f.write(want)
    cmd = [nvcc(), "-shared", "-cudart", "static", "-gencode", "arch=compute_100a,code=sm_100a", "-o", LIB] + objs
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose_ptxas="--verbose-ptxas" in sys.argv, force="--force" in sys.argv)
    print(LIB)
