"""Build libkv4.so (sm_100a) in-tree with nvcc.

    python -m compressed_kv_cache_kv4_b200.build [--force] [--verbose-ptxas]

Every translation unit is compiled for `-gencode arch=compute_100a,code=sm_100a`
and linked with the static CUDA runtime, so the library does not depend on
which libcudart another component of the process (torch) has loaded.
"""
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libkv4.so")
BUILD_DIR = os.path.join(ROOT, "_build")
SOURCES = ["kv4_api.cu", "kv4_append.cu", "kv4_decode.cu", "kv4_merge.cu", "kv_topk.cu", "kv4_noalloc.cu", "kv4_evict.cu", "smd_attn.cu", "kv4_masked.cu"]
HEADERS = ["kv4_common.cuh", "kv4_internal.h", "kv4_evict.h", "smd_attn.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc():
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "kv4.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force=False, verbose_ptxas=False):
    if not force and not _stale():
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    objs = []
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
                    "-I", os.path.join(ROOT, "include"), "-I", CSRC]
    if verbose_ptxas:
        flags += ["-Xptxas", "-v"]
    for src in SOURCES:
        obj = os.path.join(BUILD_DIR, src.replace(".cu", ".o"))
        subprocess.check_call([nvcc(), "-c", os.path.join(CSRC, src), "-o", obj] + flags)
        objs.append(obj)
    tmp = LIB + ".tmp%d" % os.getpid()
    subprocess.check_call([nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv))
