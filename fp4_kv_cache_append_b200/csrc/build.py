"""Build libcsa2.so (sm_100a) in-tree with nvcc.

    python -m fp4_kv_cache_append_b200.csrc.build [--verbose-ptxas]

Objects go to _build/ at the repository root; the shared library to
fp4_kv_cache_append_b200/lib/libcsa2.so.  The CUDA runtime is linked
statically, so loading the library needs no libcudart on the path (and works
on a machine without a GPU, for symbol checks).
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
OBJ = os.path.join(ROOT, "_build", "csa2")
LIB = os.path.join(PKG, "lib", "libcsa2.so")
SOURCES = ["api.cu", "append.cu", "project.cu", "index.cu", "topk.cu", "topk_cluster.cu", "topk_bmax.cu", "attn.cu", "attn_lat.cu", "shard.cu", "noalloc.cu"]
HEADERS = ["common.cuh", "kernels.h", os.path.join("..", "..", "include", "csa2.h")]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr"]


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose_ptxas: bool = False, force: bool = False) -> str:
    os.makedirs(OBJ, exist_ok=True)
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    hdrs = [os.path.join(HERE, h) for h in HEADERS]
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []

    def compile_one(src: str) -> str:
        s = os.path.join(HERE, src)
        o = os.path.join(OBJ, src.replace(".cu", ".o"))
        if force or verbose_ptxas or _stale(o, [s] + hdrs):
            r = subprocess.run([nvcc(), *FLAGS, *extra, "-c", s, "-o", o], capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr}")
            if verbose_ptxas:
                sys.stderr.write(r.stderr)
        return o

    with cf.ThreadPoolExecutor(len(SOURCES)) as ex:
        objs = list(ex.map(compile_one, SOURCES))
    if force or _stale(LIB, objs):
        tmp = LIB + f".tmp{os.getpid()}"
        r = subprocess.run([nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp, *objs],
                           capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr}")
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose_ptxas="--verbose-ptxas" in sys.argv, force="--force" in sys.argv))
