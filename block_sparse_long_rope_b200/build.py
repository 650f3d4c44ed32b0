"""Build libstar.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m block_sparse_long_rope_b200.build [--force] [--verbose-ptxas]
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libstar.so")
OBJ_DIR = os.path.join(HERE, "_build")

SOURCES = ["api.cu", "rope.cu", "lse_merge.cu", "phase2_decode.cu", "phase1_sm100.cu", "noalloc.cu",
           "stack.cu"]
HEADERS = ["star_common.cuh", "star_index.cuh", "star_kernels.cuh", "rope_math.cuh", "star_plan.h"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I" + INCLUDE, "-I" + CSRC]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    os.makedirs(OBJ_DIR, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "star.h")]
    objs = []
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(OBJ_DIR, src.replace(".cu", ".o"))
        objs.append(obj)
        if force or verbose_ptxas or _stale(obj, [path] + hdrs):
            cmd = [NVCC] + ARCH + FLAGS + extra + ["-c", path, "-o", obj]
            subprocess.check_call(cmd)
    if force or _stale(LIB, objs):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [NVCC] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-o", tmp] + objs + ["-lcublasLt"]
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv))
