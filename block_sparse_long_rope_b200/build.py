"""Build libstar.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m block_sparse_long_rope_b200.build [--force] [--verbose-ptxas]

Objects are rebuilt when the sources they come from change, judged by
content, not by file times: every object keeps beside it the sha256 of its
source, every header, the compiler flags and the nvcc version it was built
from, and the library keeps the digest of all of them. A tree copied with
stale objects (or objects built from other sources) is therefore rebuilt. The
library's star_version() string ends with that digest, so a process can check
that the library it loaded was built from the sources in this tree
(`loaded_matches_sources`).
"""
import hashlib
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
           "stack.cu", "gemm_sm100.cu"]
HEADERS = ["star_common.cuh", "star_index.cuh", "star_kernels.cuh", "rope_math.cuh", "star_plan.h"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I" + INCLUDE, "-I" + CSRC]
LINK = []


def _sha(paths, extra=()):
    h = hashlib.sha256()
    for p in paths:
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    for x in extra:
        h.update(str(x).encode())
    return h.hexdigest()


_NVCC_VERSION = None


def _nvcc_version():
    global _NVCC_VERSION
    if _NVCC_VERSION is None:
        try:
            _NVCC_VERSION = subprocess.check_output([NVCC, "--version"], text=True)
        except (OSError, subprocess.CalledProcessError):
            _NVCC_VERSION = "unknown"
    return _NVCC_VERSION


def _header_paths():
    return [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "star.h")]


def source_digest() -> str:
    """Digest of every source, header and build flag of the library (first 16
    hex digits); the library built from them reports it in star_version()."""
    paths = [os.path.join(CSRC, s) for s in SOURCES] + _header_paths()
    return _sha(paths, ARCH + FLAGS + LINK + [_nvcc_version()])[:16]


def _read(path):
    try:
        with open(path) as f:
            return f.read().strip()
    except OSError:
        return None


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    os.makedirs(OBJ_DIR, exist_ok=True)
    hdrs = _header_paths()
    digest = source_digest()
    objs = []
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(OBJ_DIR, src.replace(".cu", ".o"))
        objs.append(obj)
        defs = [f"-DSTAR_BUILD_DIGEST=\"{digest}\""] if src == "api.cu" else []
        want = _sha([path] + hdrs, ARCH + FLAGS + defs + [_nvcc_version()])
        stamp = obj + ".sha256"
        if force or verbose_ptxas or not os.path.exists(obj) or _read(stamp) != want:
            cmd = [NVCC] + ARCH + FLAGS + defs + extra + ["-c", path, "-o", obj]
            subprocess.check_call(cmd)
            with open(stamp, "w") as f:
                f.write(want)
    lib_stamp = LIB + ".sha256"
    if force or not os.path.exists(LIB) or _read(lib_stamp) != digest:
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [NVCC] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-o", tmp] + objs + LINK
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
        with open(lib_stamp, "w") as f:
            f.write(digest)
    return LIB


def loaded_matches_sources() -> bool:
    """True when the loaded libstar.so reports the digest of this tree's sources."""
    from . import _abi

    ver = _abi.load().star_version().decode()
    return ver.endswith(source_digest())


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv))
