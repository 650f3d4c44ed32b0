"""ctypes loader of libstar.so and the raw C signatures of include/star.h.

Argument marshalling only: every step of the hot path runs in the CUDA
library. There is no fallback; a missing library raises.
"""
import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libstar.so")

STATUS = {
    0: "STAR_OK",
    1: "STAR_ERR_INVALID_ARG",
    2: "STAR_ERR_UNSUPPORTED",
    3: "STAR_ERR_CUDA",
    4: "STAR_ERR_DEVICE_TIMEOUT",
    5: "STAR_ERR_DEVICE_BOUNDS",
}

# every entry point include/star.h declares
EXPORTS = (
    "star_last_error",
    "star_version",
    "star_rope",
    "star_phase1_workspace_bytes",
    "star_phase1_encode",
    "star_phase1_ext_workspace_bytes",
    "star_phase1_encode_ext",
    "star_phase1_encode_rotated",
    "star_phase2_partial_ext",
    "star_lse_merge_ranks",
    "star_phase2_workspace_bytes",
    "star_phase2_partial",
    "star_phase2_decode_static",
    "star_phase2_decode_static_status",
    "star_phase2_attend",
    "star_lse_merge",
    "star_rmsnorm",
    "star_linear",
    "star_linear_rope",
    "star_linear_rope_workspace_bytes",
    "star_linear_kv_cache",
    "star_device_status",
    "star_debug_index",
    "star_debug_wait_probe",
)


class StarError(RuntimeError):
    def __init__(self, status, message):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{self.name}: {message}")


_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_D = ctypes.c_double
_I64P = ctypes.POINTER(ctypes.c_int64)
_IP = ctypes.POINTER(ctypes.c_int)


def load(path: str = LIB_PATH):
    """Load the library once; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"CUDA library {path} is missing: build it with "
                "`python -m block_sparse_long_rope_b200.build` (no CPU fallback exists)")
        lib = ctypes.CDLL(path)
        lib.star_last_error.restype = ctypes.c_char_p
        lib.star_last_error.argtypes = []
        lib.star_version.restype = ctypes.c_char_p
        lib.star_version.argtypes = []
        lib.star_rope.restype = _I
        lib.star_rope.argtypes = [_P, _I64P, _P, _I64P, _P, _I64, _I, _I, _I, _I, _D, _P]
        lib.star_phase1_workspace_bytes.restype = _SZ
        lib.star_phase1_workspace_bytes.argtypes = [_I, _I, _I, _I]
        lib.star_phase1_encode.restype = _I
        lib.star_phase1_encode.argtypes = [_P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                                           _I, _D, _P, _SZ, _P]
        lib.star_phase1_ext_workspace_bytes.restype = _SZ
        lib.star_phase1_ext_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I]
        lib.star_phase1_encode_ext.restype = _I
        lib.star_phase1_encode_ext.argtypes = [_P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I,
                                               _I, _P, _P, _I, _P, _P, _P, _I, _I, _D, _P, _SZ, _P]
        lib.star_phase1_encode_rotated.restype = _I
        lib.star_phase1_encode_rotated.argtypes = [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                                                   _I, _P, _SZ, _P]
        lib.star_linear_rope_workspace_bytes.restype = _SZ
        lib.star_linear_rope_workspace_bytes.argtypes = [_I, _I, _I]
        lib.star_linear_kv_cache.restype = _I
        lib.star_linear_kv_cache.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I64, _D, _I, _P,
                                             _SZ, _P]
        lib.star_linear_rope.restype = _I
        lib.star_linear_rope.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I64, _D, _I, _P,
                                         _SZ, _P]
        lib.star_phase2_partial_ext.restype = _I
        lib.star_phase2_partial_ext.argtypes = [_P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                                _P, _P, _IP, _I, _I, _I, _I, _D, _P, _SZ, _P]
        lib.star_lse_merge_ranks.restype = _I
        lib.star_lse_merge_ranks.argtypes = [_P, _P, _I, _IP, _I, _P, _P, _I, _I, _I, _I, _P]
        lib.star_rmsnorm.restype = _I
        lib.star_rmsnorm.argtypes = [_P, _P, _P, _I, _I, ctypes.c_float, _P]
        lib.star_linear.restype = _I
        lib.star_linear.argtypes = [_P, _P, _P, _I, _I, _I, _I, _P, _SZ, _P]
        lib.star_phase2_workspace_bytes.restype = _SZ
        lib.star_phase2_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I, _I]
        lib.star_phase2_partial.restype = _I
        lib.star_phase2_partial.argtypes = [_P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _P, _P, _IP,
                                            _I, _I, _I, _I, _D, _P, _SZ, _P]
        lib.star_phase2_decode_static.restype = _I
        lib.star_phase2_decode_static.argtypes = [_P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _P, _P,
                                                  _IP, _I, _I, _I, _I, _D, _P]
        lib.star_phase2_decode_static_status.restype = _I
        lib.star_phase2_decode_static_status.argtypes = [_P]
        lib.star_phase2_attend.restype = _I
        lib.star_phase2_attend.argtypes = [_P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P,
                                           _IP, _I, _I, _I, _I, _D, _P, _SZ, _P]
        lib.star_lse_merge.restype = _I
        lib.star_lse_merge.argtypes = [_P, _P, _I, _P, _P, _I, _I, _I, _I, _P]
        lib.star_device_status.restype = _I
        lib.star_device_status.argtypes = [_P, _P]
        lib.star_debug_wait_probe.restype = _I
        lib.star_debug_wait_probe.argtypes = [_P, _D, _P]
        lib.star_debug_index.restype = _I
        lib.star_debug_index.argtypes = [_I, _I, _I, _P, _P, _P, _P]
        _lib = lib
        return lib


def check(status: int):
    if status != 0:
        msg = load().star_last_error().decode(errors="replace")
        raise StarError(status, msg)
