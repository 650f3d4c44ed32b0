"""Star Attention hot path for NVIDIA B200 (sm_100a).

The compute lives in libstar.so (C ABI in include/star.h); `star` is its thin
torch binding and `pipeline` strings the four calls into one Star Attention
layer step. Nothing here loads the library until a call needs it.
"""
__all__ = ["star", "pipeline", "configs", "inputs"]
