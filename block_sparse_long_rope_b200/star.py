"""Python binding of the C ABI (include/star.h), same names, torch tensors in.

Only argument marshalling happens here: pointers, sizes and the current CUDA
stream are passed to libstar.so, which validates and launches. PyTorch serves
for device memory and streams.
"""
import ctypes

import torch

from . import _abi


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _bf16(t, name):
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")


def _i64x3(vals):
    return (ctypes.c_int64 * 3)(*[int(v) for v in vals])


def version() -> str:
    return _abi.load().star_version().decode()


def star_rope(x, y, theta, pos=None, pos0=0, stream=None):
    """y[b,s,h,:] = RoPE(x[b,s,h,:]) at position pos[s] (or pos0 + s).
    x, y: bf16 [B, S, H, D] views (any strides with D contiguous)."""
    _bf16(x, "x")
    _bf16(y, "y")
    B, S, H, D = x.shape
    if tuple(y.shape) != (B, S, H, D):
        raise ValueError("x and y shapes differ")
    if x.stride(3) != 1 or y.stride(3) != 1:
        raise ValueError("head_dim must be contiguous")
    if pos is not None and pos.dtype != torch.int32:
        raise TypeError("pos must be int32")
    lib = _abi.load()
    _abi.check(lib.star_rope(_ptr(x), _i64x3(x.stride()[:3]), _ptr(y), _i64x3(y.stride()[:3]),
                             _ptr(pos), int(pos0), B, S, H, D, float(theta), _stream(stream)))
    return y


def star_phase1_workspace_bytes(B, L, Hq, D) -> int:
    return int(_abi.load().star_phase1_workspace_bytes(B, L, Hq, D))


def star_phase1_encode(q, k, v, o, k_cache, v_cache, block_len, anchor_len, theta, workspace,
                       lse=None, stream=None):
    """Phase 1: q[B,L,Hq,D], k/v[B,L,Hkv,D] (pre-RoPE bf16) -> o[B,L,Hq,D] bf16,
    cache rows [0,L) of k_cache/v_cache[B,Hkv,Lcap,D], lse[B,Hq,L] fp32 (optional)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _bf16(t, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    Lcap = k_cache.shape[2]
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous()):
        raise ValueError("lse must be contiguous float32")
    lib = _abi.load()
    _abi.check(lib.star_phase1_encode(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(k_cache), _ptr(v_cache), Lcap, _ptr(lse), B, L,
        Hq, Hkv, D, int(block_len), int(anchor_len), float(theta), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return o


def star_phase1_ext_workspace_bytes(B, L, Hq, Hkv, D, G=0) -> int:
    return int(_abi.load().star_phase1_ext_workspace_bytes(B, L, Hq, Hkv, D, G))


def _i32(t, name):
    if t is None:
        return
    if t.dtype != torch.int32 or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name} must be a contiguous int32 CUDA tensor")


def star_phase1_encode_ext(q, k, v, o, k_cache, v_cache, block_len, theta, workspace,
                           prefix_src=None, prefix_pos=None, prefix_bounds=None, extra_k=None,
                           extra_v=None, lse=None, ctx_pos0=0, stream=None):
    """Phase 1 with a gathered prefix table: row g is context row
    prefix_src[g] (>= 0) or row -1 - prefix_src[g] of extra_k/extra_v
    [B, NX, Hkv, D], its key rotated at prefix_pos[g]; block i sees table
    rows prefix_bounds[i, 0] .. prefix_bounds[i, 1] - 1 (int32 [n, 2])."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _bf16(t, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    Lcap = k_cache.shape[2]
    for t, n in ((prefix_src, "prefix_src"), (prefix_pos, "prefix_pos"),
                 (prefix_bounds, "prefix_bounds")):
        _i32(t, n)
    G = 0 if prefix_src is None else prefix_src.numel()
    if prefix_pos is not None and prefix_pos.numel() != G:
        raise ValueError("prefix_pos must have as many entries as prefix_src")
    NX = 0
    if extra_k is not None:
        _bf16(extra_k, "extra_k")
        _bf16(extra_v, "extra_v")
        NX = extra_k.shape[1]
    lib = _abi.load()
    _abi.check(lib.star_phase1_encode_ext(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(k_cache), _ptr(v_cache), Lcap, _ptr(lse), B, L,
        Hq, Hkv, D, int(block_len), _ptr(prefix_src), _ptr(prefix_pos), G, _ptr(prefix_bounds),
        _ptr(extra_k), _ptr(extra_v), NX, int(ctx_pos0), float(theta), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return o


def star_phase2_workspace_bytes(B, T, Hq, Hkv, D, Lcap, block_len) -> int:
    return int(_abi.load().star_phase2_workspace_bytes(B, T, Hq, Hkv, D, Lcap, block_len))


def star_phase2_partial(q, k, v, k_cache, v_cache, L, block_len, tail_len, part_o, part_lse,
                        theta, workspace, stream=None):
    """Phase 2 partials for T new tokens (q[B,T,Hq,D], k/v[B,T,Hkv,D] pre-RoPE)
    at positions L + tail_len + t. Appends k/v to the cache; writes
    part_o[B,Hq,n+1,T,D], part_lse[B,Hq,n+1,T]. Returns nsplit = n + 1."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _bf16(t, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    Lcap = k_cache.shape[2]
    ns = ctypes.c_int(0)
    lib = _abi.load()
    _abi.check(lib.star_phase2_partial(
        _ptr(q), _ptr(k), _ptr(v), T, _ptr(k_cache), _ptr(v_cache), Lcap, int(L), int(block_len),
        int(tail_len), _ptr(part_o), _ptr(part_lse), ctypes.byref(ns), B, Hq, Hkv, D,
        float(theta), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return ns.value


def star_phase2_partial_ext(q, k, v, k_cache, v_cache, L, block_len, tail_len, ctx_pos0, q_pos0,
                            with_tail, part_o, part_lse, theta, workspace, stream=None):
    """Phase-2 partials of one shard: cache row r at position ctx_pos0 + r,
    new token t at q_pos0 + t. with_tail: append k/v and add the tail split
    (q_pos0 must be ctx_pos0 + L + tail_len); otherwise context splits only
    (k, v may be None). Returns nsplit."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")) + \
            (((k, "k"), (v, "v")) if with_tail else ()):
        _bf16(t, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    B, T, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    Lcap = k_cache.shape[2]
    ns = ctypes.c_int(0)
    lib = _abi.load()
    _abi.check(lib.star_phase2_partial_ext(
        _ptr(q), _ptr(k if with_tail else None), _ptr(v if with_tail else None), T, _ptr(k_cache),
        _ptr(v_cache), Lcap, int(L), int(block_len), int(tail_len), int(ctx_pos0), int(q_pos0),
        1 if with_tail else 0, _ptr(part_o), _ptr(part_lse), ctypes.byref(ns), B, Hq, Hkv, D,
        float(theta), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return ns.value


def star_phase2_attend(q, k, v, k_cache, v_cache, L, block_len, tail_len, part_o, part_lse, o,
                       theta, workspace, lse=None, stream=None):
    """star_phase2_partial plus the exact merge in one call: writes the
    partials and o[B,T,Hq,D] bf16 / lse[B,Hq,T] (optional). Returns nsplit."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (k_cache, "k_cache"), (v_cache, "v_cache"), (o, "o")):
        _bf16(t, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    Lcap = k_cache.shape[2]
    ns = ctypes.c_int(0)
    lib = _abi.load()
    _abi.check(lib.star_phase2_attend(
        _ptr(q), _ptr(k), _ptr(v), T, _ptr(k_cache), _ptr(v_cache), Lcap, int(L), int(block_len),
        int(tail_len), _ptr(part_o), _ptr(part_lse), _ptr(o), _ptr(lse), ctypes.byref(ns), B, Hq,
        Hkv, D, float(theta), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return ns.value


def star_phase2_decode_static(q, k, v, k_cache, v_cache, L, block_len, tail_len, part_o,
                              part_lse, theta, stream=None):
    """star_phase2_partial for decode steps without a workspace: the scratch
    lives in the library's fixed 16 MiB device array (see include/star.h)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _bf16(t, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    Lcap = k_cache.shape[2]
    ns = ctypes.c_int(0)
    lib = _abi.load()
    _abi.check(lib.star_phase2_decode_static(
        _ptr(q), _ptr(k), _ptr(v), T, _ptr(k_cache), _ptr(v_cache), Lcap, int(L), int(block_len),
        int(tail_len), _ptr(part_o), _ptr(part_lse), ctypes.byref(ns), B, Hq, Hkv, D,
        float(theta), _stream(stream)))
    return ns.value


def star_phase2_decode_static_status(stream=None):
    """Reads and clears the device-error word of star_phase2_decode_static
    (synchronises the stream); raises StarError on a device error."""
    _abi.check(_abi.load().star_phase2_decode_static_status(_stream(stream)))


def star_lse_merge(part_o, part_lse, o, lse=None, stream=None):
    """Exact merge: part_o[B,Hq,S,T,D], part_lse[B,Hq,S,T] -> o[B,T,Hq,D] bf16, lse[B,Hq,T]."""
    B, Hq, S, T, D = part_o.shape
    _bf16(o, "o")
    lib = _abi.load()
    _abi.check(lib.star_lse_merge(_ptr(part_o), _ptr(part_lse), S, _ptr(o), _ptr(lse), B, T, Hq,
                                  D, _stream(stream)))
    return o


def star_lse_merge_ranks(part_o, part_lse, nsplit_of_rank, slots, o, lse=None, stream=None):
    """Merge partials gathered from ranks: part_o / part_lse hold one slot of
    B*Hq*slots*T*D / B*Hq*slots*T floats per rank, rank r's slot beginning
    with its [B, Hq, nsplit_of_rank[r], T, (D)] partials -> o[B,T,Hq,D]
    bf16, lse[B,Hq,T]."""
    B, T, Hq, D = o.shape
    R = len(nsplit_of_rank)
    S = int(slots)
    if part_o.numel() < R * B * Hq * S * T * D or part_lse.numel() < R * B * Hq * S * T:
        raise ValueError("gathered buffers smaller than nranks slots")
    _bf16(o, "o")
    ns = (ctypes.c_int * R)(*[int(x) for x in nsplit_of_rank])
    lib = _abi.load()
    _abi.check(lib.star_lse_merge_ranks(_ptr(part_o), _ptr(part_lse), R, ns, S, _ptr(o), _ptr(lse),
                                        B, T, Hq, D, _stream(stream)))
    return o


def star_rmsnorm(x, gamma, y, eps=1e-5, stream=None):
    """y = x / rms(x) * gamma over the last dim (bf16 [..., dm])."""
    for t, n in ((x, "x"), (gamma, "gamma"), (y, "y")):
        _bf16(t, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    dm = x.shape[-1]
    lib = _abi.load()
    _abi.check(lib.star_rmsnorm(_ptr(x), _ptr(gamma), _ptr(y), x.numel() // dm, dm, float(eps),
                                _stream(stream)))
    return y


def star_linear(x, w, y, accumulate=False, workspace=None, stream=None):
    """y[M, N] = x[M, K] w[N, K]^T (+ y when accumulate), bf16 row-major."""
    for t, n in ((x, "x"), (w, "w"), (y, "y")):
        _bf16(t, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    N, K = w.shape
    M = x.numel() // K
    if y.numel() != M * N:
        raise ValueError("y must hold M x N elements")
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    lib = _abi.load()
    _abi.check(lib.star_linear(_ptr(x), _ptr(w), _ptr(y), M, N, K, 1 if accumulate else 0,
                               _ptr(workspace), wsb, _stream(stream)))
    return y


def star_linear_rope(x, w, y, head_dim, rotate, seq_len, pos0, theta, cache_rows, workspace,
                     stream=None):
    """A projection p = bf16(x[M, K] w[N, K]^T) whose heads of head_dim
    columns are RoPE'd (rotate) at positions pos0 + row % seq_len and/or
    stored head-major into a KV cache [M / seq_len, N / head_dim,
    cache_rows, head_dim] (cache_rows > 0); y row-major [M, N] otherwise."""
    for t, n in ((x, "x"), (w, "w"), (y, "y")):
        _bf16(t, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    N, K = w.shape
    M = x.numel() // K
    lib = _abi.load()
    _abi.check(lib.star_linear_rope(_ptr(x), _ptr(w), _ptr(y), M, N, K, int(head_dim),
                                    1 if rotate else 0, int(seq_len), int(pos0), float(theta),
                                    int(cache_rows), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)))
    return y


def star_linear_kv_cache(x, w_kv, k_cache, v_cache, seq_len, pos0, theta, workspace,
                         stream=None):
    """A layer's K and V projections in one GEMM (w_kv = [Wk; Wv], [2N, K]):
    rotated keys into k_cache, values into v_cache (head-major [B, Hkv,
    cache_rows, D]), token t of each sequence in cache row t."""
    for t, n in ((x, "x"), (w_kv, "w_kv"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _bf16(t, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    N2, K = w_kv.shape
    M = x.numel() // K
    D, rows = k_cache.shape[3], k_cache.shape[2]
    lib = _abi.load()
    _abi.check(lib.star_linear_kv_cache(_ptr(x), _ptr(w_kv), _ptr(k_cache), _ptr(v_cache), M,
                                        N2 // 2, K, D, int(seq_len), int(pos0), float(theta),
                                        rows, _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)))


def star_linear_rope_workspace_bytes(seq_len, head_dim, rotate) -> int:
    return int(_abi.load().star_linear_rope_workspace_bytes(int(seq_len), int(head_dim),
                                                            1 if rotate else 0))


def star_phase1_encode_rotated(q_rot, o, k_cache, v_cache, L, block_len, anchor_len, workspace,
                               lse=None, stream=None):
    """Phase 1 attention when q_rot[B,L,Hq,D] is already rotated and cache rows
    [0, L) hold the rotated keys and the values (see star_linear_rope)."""
    for t, n in ((q_rot, "q_rot"), (o, "o"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _bf16(t, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    B, Lq, Hq, D = q_rot.shape
    Hkv, Lcap = k_cache.shape[1], k_cache.shape[2]
    lib = _abi.load()
    _abi.check(lib.star_phase1_encode_rotated(
        _ptr(q_rot), _ptr(o), _ptr(k_cache), _ptr(v_cache), Lcap, _ptr(lse), B, int(L), Hq, Hkv,
        D, int(block_len), int(anchor_len), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return o


def star_device_status(workspace, stream=None):
    """Synchronise, read and clear the device status word; raises on a device error."""
    lib = _abi.load()
    _abi.check(lib.star_device_status(_ptr(workspace), _stream(stream)))


def star_debug_wait_probe(workspace, seconds=0.05, stream=None):
    """Make a kernel's bounded wait run out on purpose (no fault): the
    following star_device_status raises STAR_ERR_DEVICE_TIMEOUT."""
    lib = _abi.load()
    _abi.check(lib.star_debug_wait_probe(_ptr(workspace), float(seconds), _stream(stream)))


def star_debug_index(L, block_len, anchor_len, device="cuda", stream=None):
    """Device-evaluated index math: (blk[L], pos[L], kv_ranges[L,4]) int32."""
    blk = torch.empty(L, dtype=torch.int32, device=device)
    pos = torch.empty(L, dtype=torch.int32, device=device)
    rng = torch.empty((L, 4), dtype=torch.int32, device=device)
    lib = _abi.load()
    _abi.check(lib.star_debug_index(L, block_len, anchor_len, _ptr(blk), _ptr(pos), _ptr(rng),
                                    _stream(stream)))
    return blk, pos, rng


def alloc_workspace(nbytes, device="cuda"):
    """A caller-owned, zero-filled workspace (the library itself allocates
    nothing; a workspace must be zero before its first use)."""
    n = max(256, (int(nbytes) + 255) // 256 * 256)
    return torch.zeros(n, dtype=torch.uint8, device=device)
