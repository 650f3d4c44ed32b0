"""ctypes front end of the fp64 C++ oracle (test infrastructure only).

Inputs are the bf16 tensors the method consumes, passed as their raw 16-bit
patterns so that the oracle sees exactly the values the device sees; every
result is float64. The arithmetic lives in star_oracle.cpp; this file only
marshals arrays.
"""
import ctypes
import threading

import numpy as np

from . import build_oracle

_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_I = ctypes.c_int64


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build_oracle.build())
            lib.orc_round_bf16.argtypes = [_P, _I]
            lib.orc_rope.argtypes = [_P, _I, _I, _I, _I, _P, ctypes.c_double, ctypes.c_int, _P]
            lib.orc_phase1_ranges.argtypes = [_I, _I, _I, _P, _P]
            lib.orc_phase1_rows.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                            ctypes.c_double, ctypes.c_int, _I, _P, _P, _P,
                                            _P, _P, _P]
            lib.orc_phase1_rows_sel.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I,
                                                ctypes.c_double, ctypes.c_int, _I, _P, _P, _P,
                                                _P, _P, _P]
            lib.orc_phase1_gather_rows.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _I,
                                                   _P, _P, _P, _I, ctypes.c_double, ctypes.c_int,
                                                   _I, _P, _P, _P, _P, _P, _P]
            lib.orc_phase2_rows.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                            _I, _I, ctypes.c_double, ctypes.c_int, _I, _P,
                                            _P, _P, _P, _P]
            lib.orc_global_rows.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                            _I, ctypes.c_double, ctypes.c_int, _I, _P, _P,
                                            _P, _P, _P]
            lib.orc_lse_merge.argtypes = [_P, _P, _I, _I, _I, _P, _P]
            for f in ("orc_round_bf16", "orc_rope", "orc_phase1_ranges", "orc_phase1_rows",
                      "orc_phase1_rows_sel", "orc_phase1_gather_rows",
                      "orc_phase2_rows", "orc_global_rows", "orc_lse_merge"):
                getattr(lib, f).restype = None
            _lib = lib
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def bf16_bits(x):
    """uint16 bit patterns of a bf16 tensor (torch) or of an existing uint16 array."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch

    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def round_bf16(x):
    """Round float64 values to bf16 (nearest, ties to even), returned as float64."""
    a = np.array(x, dtype=np.float64, copy=True, order="C")
    _load().orc_round_bf16(_ptr(a), a.size)
    return a


def rope(x, pos, theta, round_out=False):
    """RoPE of x[B,S,H,D] (bf16) at positions pos[S]; float64 result."""
    xb = bf16_bits(x)
    B, S, H, D = xb.shape
    p = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    assert p.shape == (S,)
    y = np.empty((B, S, H, D), dtype=np.float64)
    _load().orc_rope(_ptr(xb), B, S, H, D, _ptr(p), float(theta), int(bool(round_out)), _ptr(y))
    return y


def phase1_ranges(L, block_len, anchor_len):
    """Block id and visible ranges {anchor_lo, anchor_hi, own_lo, own_hi} per row."""
    blk = np.empty((L,), dtype=np.int64)
    rng = np.empty((L, 4), dtype=np.int64)
    _load().orc_phase1_ranges(L, block_len, anchor_len, _ptr(blk), _ptr(rng))
    return blk, rng


def phase1_rows(q, k, v, block_len, anchor_len, theta, qb, qh, qr, round_qk=True):
    """Phase-1 output and LSE for the listed (batch, head, row) queries."""
    qbits, kbits, vbits = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    B, L, Hq, D = qbits.shape
    Hkv = kbits.shape[2]
    qb = np.ascontiguousarray(qb, dtype=np.int64)
    qh = np.ascontiguousarray(qh, dtype=np.int64)
    qr = np.ascontiguousarray(qr, dtype=np.int64)
    nq = qb.size
    o = np.empty((nq, D), dtype=np.float64)
    lse = np.empty((nq,), dtype=np.float64)
    nvis = np.empty((nq,), dtype=np.int64)
    _load().orc_phase1_rows(_ptr(qbits), _ptr(kbits), _ptr(vbits), B, L, Hq, Hkv, D, block_len,
                            anchor_len, float(theta), int(bool(round_qk)), nq, _ptr(qb), _ptr(qh),
                            _ptr(qr), _ptr(o), _ptr(lse), _ptr(nvis))
    return o, lse, nvis


def phase1_rows_selected(q_sel, k, v, block_len, anchor_len, theta, qb, qh, qr, Hq,
                         round_qk=True):
    """As phase1_rows, with q_sel[nq, D] (bf16) holding only the listed queries'
    pre-RoPE vectors (for contexts too long to copy Q to the host whole)."""
    qbits, kbits, vbits = bf16_bits(q_sel), bf16_bits(k), bf16_bits(v)
    B, L, Hkv, D = kbits.shape
    qb = np.ascontiguousarray(qb, dtype=np.int64)
    qh = np.ascontiguousarray(qh, dtype=np.int64)
    qr = np.ascontiguousarray(qr, dtype=np.int64)
    nq = qb.size
    assert qbits.shape == (nq, D)
    o = np.empty((nq, D), dtype=np.float64)
    lse = np.empty((nq,), dtype=np.float64)
    nvis = np.empty((nq,), dtype=np.int64)
    _load().orc_phase1_rows_sel(_ptr(qbits), _ptr(kbits), _ptr(vbits), L, Hq, Hkv, D, block_len,
                                anchor_len, float(theta), int(bool(round_qk)), nq, _ptr(qb),
                                _ptr(qh), _ptr(qr), _ptr(o), _ptr(lse), _ptr(nvis))
    return o, lse, nvis


def phase1_gather_rows(q, k, v, block_len, src, pos, bounds, theta, qb, qh, qr, extra_k=None,
                       extra_v=None, round_qk=True):
    """Generalised Phase 1 for the listed queries. The prefix table has G
    rows: row t is context row src[t] (src >= 0) or extra row -1 - src[t]
    (extra_k/v [B, NX, Hkv, D] bf16), its key rotated at pos[t]; block i sees
    table rows [bounds[i, 0], bounds[i, 1]) and, causally, itself."""
    qbits, kbits, vbits = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    B, L, Hq, D = qbits.shape
    Hkv = kbits.shape[2]
    n = -(-L // block_len)
    src = np.ascontiguousarray(np.asarray(src, dtype=np.int64).reshape(-1))
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(-1))
    G = src.size
    assert pos.shape == (G,)
    bnd = np.ascontiguousarray(np.asarray(bounds, dtype=np.int64))
    assert bnd.shape == (n, 2)
    assert ((0 <= bnd) & (bnd <= G)).all()
    if extra_k is None:
        xk = np.zeros((1,), dtype=np.uint16)
        xv = xk
        NX = 0
    else:
        xk, xv = bf16_bits(extra_k), bf16_bits(extra_v)
        NX = xk.shape[1]
    assert ((src < L) & (src >= -NX)).all()
    qb = np.ascontiguousarray(qb, dtype=np.int64)
    qh = np.ascontiguousarray(qh, dtype=np.int64)
    qr = np.ascontiguousarray(qr, dtype=np.int64)
    nq = qb.size
    o = np.empty((nq, D), dtype=np.float64)
    lse = np.empty((nq,), dtype=np.float64)
    nvis = np.empty((nq,), dtype=np.int64)
    _load().orc_phase1_gather_rows(_ptr(qbits), _ptr(kbits), _ptr(vbits), L, Hq, Hkv, D,
                                   block_len, _ptr(src), _ptr(pos), G, _ptr(bnd), _ptr(xk),
                                   _ptr(xv), NX, float(theta), int(bool(round_qk)), nq, _ptr(qb),
                                   _ptr(qh), _ptr(qr), _ptr(o), _ptr(lse), _ptr(nvis))
    return o, lse, nvis


def phase1_full(q, k, v, block_len, anchor_len, theta, round_qk=True):
    """Phase 1 over every row: o[B,L,Hq,D], lse[B,Hq,L] (float64)."""
    qbits = bf16_bits(q)
    B, L, Hq, D = qbits.shape
    bb, hh, rr = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(L), indexing="ij")
    o, lse, _ = phase1_rows(qbits, k, v, block_len, anchor_len, theta, bb.ravel(), hh.ravel(),
                            rr.ravel(), round_qk)
    o = o.reshape(B, Hq, L, D).transpose(0, 2, 1, 3).copy()
    return o, lse.reshape(B, Hq, L)


def phase2_rows(qn, kc, vc, kt, vt, block_len, tail_len, theta, qb, qh, qt, round_qk=True):
    """Per-split partials for new tokens: part_o[nq, n+1, D], part_lse[nq, n+1]."""
    qbits, kcb, vcb, ktb, vtb = (bf16_bits(t) for t in (qn, kc, vc, kt, vt))
    B, T, Hq, D = qbits.shape
    L = kcb.shape[1]
    Hkv = kcb.shape[2]
    Ltail = ktb.shape[1]
    assert Ltail >= tail_len + T
    n = (L + block_len - 1) // block_len
    qb = np.ascontiguousarray(qb, dtype=np.int64)
    qh = np.ascontiguousarray(qh, dtype=np.int64)
    qt = np.ascontiguousarray(qt, dtype=np.int64)
    nq = qb.size
    po = np.empty((nq, n + 1, D), dtype=np.float64)
    pl = np.empty((nq, n + 1), dtype=np.float64)
    _load().orc_phase2_rows(_ptr(qbits), _ptr(kcb), _ptr(vcb), _ptr(ktb), _ptr(vtb), B, L, Ltail,
                            T, Hq, Hkv, D, block_len, tail_len, float(theta), int(bool(round_qk)),
                            nq, _ptr(qb), _ptr(qh), _ptr(qt), _ptr(po), _ptr(pl))
    return po, pl


def global_rows(qn, kc, vc, kt, vt, tail_len, theta, qb, qh, qt, round_qk=True):
    """One-shot softmax attention of new tokens over every cached key."""
    qbits, kcb, vcb, ktb, vtb = (bf16_bits(t) for t in (qn, kc, vc, kt, vt))
    B, T, Hq, D = qbits.shape
    L = kcb.shape[1]
    Hkv = kcb.shape[2]
    Ltail = ktb.shape[1]
    qb = np.ascontiguousarray(qb, dtype=np.int64)
    qh = np.ascontiguousarray(qh, dtype=np.int64)
    qt = np.ascontiguousarray(qt, dtype=np.int64)
    nq = qb.size
    o = np.empty((nq, D), dtype=np.float64)
    lse = np.empty((nq,), dtype=np.float64)
    _load().orc_global_rows(_ptr(qbits), _ptr(kcb), _ptr(vcb), _ptr(ktb), _ptr(vtb), B, L, Ltail,
                            T, Hq, Hkv, D, tail_len, float(theta), int(bool(round_qk)), nq,
                            _ptr(qb), _ptr(qh), _ptr(qt), _ptr(o), _ptr(lse))
    return o, lse


def lse_merge(part_o, part_lse):
    """Exact merge of per-split (o, lse): part_o[R, S, D], part_lse[R, S] -> o[R, D], lse[R]."""
    po = np.ascontiguousarray(part_o, dtype=np.float64)
    pl = np.ascontiguousarray(part_lse, dtype=np.float64)
    R, S, D = po.shape
    o = np.empty((R, D), dtype=np.float64)
    lse = np.empty((R,), dtype=np.float64)
    _load().orc_lse_merge(_ptr(po), _ptr(pl), R, S, D, _ptr(o), _ptr(lse))
    return o, lse
