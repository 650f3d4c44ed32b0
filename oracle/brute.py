"""Brute-force NumPy fp64 checkers for tiny inputs (test infrastructure only).

Written independently of star_oracle.cpp, in a different formulation, so
that agreement pins the oracle:
  * RoPE as complex multiplication of the pair (x_i, x_{i+D/2}) by
    exp(i * p * theta_i);
  * Phase 1 through a dense L x L boolean mask built from the pages' wording
    ([pith 2WVXFXZ2, "What carries the argument"]: block i >= 2 sees the
    anchor c1 and, causally, itself; c'_1 = c1 per the minor comment on
    Section 2.1);
  * Phase 1 "literally": materialise the augmented block [c1 || c_i] as a new
    sequence (copies of the anchor rows at their original positions), run
    plain causal attention on it and keep the c_i rows.
"""
import numpy as np


def bits_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rope_complex(x, pos, theta):
    """x[..., S, H, D] float64, pos[S] -> rotated copy (complex-multiply form)."""
    D = x.shape[-1]
    h = D // 2
    freq = theta ** (-2.0 * np.arange(h) / D)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * freq[None, :]  # [S, h]
    rot = np.exp(1j * ang)[:, None, :]  # broadcast over heads
    z = (x[..., :h] + 1j * x[..., h:]) * rot
    return np.concatenate([z.real, z.imag], axis=-1)


def phase1_mask(L, b, a):
    """Dense mask M[r, c] = True iff context row r sees key c in Phase 1."""
    M = np.zeros((L, L), dtype=bool)
    for r in range(L):
        i = r // b
        if i == 0:
            M[r, : r + 1] = True
        else:
            M[r, :a] = True
            M[r, i * b : r + 1] = True
    return M


def masked_attention(q, k, v, mask):
    """q[Lq,D], k/v[Lk,D], mask[Lq,Lk] -> o[Lq,D], lse[Lq] (scale 1/sqrt(D))."""
    D = q.shape[-1]
    s = (q @ k.T) / np.sqrt(D)
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    w = np.exp(s - m)
    z = w.sum(axis=1, keepdims=True)
    return (w @ v) / z, (m + np.log(z))[:, 0]


def phase1_dense(qr, kr, v, b, a):
    """qr[L,Hq,D] (rotated), kr/v[L,Hkv,D] -> o[L,Hq,D], lse[Hq,L] via the dense mask."""
    L, Hq, D = qr.shape
    Hkv = kr.shape[1]
    g = Hq // Hkv
    M = phase1_mask(L, b, a)
    o = np.empty_like(qr)
    lse = np.empty((Hq, L))
    for h in range(Hq):
        o[:, h], lse[h] = masked_attention(qr[:, h], kr[:, h // g], v[:, h // g], M)
    return o, lse


def phase1_literal(q, k, v, b, a, theta):
    """Augmented-block form: for block i >= 1 build [c1[:a] || c_i] with the
    anchor's original positions, rotate, run causal attention, keep c_i rows.
    q[L,Hq,D], k/v[L,Hkv,D] are pre-RoPE float64."""
    L, Hq, D = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    o = np.empty_like(q)
    lse = np.empty((Hq, L))
    n = -(-L // b)
    for i in range(n):
        own = np.arange(i * b, min((i + 1) * b, L))
        anchor = np.arange(a) if i > 0 else np.arange(0)
        idx = np.concatenate([anchor, own])  # original positions, copies of rows
        qa = rope_complex(q[idx], idx, theta)
        ka = rope_complex(k[idx], idx, theta)
        va = v[idx]
        n_tok = idx.size
        causal = np.tril(np.ones((n_tok, n_tok), dtype=bool))
        keep = slice(anchor.size, n_tok)
        for h in range(Hq):
            oo, ll = masked_attention(qa[:, h], ka[:, h // g], va[:, h // g], causal)
            o[own, h] = oo[keep]
            lse[h, own] = ll[keep]
    return o, lse


def causal_full(qr, kr, v):
    """Plain causal attention over the whole context (textbook reference)."""
    L = qr.shape[0]
    Hq = qr.shape[1]
    g = Hq // kr.shape[1]
    M = np.tril(np.ones((L, L), dtype=bool))
    o = np.empty_like(qr)
    lse = np.empty((Hq, L))
    for h in range(Hq):
        o[:, h], lse[h] = masked_attention(qr[:, h], kr[:, h // g], v[:, h // g], M)
    return o, lse


def round_bf16_np(x):
    """bf16 rounding by mantissa scaling (normal range only): keep 8
    significant bits, ties to even (np.round rounds halves to even)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)  # x = m * 2^e, |m| in [0.5, 1)
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def prefix_mask(L, b, prefix):
    """Dense mask of the generalised Phase 1 over context keys: block i sees
    the context rows of its ranges prefix[i] (list of [s, e)) and, causally,
    itself."""
    M = np.zeros((L, L), dtype=bool)
    for r in range(L):
        i = r // b
        for s, e in prefix[i]:
            if e > s:
                M[r, s:e] = True
        M[r, i * b:r + 1] = True
    return M


def gathered_prefix_literal(q, k, v, b, pk, pv, ppos, bounds, theta):
    """Augmented block [prefix rows || c_i] built literally: block i takes
    the prefix rows pk/pv[bounds[i,0]:bounds[i,1]] (pre-RoPE content, keys
    rotated at ppos), then itself at its own positions; plain causal
    attention in which every prefix row is visible; keep the c_i rows.
    q[L,Hq,D], k/v[L,Hkv,D], pk/pv[G,Hkv,D] float64, ppos[G]."""
    L, Hq, D = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    o = np.empty_like(q)
    lse = np.empty((Hq, L))
    ppos = np.asarray(ppos)
    for i in range(-(-L // b)):
        own = np.arange(i * b, min((i + 1) * b, L))
        qo = rope_complex(q[own], own, theta)
        ko = rope_complex(k[own], own, theta)
        gs, ge = bounds[i]
        if ge > gs:
            kk = np.concatenate([rope_complex(pk[gs:ge], ppos[gs:ge], theta), ko], axis=0)
            vv = np.concatenate([pv[gs:ge], v[own]], axis=0)
        else:
            kk, vv = ko, v[own]
        na = kk.shape[0] - own.size
        # row j of the block sees every prefix row and block rows 0..j
        mask = np.zeros((own.size, kk.shape[0]), dtype=bool)
        mask[:, :na] = True
        mask[:, na:] = np.tril(np.ones((own.size, own.size), dtype=bool))
        for h in range(Hq):
            oo, ll = masked_attention(qo[:, h], kk[:, h // g], vv[:, h // g], mask)
            o[own, h] = oo
            lse[h, own] = ll
    return o, lse


def stack_literal(x0, layers, b, a, Hq, Hkv, D, theta, eps, rnd):
    """Decoder stack with Star Phase 1 built literally: every block i >= 1
    runs the whole stack on its own augmented sequence [c_1[:a] || c_i]
    (anchor rows at positions 0..a-1, block rows at their own positions,
    plain causal attention, the anchor recomputed in every block), block 0
    on c_1 alone; the c_i rows are kept. x0 [L, dm] float64; layers: dicts
    of float64 gamma/wq/wk/wv/wo; rnd: the rounding applied to every stored
    intermediate (identity or bf16). Rotated q/k are rounded like the rest."""
    L, dm = x0.shape
    g = Hq // Hkv
    out = np.empty_like(x0)
    for i in range(-(-L // b)):
        own = np.arange(i * b, min((i + 1) * b, L))
        idx = own if (i == 0 or a == 0) else np.concatenate([np.arange(a), own])
        X = x0[idx].copy()
        S = idx.size
        for ly in layers:
            h = rnd(X / np.sqrt(np.mean(X * X, axis=-1, keepdims=True) + eps) * ly["gamma"])
            q = rnd(h @ ly["wq"].T).reshape(S, Hq, D)
            k = rnd(h @ ly["wk"].T).reshape(S, Hkv, D)
            v = rnd(h @ ly["wv"].T).reshape(S, Hkv, D)
            qr, kr = rnd(rope_complex(q, idx, theta)), rnd(rope_complex(k, idx, theta))
            mask = np.tril(np.ones((S, S), dtype=bool))
            o = np.empty((S, Hq, D))
            for hq in range(Hq):
                o[:, hq], _ = masked_attention(qr[:, hq], kr[:, hq // g], v[:, hq // g], mask)
            X = rnd(X + rnd(rnd(o.reshape(S, Hq * D)) @ ly["wo"].T))
        out[own] = X[S - own.size:]
    return out
