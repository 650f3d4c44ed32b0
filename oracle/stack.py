"""Oracle of a decoder stack around Star attention (TEST INFRASTRUCTURE ONLY;
only the tests, the smoke check and the benchmark's CPU legs use it).

Star Attention replaces only attention and needs no retraining [pith
2WVXFXZ2, the paper's abstract]. A layer here is an attention block:
    h = RMSNorm(x) * gamma;  q, k, v = h Wq^T, h Wk^T, h Wv^T;
    o = Star Phase 1 (or, for new tokens, global attention);  x = x + o Wo^T
with every stored intermediate (h, q, k, v, o, the projection o Wo^T and x)
rounded to bf16, as the GPU path stores them: the residual add rounds the
bf16 projection output plus x once more. The attention is the fp64 oracle of this package
(phase1_full / global_rows), so in layer l every block's anchor is the
layer-l hidden state of rows 0..a-1 of the whole sequence — block 1's, since
the anchor is a causal prefix of every augmented block [pith 2WVXFXZ2, "What
carries the argument": the anchor's KV is computed with each block, never
shared]. brute.stack_literal recomputes the anchor inside every augmented
block instead; the two agree (tests/test_oracle_stack.py).
"""
import numpy as np
import torch

from . import oracle as orc


def _f64(t):
    return t.detach().float().cpu().double().numpy() if isinstance(t, torch.Tensor) else \
        np.asarray(t, dtype=np.float64)


def _bf16(a):
    """float64 values that are bf16-exact -> torch bf16 (exact)."""
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)


def rmsnorm(x, gamma, eps):
    """x / sqrt(mean(x^2) + eps) * gamma over the last axis (fp64)."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * gamma


def stack_encode(x0, layers, block_len, anchor_len, Hq, Hkv, D, theta, eps=1e-5):
    """Phase 1 through the stack. x0 [B, L, dm] bf16; layers: dicts of bf16
    gamma/wq/wk/wv/wo. Returns (x [B, L, dm] float64, bf16-exact values, and
    per layer the pre-RoPE (k, v) bf16 [B, L, Hkv, D] its cache holds)."""
    rnd = orc.round_bf16
    x = _f64(x0)
    B, L, dm = x.shape
    kv = []
    for ly in layers:
        h = rnd(rmsnorm(x, _f64(ly["gamma"]), eps))
        q = rnd(h @ _f64(ly["wq"]).T).reshape(B, L, Hq, D)
        k = rnd(h @ _f64(ly["wk"]).T).reshape(B, L, Hkv, D)
        v = rnd(h @ _f64(ly["wv"]).T).reshape(B, L, Hkv, D)
        o, _ = orc.phase1_full(_bf16(q), _bf16(k), _bf16(v), block_len, anchor_len, theta)
        o = rnd(o).reshape(B, L, Hq * D)
        x = rnd(x + rnd(o @ _f64(ly["wo"]).T))
        kv.append((_bf16(k), _bf16(v)))
    return x, kv


def stack_step(x_new, layers, ctx_kv, new_kv, tail_len, Hq, Hkv, D, theta, eps=1e-5):
    """New tokens x_new [B, T, dm] (positions L + tail_len + t) through the
    stack with global attention over each layer's cache. ctx_kv: per layer
    the context (k, v) from stack_encode; new_kv: per layer a list of the
    earlier new tokens' (k, v) bf16 [B, t, Hkv, D], extended in place.
    Returns x [B, T, dm] float64 (bf16-exact)."""
    rnd = orc.round_bf16
    x = _f64(x_new)
    B, T, dm = x.shape
    for ly, (kc, vc), prev in zip(layers, ctx_kv, new_kv):
        h = rnd(rmsnorm(x, _f64(ly["gamma"]), eps))
        q = _bf16(rnd(h @ _f64(ly["wq"]).T).reshape(B, T, Hq, D))
        k = _bf16(rnd(h @ _f64(ly["wk"]).T).reshape(B, T, Hkv, D))
        v = _bf16(rnd(h @ _f64(ly["wv"]).T).reshape(B, T, Hkv, D))
        prev.append((k, v))
        kt = torch.cat([p[0] for p in prev], dim=1)
        vt = torch.cat([p[1] for p in prev], dim=1)
        bb, hh, tt = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(T), indexing="ij")
        o, _ = orc.global_rows(q, kc, vc, kt, vt, tail_len, theta, bb.ravel(), hh.ravel(),
                               tt.ravel())
        o = rnd(o.reshape(B, Hq, T, D).transpose(0, 2, 1, 3)).reshape(B, T, Hq * D)
        x = rnd(x + rnd(o @ _f64(ly["wo"]).T))
    return x
