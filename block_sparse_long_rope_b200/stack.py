"""A decoder stack of attention blocks around Star attention, through the C ABI.

Star Attention changes only attention and needs no retraining [pith
2WVXFXZ2, the paper's abstract], so a layer here is
    h = RMSNorm(x) * gamma                      (star_rmsnorm)
    q, k, v = h Wq^T, h Wk^T, h Wv^T            (star_linear)
    o = Star Phase 1 over the layer's context   (star_phase1_encode)
        or, for new tokens, partials + merge    (star_phase2_attend)
    x = x + o Wo^T                              (star_linear, residual fused)
Every layer encodes its own anchor: in layer l block i's anchor is rows
0..a-1 of the layer-l hidden state, which is block 1's (the anchor is a
causal prefix of every augmented block), read in place from that layer's
cache [pith 2WVXFXZ2, "What carries the argument"]. The weights are random
(no trained checkpoint is available); the MLP of a full decoder layer is
row-wise like RMSNorm and is left out.
"""
import torch

from . import star
from .configs import Workload
from .pipeline import StarLayer



class StarStack:
    """Caller-owned buffers of an n-layer stack for workload `w` with model
    width dm; `weights` is a list of per-layer dicts of bf16 device tensors
    (gamma [dm], wq [Hq*D, dm], wk / wv [Hkv*D, dm], wo [dm, Hq*D])."""

    def __init__(self, w: Workload, dm, weights, eps=1e-5, device="cuda"):
        self.w, self.dm, self.weights, self.eps = w, dm, weights, eps
        dev = torch.device(device)
        B, L, Hq, Hkv, D = w.B, w.L, w.Hq, w.Hkv, w.D
        self.layers = [StarLayer(w, device=dev) for _ in weights]
        bf = dict(dtype=torch.bfloat16, device=dev)
        self.h = torch.empty((B, L, dm), **bf)
        self.q = torch.empty((B, L, Hq, D), **bf)
        Tmax = max(w.Tq, 1)
        self.h2 = torch.empty((B * Tmax * dm,), **bf)
        self.q2 = torch.empty((B * Tmax * Hq * D,), **bf)
        self.k2 = torch.empty((B * Tmax * Hkv * D,), **bf)
        self.v2 = torch.empty((B * Tmax * Hkv * D,), **bf)
        # each layer's K and V projection weights stacked, for one K/V GEMM
        self.w_kv = [torch.cat([wt["wk"], wt["wv"]], dim=0).contiguous() for wt in weights]
        # the GEMMs' status word and the RoPE epilogue's cos/sin table
        self.gemm_ws = star.alloc_workspace(
            star.star_linear_rope_workspace_bytes(max(L, Tmax), D, True), dev)

    def encode_layer(self, x, index):
        """Phase 1 of layer `index` on the residual stream x [B, L, dm] bf16
        (updated in place); fills that layer's KV cache rows [0, L). The Q
        projection leaves Q rotated, one K/V projection writes the layer's
        cache (K rotated) directly, then only the attention runs."""
        w = self.w
        ly, wt = self.layers[index], self.weights[index]
        b = ly.buf
        star.star_rmsnorm(x, wt["gamma"], self.h, self.eps)
        star.star_linear_rope(self.h, wt["wq"], self.q, w.D, True, w.L, 0, w.theta, 0,
                              self.gemm_ws)
        star.star_linear_kv_cache(self.h, self.w_kv[index], b.k_cache, b.v_cache, w.L, 0,
                                  w.theta, self.gemm_ws)
        star.star_phase1_encode_rotated(self.q, b.o, b.k_cache, b.v_cache, w.L, w.block_len,
                                        w.anchor_len, b.ws1)
        star.star_linear(b.o, wt["wo"], x, accumulate=True, workspace=self.gemm_ws)
        return x

    def encode(self, x):
        """Phase 1 through every layer; x [B, L, dm] bf16 (the residual
        stream) is updated in place and returned."""
        for i in range(len(self.layers)):
            self.encode_layer(x, i)
        return x

    def step(self, x, tail_len):
        """T new tokens x [B, T, dm] (positions L + tail_len + t) through
        every layer: each layer appends their k/v to its cache and attends
        globally (partials + exact merge). x is updated in place."""
        w = self.w
        B, T, dm = x.shape
        h = self.h2[:B * T * dm].view(B, T, dm)
        q = self.q2[:B * T * w.Hq * w.D].view(B, T, w.Hq, w.D)
        k = self.k2[:B * T * w.Hkv * w.D].view(B, T, w.Hkv, w.D)
        v = self.v2[:B * T * w.Hkv * w.D].view(B, T, w.Hkv, w.D)
        for ly, wt in zip(self.layers, self.weights):
            star.star_rmsnorm(x, wt["gamma"], h, self.eps)
            star.star_linear(h, wt["wq"], q, workspace=self.gemm_ws)
            star.star_linear(h, wt["wk"], k, workspace=self.gemm_ws)
            star.star_linear(h, wt["wv"], v, workspace=self.gemm_ws)
            o, _ = ly.attend(q, k, v, tail_len)
            star.star_linear(o, wt["wo"], x, accumulate=True, workspace=self.gemm_ws)
        return x

    def flops_encode(self):
        """Projection FLOPs plus Star Phase-1 unmasked attention FLOPs of one
        encode (2 per multiply-add)."""
        w = self.w
        rows = w.B * w.L
        proj = 2.0 * rows * self.dm * (2 * w.Hq * w.D + 2 * w.Hkv * w.D)
        return len(self.layers) * (proj + w.phase1_flops())
