"""GPU parity of the decoder stack around Star attention (StarStack:
star_rmsnorm, the library's tcgen05 GEMM in star_linear / star_linear_rope,
star_phase1_encode_rotated, star_phase2_attend) against the stack oracle,
plus the row-wise calls on their own. bf16 values of magnitude above 1 (the residual stream) are
compared relative to max(1, |ref|): one bf16 ulp is 2^-8 of the value."""
import numpy as np
import pytest
import torch

from block_sparse_long_rope_b200 import inputs, star
from block_sparse_long_rope_b200.configs import Workload
from block_sparse_long_rope_b200.pipeline import phase2_calls
from block_sparse_long_rope_b200.stack import StarStack
from oracle import oracle as orc
from oracle import stack as ost

from gpu_util import to64

pytestmark = pytest.mark.gpu

W = Workload(index=60, name="stack-test", B=1, Hq=8, Hkv=2, D=64, theta=1.0e4, L=1536,
             block_len=512, anchor_len=512, Tq=24, Tdec=3)
DM = 512
LAYERS = 3
# One layer, given the same input: the residual stream rounds twice (the
# projection output, the residual add), and a difference upstream (fp32
# versus fp64 RMSNorm and projections, attention within its tolerance) can
# move each rounding by one bf16 ulp (2^-8 of the value) and add about 2e-3
# through Wo: 2^-6 relative to max(1, |x|) bounds a layer. RMSNorm
# renormalises and attention averages, so layer errors add: the whole stack
# is bounded by LAYERS * 2^-6.
TOL_LAYER = 2.0 ** -6
TOL_X = LAYERS * TOL_LAYER


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_long_rope_b200 import build as star_build

    star_build.build()
    torch.cuda.init()


def _rel(got, ref):
    got, ref = np.asarray(got, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(got - ref) / np.maximum(1.0, np.abs(ref))))


def test_rmsnorm_matches_fp64_within_one_rounding():
    x = inputs.randn_bf16((300, 1024), 1, scale=3.0)
    g = inputs.randn_bf16((1024,), 2, scale=0.2) + 1.0
    g = g.to(torch.bfloat16)
    y = torch.empty((300, 1024), dtype=torch.bfloat16, device="cuda")
    star.star_rmsnorm(x.cuda(), g.cuda(), y, 1e-5)
    torch.cuda.synchronize()
    ref = ost.rmsnorm(x.double().numpy(), g.double().numpy(), 1e-5)
    # fp32 arithmetic, one bf16 rounding: within one ulp of the fp64 value
    assert _rel(to64(y), ref) <= 2.0 ** -8


@pytest.mark.parametrize("M,N,K", [(1536, 512, 512), (1000, 640, 4096), (24, 4096, 512),
                                   (300, 264, 520), (2048, 4096, 4096)])
def test_linear_product_and_residual_add(M, N, K):
    x = inputs.randn_bf16((M, K), 3)
    w = inputs.randn_bf16((N, K), 4, scale=K ** -0.5)
    y0 = inputs.randn_bf16((M, N), 5)
    ws = star.alloc_workspace(32 << 20)
    p = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    star.star_linear(x.cuda(), w.cuda(), p, accumulate=False, workspace=ws)
    y = y0.clone().cuda()
    star.star_linear(x.cuda(), w.cuda(), y, accumulate=True, workspace=ws)
    torch.cuda.synchronize()
    # the product: fp32 accumulation of K exact bf16 products, one rounding
    ab = x.double().numpy() @ w.double().numpy().T
    assert float(np.max(np.abs(to64(p) - ab) / np.maximum(1.0, np.abs(ab)))) <= 2.0 ** -8
    # the residual add: the bf16 product plus y, rounded once more
    assert np.array_equal(to64(y), orc.round_bf16(to64(p) + y0.double().numpy()))


@pytest.mark.parametrize("B,S,H,D,K,pos0", [(1, 1536, 8, 64, 512, 0), (2, 700, 4, 128, 1024, 0),
                                            (1, 300, 3, 128, 264, 123456),
                                            (1, 4096, 8, 128, 4096, 0)])
def test_linear_rope_equals_linear_then_rope(B, S, H, D, K, pos0):
    """The RoPE and cache epilogues give the bits of star_linear followed by
    star_rope (the projection is rounded to bf16, then rotated with the
    correctly rounded rotation), token-major or head-major into a cache."""
    dev = "cuda"
    theta = 5e5
    M, N = B * S, H * D
    x = inputs.randn_bf16((M, K), 11).to(dev)
    w = inputs.randn_bf16((N, K), 12, scale=K ** -0.5).to(dev)
    ws = star.alloc_workspace(star.star_linear_rope_workspace_bytes(S, D, True))
    p = torch.empty((B, S, H, D), dtype=torch.bfloat16, device=dev)
    star.star_linear(x, w, p, workspace=ws)
    ref = torch.empty_like(p)
    star.star_rope(p, ref, theta, pos0=pos0)
    # rotated, token-major
    q = torch.full_like(p, float("nan"))
    star.star_linear_rope(x, w, q, D, True, S, pos0, theta, 0, ws)
    # rotated, and plain, into head-major caches with spare rows
    Lcap = S + 5
    kc = torch.full((B, H, Lcap, D), float("nan"), dtype=torch.bfloat16, device=dev)
    vc = torch.full_like(kc, float("nan"))
    star.star_linear_rope(x, w, kc, D, True, S, pos0, theta, Lcap, ws)
    star.star_linear_rope(x, w, vc, D, False, S, pos0, theta, Lcap, ws)
    star.star_device_status(ws)
    torch.cuda.synchronize()
    assert torch.equal(q, ref)
    assert torch.equal(kc[:, :, :S], ref.permute(0, 2, 1, 3))
    assert torch.equal(vc[:, :, :S], p.permute(0, 2, 1, 3))
    assert torch.isnan(kc[:, :, S:].float()).all() and torch.isnan(vc[:, :, S:].float()).all()
    # and against the oracle's correctly rounded rotation of the bf16 projection
    rot = orc.rope(p.cpu(), np.arange(pos0, pos0 + S), theta, round_out=True)
    np.testing.assert_array_equal(to64(q), rot)
    # K and V in one GEMM (w_kv = [Wk; Wv]): the same bits as the two calls
    wv = inputs.randn_bf16((N, K), 13, scale=K ** -0.5).to(dev)
    pv = torch.empty((B, S, H, D), dtype=torch.bfloat16, device=dev)
    star.star_linear(x, wv, pv, workspace=ws)
    kc2 = torch.full_like(kc, float("nan"))
    vc2 = torch.full_like(vc, float("nan"))
    star.star_linear_kv_cache(x, torch.cat([w, wv]).contiguous(), kc2, vc2, S, pos0, theta, ws)
    star.star_device_status(ws)
    torch.cuda.synchronize()
    assert torch.equal(kc2[:, :, :S], ref.permute(0, 2, 1, 3))
    assert torch.equal(vc2[:, :, :S], pv.permute(0, 2, 1, 3))
    assert torch.isnan(kc2[:, :, S:].float()).all() and torch.isnan(vc2[:, :, S:].float()).all()


def test_stack_encode_and_steps_match_the_oracle():
    dev = torch.device("cuda")
    wts = inputs.make_stack_weights(LAYERS, DM, W.Hq, W.Hkv, W.D, W.index)
    st = StarStack(W, DM, [{k: v.to(dev) for k, v in ly.items()} for ly in wts], device=dev)
    x0 = inputs.make_hidden(W.B, W.L, DM, W.index)
    x = x0.to(dev)
    for i in range(LAYERS):
        # each layer against the oracle's layer on the same (GPU) input
        x_in = x.cpu()
        st.encode_layer(x, i)
        torch.cuda.synchronize()
        star.star_device_status(st.layers[i].buf.ws1)
        ref_i, kv_i = ost.stack_encode(x_in, wts[i:i + 1], W.block_len, W.anchor_len, W.Hq, W.Hkv,
                                       W.D, W.theta)
        assert _rel(to64(x), ref_i) <= TOL_LAYER
        # its cache holds its own K, rotated at the original positions
        rot = orc.rope(kv_i[0][0], np.arange(W.L), W.theta, round_out=True)  # [B, L, Hkv, D]
        got = to64(st.layers[i].buf.k_cache[:, :, :W.L]).transpose(0, 2, 1, 3)
        assert _rel(got, rot) <= TOL_LAYER
    # the whole stack against the oracle's stack from the same start
    ref, ctx_kv = ost.stack_encode(x0, wts, W.block_len, W.anchor_len, W.Hq, W.Hkv, W.D, W.theta)
    assert _rel(to64(x), ref) <= TOL_X

    # Phase 2 through the stack: the query chunk, then decode steps
    xn_all = inputs.make_hidden(W.B, W.Tq + W.Tdec, DM, W.index, name="x2")
    prev = [[] for _ in wts]
    calls = phase2_calls(W, xn_all.view(W.B, W.Tq + W.Tdec, 1, DM), xn_all.view(W.B, -1, 1, DM),
                         xn_all.view(W.B, -1, 1, DM))
    for (xs, _, _, tail) in calls:
        xs = xs.view(W.B, -1, DM)
        xg = xs.to(dev).contiguous()
        st.step(xg, tail)
        torch.cuda.synchronize()
        for ly in st.layers:
            star.star_device_status(ly.buf.ws2)
        want = ost.stack_step(xs, wts, ctx_kv, prev, tail, W.Hq, W.Hkv, W.D, W.theta)
        assert _rel(to64(xg), want) <= TOL_X
