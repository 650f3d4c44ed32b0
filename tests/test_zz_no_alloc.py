"""The decode entry point that allocates nothing (star_phase2_decode_static).

It serves callers that cannot allocate device memory themselves (a plugin
whose host owns every device allocation, a serving loop that must not block
in cudaMalloc/cudaFree): its scratch lives in a fixed device array inside the
library. This test calls it through the C ABI on two calls in a row and
checks its partials against the fp64 oracle (the tolerances of the other
parity tests) and against star_phase2_partial with a caller workspace (the
same decode kernel with another chunk size: fp32 sums, bf16 weights), then
reads the array's status word back through
star_phase2_decode_static_status. The file is collected last so that a stop
at the first failure has already run every other test; it also passes alone
in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_long_rope_b200 import _abi
from block_sparse_long_rope_b200 import build as star_build
from block_sparse_long_rope_b200 import star
from oracle import oracle as orc

pytestmark = pytest.mark.gpu

TOL_O = 2e-2      # against the oracle: bf16-path tolerances of every parity test
TOL_LSE = 1e-3
# Against the workspace entry point: the same kernel with another chunk size.
# Its row sums (hence the LSE) are fp32, so those agree to fp32 rounding; the
# P*V product takes P in bf16 (8 significant bits) relative to each chunk's
# own running max, so two chunkings of one split round each weight
# differently by up to 2^-9 relative, which on averaged N(0,1) values stays
# well inside 2e-3.
TOL_SAME_O = 2e-3
TOL_SAME_LSE = 1e-5


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16).cuda()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _to64(t):
    return t.detach().float().cpu().double().numpy()


@pytest.mark.parametrize("B,L,Hq,Hkv,D,b,T", [(1, 2048, 4, 1, 64, 512, 1),
                                               (2, 4000, 32, 8, 128, 1024, 1),
                                               (1, 3000, 16, 2, 128, 700, 2)])
def test_static_scratch_decode_matches_oracle_and_workspace_entry(B, L, Hq, Hkv, D, b, T):
    star_build.build()
    lib = _abi.load()
    theta = 5e5
    steps = 2
    Lcap = L + steps * T
    q = _rand((B, L, Hq, D), 1)
    k = _rand((B, L, Hkv, D), 2)
    v = _rand((B, L, Hkv, D), 3)
    o = torch.empty_like(q)
    kc = torch.zeros((B, Hkv, Lcap, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    ws1 = star.alloc_workspace(star.star_phase1_workspace_bytes(B, L, Hq, D))
    star.star_phase1_encode(q, k, v, o, kc, vc, b, b, theta, ws1)
    kc2, vc2 = kc.clone(), vc.clone()  # the static entry point works on its own cache copy
    n = -(-L // b)
    ws2 = star.alloc_workspace(star.star_phase2_workspace_bytes(B, T, Hq, Hkv, D, Lcap, b))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    qn_all = _rand((B, steps * T, Hq, D), 10)
    kn_all = _rand((B, steps * T, Hkv, D), 20)
    vn_all = _rand((B, steps * T, Hkv, D), 30)
    for step in range(steps):  # two calls in a row (the tail grows by T)
        tail = step * T
        qn = qn_all[:, tail:tail + T].contiguous()
        kn = kn_all[:, tail:tail + T].contiguous()
        vn = vn_all[:, tail:tail + T].contiguous()
        po_ref = torch.empty((B, Hq, n + 1, T, D), device="cuda")
        pl_ref = torch.empty((B, Hq, n + 1, T), device="cuda")
        star.star_phase2_partial(qn, kn, vn, kc, vc, L, b, tail, po_ref, pl_ref, theta, ws2)
        po = torch.full((B, Hq, n + 1, T, D), float("nan"), device="cuda")
        pl = torch.full((B, Hq, n + 1, T), float("nan"), device="cuda")
        ns = ctypes.c_int(0)
        status = lib.star_phase2_decode_static(
            _p(qn), _p(kn), _p(vn), T, _p(kc2), _p(vc2), Lcap, L, b, tail, _p(po), _p(pl),
            ctypes.byref(ns), B, Hq, Hkv, D, theta, stream)
        assert status == 0, lib.star_last_error()
        assert ns.value == n + 1
        # no device error was recorded (the read-back synchronises the stream)
        assert lib.star_phase2_decode_static_status(stream) == 0, lib.star_last_error()
        star.star_device_status(ws2)
        assert torch.isfinite(po).all() and torch.isfinite(pl).all()
        # the same kernel with a caller workspace: fp32 rounding apart, equal
        assert (po - po_ref).abs().max().item() <= TOL_SAME_O
        assert (pl - pl_ref).abs().max().item() <= TOL_SAME_LSE
        # against the fp64 oracle, every (batch, head, token) and split
        bb, hh, tt = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(T), indexing="ij")
        bb, hh, tt = bb.ravel(), hh.ravel(), tt.ravel()
        rpo, rpl = [], []
        for bi in range(B):
            sel = bb == bi
            o_, l_ = orc.phase2_rows(qn[bi:bi + 1].cpu(), k[bi:bi + 1].cpu(), v[bi:bi + 1].cpu(),
                                     kn_all[bi:bi + 1, :tail + T].cpu(),
                                     vn_all[bi:bi + 1, :tail + T].cpu(), b, tail, theta,
                                     np.zeros(sel.sum()), hh[sel], tt[sel])
            rpo.append(o_)
            rpl.append(l_)
        gpo = _to64(po).transpose(0, 1, 3, 2, 4).reshape(-1, n + 1, D)
        gpl = _to64(pl).transpose(0, 1, 3, 2).reshape(-1, n + 1)
        assert np.abs(gpo - np.concatenate(rpo)).max() <= TOL_O
        assert np.abs(gpl - np.concatenate(rpl)).max() <= TOL_LSE
        # both entry points appended the same rotated key/value rows
        assert torch.equal(kc2[:, :, L + tail:L + tail + T], kc[:, :, L + tail:L + tail + T])
        assert torch.equal(vc2[:, :, L + tail:L + tail + T], vc[:, :, L + tail:L + tail + T])


def test_static_scratch_rejects_oversized_problems():
    star_build.build()
    lib = _abi.load()
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check fails first
    ns = ctypes.c_int(0)
    # T * g = 32 > 16: not a decode step
    st = lib.star_phase2_decode_static(fake, fake, fake, 8, fake, fake, 5000, 4000, 1000, 0, fake,
                                       fake, ctypes.byref(ns), 1, 32, 8, 128, 5e5, None)
    assert st == 1 and b"decode" in lib.star_last_error()
    # 1024 sequences x 8 KV heads of 1M tokens: the partials exceed 16 MiB at any chunk size
    st = lib.star_phase2_decode_static(fake, fake, fake, 1, fake, fake, 1048600, 1048576, 131072, 0,
                                       fake, fake, ctypes.byref(ns), 1024, 32, 8, 128, 5e5, None)
    assert st == 1 and b"static scratch" in lib.star_last_error()
