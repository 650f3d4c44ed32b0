"""Parity at the full sizes of every workload, in the launch configuration the
benchmark times (StarLayer: Phase 1, the Phase-2 query chunk, decode steps).

The oracle computes sampled outputs one by one: Phase-1 rows at every block
start and end, at 128-row tile edges and at random, for a few query heads of
two KV groups; the query chunk's per-split partials and merged output for
sampled (token, head) pairs; and the merged output of decode steps. A
Phase-1 row depends only on its own query and the keys it sees, so sampling
is exact.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_rope_b200 import build as star_build
from block_sparse_long_rope_b200 import inputs, star
from block_sparse_long_rope_b200.configs import WORKLOADS
from block_sparse_long_rope_b200.pipeline import StarLayer, phase2_calls
from oracle import oracle as orc

from gpu_util import TOL_LSE, TOL_O, max_abs, sample_rows, to64

pytestmark = pytest.mark.gpu

DEC_STEPS_CHECKED = 2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    star_build.build()
    torch.cuda.init()


@pytest.mark.parametrize("w", WORKLOADS, ids=[w.name for w in WORKLOADS])
def test_full_size_sampled_parity(w):
    free, _ = torch.cuda.mem_get_info()
    need = (w.B * w.L * (w.Hq * 3 + w.Hkv * 6) * w.D * 2) * 1.2
    if need > free:
        pytest.skip(f"needs ~{need / 2**30:.1f} GiB of device memory")
    dev = torch.device("cuda")
    rng = np.random.default_rng(w.L + w.B)
    q, k, v = inputs.make_context(w.B, w.L, w.Hq, w.Hkv, w.D, w.index, device=dev)
    q2, k2, v2 = inputs.make_new_tokens(w.B, w.Tq + w.Tdec, w.Hq, w.Hkv, w.D, w.index, device=dev)
    calls = phase2_calls(w, q2, k2, v2)
    layer = StarLayer(w, device=dev)
    layer.encode(q, k, v)
    outs = []
    chunk_parts = None
    for i, (a, b_, c, tail) in enumerate(calls):
        o, lse = layer.attend(a, b_, c, tail)
        if i == 0:
            T0 = a.shape[1]
            S = layer.buf.part_o.shape[2]
            n_el = w.B * w.Hq * S * T0
            chunk_parts = (layer.buf.part_o.view(-1)[: n_el * w.D].view(w.B, w.Hq, S, T0, w.D).clone(),
                           layer.buf.part_lse.view(-1)[: n_el].view(w.B, w.Hq, S, T0).clone())
        if i < 1 + DEC_STEPS_CHECKED or i == len(calls) - 1:
            outs.append((i, tail, o.clone(), lse.clone()))
    star.star_device_status(layer.buf.ws1)
    star.star_device_status(layer.buf.ws2)
    torch.cuda.synchronize()

    n = w.n_blocks
    kc, vc = k.cpu(), v.cpu()
    k2c, v2c = k2.cpu(), v2.cpu()
    g = w.Hq // w.Hkv
    bsel = w.B - 1  # the last sequence of the batch
    # ---- Phase 1: sampled rows of two KV groups --------------------------------
    rows = sample_rows(w.L, w.block_len, rng, extra=8)
    kvs = sorted({0, w.Hkv - 1})
    qb, qh, qr = [], [], []
    for kvh in kvs:
        for r in rows:
            h = kvh * g + int(rng.integers(0, g))
            qb.append(bsel)
            qh.append(h)
            qr.append(int(r))
    qb, qh, qr = map(np.array, (qb, qh, qr))
    ib, ih, ir = (torch.from_numpy(x).to(dev) for x in (qb, qh, qr))
    q_sel = q[ib, ir, ih].cpu()  # [nq, D]
    ro, rl, _ = orc.phase1_rows_selected(q_sel, kc, vc, w.block_len, w.anchor_len, w.theta,
                                         qb, qh, qr, w.Hq)
    go = to64(layer.buf.o[ib, ir, ih])
    gl = to64(layer.buf.lse[ib, ih, ir])
    assert max_abs(go, ro) <= TOL_O
    assert max_abs(gl, rl) <= TOL_LSE
    # ---- Phase 2: per-split partials of the first call ---------------------------
    po, pl = chunk_parts
    T0 = po.shape[3]
    ts = np.unique(np.concatenate([[0, T0 - 1], rng.integers(0, T0, size=3)]))
    hs = np.unique(np.concatenate([[0, w.Hq - 1], rng.integers(0, w.Hq, size=2)]))
    tt, hh = np.meshgrid(ts, hs, indexing="ij")
    tt, hh = tt.ravel(), hh.ravel()
    rpo, rpl = orc.phase2_rows(q2[bsel:bsel + 1, :T0].cpu(), kc[bsel:bsel + 1], vc[bsel:bsel + 1],
                               k2c[bsel:bsel + 1, :T0], v2c[bsel:bsel + 1, :T0], w.block_len, 0,
                               w.theta, np.zeros(tt.size), hh, tt)
    assert rpo.shape[1] == n + 1
    th, tt_ = torch.from_numpy(hh).to(dev), torch.from_numpy(tt).to(dev)
    assert max_abs(to64(po[bsel][th, :, tt_]), rpo) <= TOL_O
    assert max_abs(to64(pl[bsel][th, :, tt_]), rpl) <= TOL_LSE
    # ---- Phase 2: merged outputs of the query chunk and decode steps ------------
    for (i, tail, o, lse) in outs:
        T = o.shape[1]
        ts = np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, size=3)]))
        hs = np.unique(np.concatenate([[0, w.Hq - 1], rng.integers(0, w.Hq, size=2)]))
        tt, hh = np.meshgrid(ts, hs, indexing="ij")
        tt, hh = tt.ravel(), hh.ravel()
        qn = q2[bsel:bsel + 1, tail:tail + T].cpu()
        mo, ml = orc.global_rows(qn, kc[bsel:bsel + 1], vc[bsel:bsel + 1],
                                 k2c[bsel:bsel + 1, : tail + T], v2c[bsel:bsel + 1, : tail + T],
                                 tail, w.theta, np.zeros(tt.size), hh, tt)
        ti, hi = torch.from_numpy(tt).to(dev), torch.from_numpy(hh).to(dev)
        go = to64(o[bsel][ti, hi])
        gl = to64(lse[bsel][hi, ti])
        assert max_abs(go, mo) <= TOL_O, f"call {i}"
        assert max_abs(gl, ml) <= TOL_LSE, f"call {i}"
