"""Pins of the oracle's Phase 2 partials and LSE merge.

The exact-merge identity (pith 2WVXFXZ2, Circularity check: each host's local
output and softmax statistic are re-weighted into exact global attention;
minor comment on Algorithm 2: the weight is exp(s_h - s_global)) is checked
against one-shot softmax over the concatenated keys, on uneven and empty
splits, and against a closed-form two-split example.
"""
import numpy as np
import pytest
import torch

from oracle import brute
from oracle import oracle as orc


def _rand(shape, gen):
    return torch.randn(*shape, generator=gen).to(torch.bfloat16)


def _setup(L, b, T, tail_len, Hq, Hkv, D, seed):
    gen = torch.Generator().manual_seed(seed)
    kc, vc = _rand((1, L, Hkv, D), gen), _rand((1, L, Hkv, D), gen)
    Ltail = tail_len + T
    kt, vt = _rand((1, Ltail, Hkv, D), gen), _rand((1, Ltail, Hkv, D), gen)
    qn = _rand((1, T, Hq, D), gen)
    return qn, kc, vc, kt, vt


def _all_rows(T, Hq):
    hh, tt = np.meshgrid(np.arange(Hq), np.arange(T), indexing="ij")
    return np.zeros(hh.size, dtype=np.int64), hh.ravel(), tt.ravel()


@pytest.mark.parametrize("L,b,T,tail_len", [(64, 16, 4, 0), (50, 12, 3, 5), (37, 37, 1, 9),
                                            (40, 7, 2, 0), (96, 32, 1, 20)])
def test_merge_of_partials_equals_global_attention(L, b, T, tail_len):
    Hq, Hkv, D = 4, 2, 8
    qn, kc, vc, kt, vt = _setup(L, b, T, tail_len, Hq, Hkv, D, seed=L * 31 + T)
    qb, qh, qt = _all_rows(T, Hq)
    po, pl = orc.phase2_rows(qn, kc, vc, kt, vt, b, tail_len, 1e4, qb, qh, qt, round_qk=False)
    assert po.shape[1] == -(-L // b) + 1
    o, lse = orc.lse_merge(po, pl)
    go, gl = orc.global_rows(qn, kc, vc, kt, vt, tail_len, 1e4, qb, qh, qt, round_qk=False)
    np.testing.assert_allclose(o, go, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, gl, rtol=0, atol=1e-12)


def test_partials_match_brute_force_per_split():
    L, b, T, tail_len, Hq, Hkv, D, theta = 45, 10, 3, 4, 4, 2, 8, 1e4
    qn, kc, vc, kt, vt = _setup(L, b, T, tail_len, Hq, Hkv, D, seed=3)
    qb, qh, qt = _all_rows(T, Hq)
    po, pl = orc.phase2_rows(qn, kc, vc, kt, vt, b, tail_len, theta, qb, qh, qt, round_qk=False)
    # brute: rotate everything at its position, attend per split with an explicit key set
    kall = np.concatenate([kc.double().numpy()[0], kt.double().numpy()[0]], axis=0)
    vall = np.concatenate([vc.double().numpy()[0], vt.double().numpy()[0]], axis=0)
    kr = brute.rope_complex(kall, np.arange(kall.shape[0]), theta)
    g = Hq // Hkv
    n = -(-L // b)
    for i, (h, t) in enumerate(zip(qh, qt)):
        p = L + tail_len + t
        qr = brute.rope_complex(qn.double().numpy()[0, t:t + 1], np.array([p]), theta)[0, h]
        splits = [np.arange(j * b, min((j + 1) * b, L)) for j in range(n)]
        splits.append(np.arange(L, p + 1))
        for j, keys in enumerate(splits):
            mask = np.ones((1, keys.size), dtype=bool)
            oo, ll = brute.masked_attention(qr[None], kr[keys, h // g], vall[keys, h // g], mask)
            np.testing.assert_allclose(po[i, j], oo[0], rtol=0, atol=1e-12)
            np.testing.assert_allclose(pl[i, j], ll[0], rtol=0, atol=1e-12)


def test_merge_random_partitions_with_empty_parts():
    rng = np.random.default_rng(0)
    D = 16
    for trial in range(20):
        nk = int(rng.integers(1, 60))
        q = rng.standard_normal(D)
        k = rng.standard_normal((nk, D))
        v = rng.standard_normal((nk, D))
        full_o, full_l = brute.masked_attention(q[None], k, v, np.ones((1, nk), dtype=bool))
        cuts = np.sort(rng.integers(0, nk + 1, size=int(rng.integers(1, 6))))
        bounds = np.concatenate([[0], cuts, [nk]])
        po, pl = [], []
        for lo, hi in zip(bounds[:-1], bounds[1:]):
            if hi == lo:  # empty split: -inf statistic, output unused
                po.append(np.full(D, 123.0))
                pl.append(-np.inf)
                continue
            o, l = brute.masked_attention(q[None], k[lo:hi], v[lo:hi], np.ones((1, hi - lo), bool))
            po.append(o[0])
            pl.append(l[0])
        o, l = orc.lse_merge(np.array(po)[None], np.array(pl)[None])
        np.testing.assert_allclose(o[0], full_o[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[0], full_l[0], rtol=0, atol=1e-12)


def test_merge_closed_form_two_splits():
    # two splits with equal statistics: the merged output is the mean and the
    # merged log-sum-exp adds log 2
    po = np.array([[[1.0, -2.0], [3.0, 4.0]]])
    pl = np.array([[0.5, 0.5]])
    o, l = orc.lse_merge(po, pl)
    np.testing.assert_allclose(o[0], [2.0, 1.0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(l[0], 0.5 + np.log(2.0), rtol=0, atol=1e-15)
    # weights e^1 : e^0 for statistics (1, 0)
    pl = np.array([[1.0, 0.0]])
    o, l = orc.lse_merge(po, pl)
    w = np.e / (np.e + 1)
    np.testing.assert_allclose(o[0], w * po[0, 0] + (1 - w) * po[0, 1], rtol=0, atol=1e-15)
    np.testing.assert_allclose(l[0], np.log(np.e + 1), rtol=0, atol=1e-15)


def test_tail_split_is_causal_over_this_calls_tokens():
    # token t of a call must not see tail tokens after it: changing the k/v of
    # the last token leaves every earlier token's partials unchanged
    L, b, T, tail_len = 32, 8, 4, 3
    qn, kc, vc, kt, vt = _setup(L, b, T, tail_len, 2, 1, 8, seed=8)
    qb, qh, qt = _all_rows(T, 2)
    po, pl = orc.phase2_rows(qn, kc, vc, kt, vt, b, tail_len, 1e4, qb, qh, qt)
    kt2, vt2 = kt.clone(), vt.clone()
    kt2[0, -1] = 5.0
    vt2[0, -1] = -5.0
    po2, pl2 = orc.phase2_rows(qn, kc, vc, kt2, vt2, b, tail_len, 1e4, qb, qh, qt)
    early = qt < T - 1
    np.testing.assert_array_equal(po[early], po2[early])
    np.testing.assert_array_equal(pl[early], pl2[early])
    assert not np.array_equal(po[~early, -1], po2[~early, -1])
