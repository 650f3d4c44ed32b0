"""Pins of the decoder-stack oracle (oracle/stack.py).

The central pin: Star Phase 1 through several layers, where every block
reads the anchor's layer-l hidden state from the one sequence-wide pass,
equals the literal per-host computation in which every block runs the whole
stack on its own augmented input [c_1 || c_i] and recomputes the anchor at
each layer [pith 2WVXFXZ2, "What carries the argument"]. Plus closed forms
of RMSNorm, the residual identity, and chunked-versus-one-shot processing of
new tokens.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_rope_b200 import inputs
from oracle import brute
from oracle import oracle as orc
from oracle import stack as ost


def _weights(n, dm, Hq, Hkv, D, seed):
    return inputs.make_stack_weights(n, dm, Hq, Hkv, D, seed)


def _f64(ly):
    return {k: v.float().double().numpy() for k, v in ly.items()}


def test_rmsnorm_closed_form():
    # a constant row c: c / sqrt(c^2 + eps) * gamma
    x = np.full((3, 16), -2.5)
    g = np.linspace(0.5, 1.5, 16)
    want = np.broadcast_to(-2.5 / np.sqrt(6.25 + 1e-5) * g, x.shape)
    np.testing.assert_allclose(ost.rmsnorm(x, g, 1e-5), want, rtol=1e-15)
    # scale invariance with eps = 0
    y = np.random.default_rng(0).normal(size=(4, 16))
    np.testing.assert_allclose(ost.rmsnorm(7.0 * y, g, 0.0), ost.rmsnorm(y, g, 0.0), rtol=1e-14)


def test_zero_output_projection_keeps_the_residual():
    L, dm, Hq, Hkv, D = 64, 32, 4, 2, 8
    lys = _weights(2, dm, Hq, Hkv, D, seed=1)
    for ly in lys:
        ly["wo"] = torch.zeros_like(ly["wo"])
    x0 = inputs.make_hidden(1, L, dm, 1)
    x, _ = ost.stack_encode(x0, lys, 16, 16, Hq, Hkv, D, 1e4)
    np.testing.assert_array_equal(x, x0.float().double().numpy())


@pytest.mark.parametrize("a", [32, 12, 0])
def test_star_stack_equals_per_block_literal_recomputation(a):
    L, b, dm, Hq, Hkv, D, theta, eps = 112, 32, 32, 4, 2, 8, 1e4, 1e-5
    lys = _weights(3, dm, Hq, Hkv, D, seed=2 + a)
    x0 = inputs.make_hidden(1, L, dm, 2 + a)
    x, _ = ost.stack_encode(x0, lys, b, a, Hq, Hkv, D, theta, eps)
    lit = brute.stack_literal(x0.float().double().numpy()[0], [_f64(ly) for ly in lys], b, a,
                              Hq, Hkv, D, theta, eps, orc.round_bf16)
    np.testing.assert_allclose(x[0], lit, rtol=0, atol=1e-9)


def test_new_tokens_one_at_a_time_equal_one_chunk():
    L, b, a, dm, Hq, Hkv, D, theta = 64, 16, 16, 32, 4, 2, 8, 1e4
    lys = _weights(2, dm, Hq, Hkv, D, seed=5)
    x0 = inputs.make_hidden(1, L, dm, 5)
    _, ctx_kv = ost.stack_encode(x0, lys, b, a, Hq, Hkv, D, theta)
    xn = inputs.make_hidden(1, 5, dm, 5, name="x2")
    whole = ost.stack_step(xn, lys, ctx_kv, [[] for _ in lys], 0, Hq, Hkv, D, theta)
    prev = [[] for _ in lys]
    parts = [ost.stack_step(xn[:, t:t + 1], lys, ctx_kv, prev, t, Hq, Hkv, D, theta)
             for t in range(5)]
    np.testing.assert_allclose(np.concatenate(parts, axis=1), whole, rtol=0, atol=1e-12)
