"""Pins of the oracle's RoPE and bf16 rounding against independent facts.

RoPE: rotate-half at original global positions (Star Attention keeps the
anchor's original position IDs, pith 2WVXFXZ2 "What carries the argument";
position IDs preserve RoPE distances, pith 2607.20457 "What carries the
argument"). The checks are closed forms (identity at p = 0, the golden
table), the complex-multiplication form, norm preservation and
relative-position invariance.
"""
import os

import numpy as np
import pytest
import torch

from oracle import brute
from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rope_closed_form.txt")


def _bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _load_golden():
    cases = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            lhs, rhs = line.split("|")
            tok = lhs.split()
            D, theta, p = int(tok[0]), float(tok[1]), int(tok[2])
            x = [float(t) for t in tok[3:]]
            y = [float(t) for t in rhs.split()]
            assert len(x) == D and len(y) == D
            cases.append((D, theta, p, x, y))
    return cases


@pytest.mark.parametrize("case", _load_golden())
def test_rope_golden_closed_form(case):
    D, theta, p, x, y = case
    xt = _bf16(x).reshape(1, 1, 1, D)
    got = orc.rope(xt, [p], theta)[0, 0, 0]
    np.testing.assert_allclose(got, y, rtol=0, atol=1e-15)


def test_rope_identity_at_position_zero():
    x = torch.randn(2, 1, 3, 128).to(torch.bfloat16)
    got = orc.rope(x, [0], 5e5)
    np.testing.assert_array_equal(got, x.double().numpy())


@pytest.mark.parametrize("D,theta", [(4, 1e4), (64, 1e4), (128, 5e5)])
def test_rope_equals_complex_multiplication(D, theta):
    torch.manual_seed(0)
    S, H = 9, 3
    x = torch.randn(1, S, H, D).to(torch.bfloat16)
    pos = np.array([0, 1, 2, 7, 511, 4096, 65535, 131071, 1048575], dtype=np.int64)
    got = orc.rope(x, pos, theta)[0]
    ref = brute.rope_complex(x.double().numpy()[0], pos, theta)
    # large angles: cos/sin of p*theta_i evaluated by two libraries agree to a
    # few ulps of the angle (|angle| <= 1.1e6 -> ~2e-10 absolute)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-9)


def test_rope_preserves_pair_norms():
    torch.manual_seed(1)
    D = 128
    x = torch.randn(1, 5, 2, D).to(torch.bfloat16)
    pos = np.array([3, 100, 4097, 300000, 1000000])
    y = orc.rope(x, pos, 5e5)
    xd = x.double().numpy()
    h = D // 2
    nx = xd[..., :h] ** 2 + xd[..., h:] ** 2
    ny = y[..., :h] ** 2 + y[..., h:] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-12, atol=1e-12)


def test_rope_scores_depend_only_on_relative_position():
    torch.manual_seed(2)
    D = 64
    q = torch.randn(1, 1, 1, D).to(torch.bfloat16)
    k = torch.randn(1, 1, 1, D).to(torch.bfloat16)
    for p, pp in [(5, 2), (700, 11), (4096, 4000)]:
        for delta in (0, 1, 37, 12345):
            a = orc.rope(q, [p + delta], 1e4)[0, 0, 0] @ orc.rope(k, [pp + delta], 1e4)[0, 0, 0]
            b = orc.rope(q, [p], 1e4)[0, 0, 0] @ orc.rope(k, [pp], 1e4)[0, 0, 0]
            assert abs(a - b) < 1e-12 * max(1.0, abs(b)) * 100


def test_round_bf16_ties_to_even_and_known_values():
    one = 1.0
    cases = {
        one: one,
        one + 2.0 ** -8: one,                     # tie -> even (1.0)
        one + 3 * 2.0 ** -8: one + 2.0 ** -6,     # tie -> even (1 + 2^-6)
        one + 2.0 ** -8 + 2.0 ** -30: one + 2.0 ** -7,  # just above the tie
        -(one + 2.0 ** -8): -one,
        3.4e38: float("inf"),                    # above max + half an ulp
        2.0 ** -133: 2.0 ** -133,                # smallest bf16 subnormal
        2.0 ** -134: 0.0,                        # tie -> even (0)
        0.0: 0.0,
    }
    xs = np.array(list(cases.keys()))
    got = orc.round_bf16(xs)
    np.testing.assert_array_equal(got, np.array(list(cases.values())))


def test_round_bf16_matches_single_rounding_from_float32():
    # torch rounds fp32 -> bf16 once (nearest even); on fp32 inputs the
    # oracle's direct fp64 rounding must agree bit for bit.
    torch.manual_seed(3)
    x32 = torch.randn(100000) * 10
    ref = x32.to(torch.bfloat16).double().numpy()
    got = orc.round_bf16(x32.double().numpy())
    np.testing.assert_array_equal(got, ref)


def test_round_bf16_matches_mantissa_scaling_on_doubles():
    rng = np.random.default_rng(4)
    x = rng.standard_normal(100000) * 3
    np.testing.assert_array_equal(orc.round_bf16(x), brute.round_bf16_np(x))
