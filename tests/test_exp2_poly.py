"""The polynomial exp2 that the attention kernel evaluates on the FMA pipe for
part of the softmax: its coefficients are the ones the fit script produces,
its relative error on the reduced interval is below 3e-6, and the full
range-reduction (x = n + f, 2^n added to the exponent bits) emulated in fp32
matches 2^x to 5e-6 over the softmax's range."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_long_rope_b200", "csrc")
sys.path.insert(0, CSRC)

import fit_exp2_poly  # noqa: E402


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "phase1_sm100.cu")).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[: body.index("return")]
    nums = [float(x) for x in re.findall(r"([0-9]\.[0-9]+e[-+][0-9]+)f", body)]
    # fmaf(c4, f, c3) then c2, c1, c0
    c4, c3, c2, c1, c0 = nums
    return np.array([c0, c1, c2, c3, c4], dtype=np.float32)


def test_coefficients_come_from_the_fit():
    np.testing.assert_array_equal(_kernel_coefficients(), fit_exp2_poly.fit())


def test_relative_error_on_reduced_interval():
    assert fit_exp2_poly.max_rel_error(_kernel_coefficients()) < 3e-6


def _emulate(x):
    """fp32 emulation of exp2_poly as the kernel computes it."""
    c = _kernel_coefficients()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)
    n = t.view(np.int32) - np.int32(0x4B400000)
    p = np.float32(c[4])
    for a in (c[3], c[2], c[1], c[0]):
        p = (p * f + a).astype(np.float32)  # one fp32 rounding per step (fma rounds once)
    return (p.view(np.int32) + (n << 23)).view(np.float32)


def test_full_range_matches_exp2():
    x = np.linspace(-120.0, 8.0, 400001, dtype=np.float32)
    got = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1.0)) < 5e-6
    # at the clamp the result is negligible next to the row maximum (2^0)
    assert _emulate(np.array([-1e9, -np.inf], dtype=np.float32)).max() < 2.0 ** -124
