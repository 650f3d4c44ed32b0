"""GPU parity of each kernel through the C ABI against the fp64 oracle.

Tolerances: bf16 outputs max-abs 2e-2, fp32 LSE max-abs 1e-3; index math
bit-exact. The oracle rounds rotated Q/K to bf16, the precision in which the
KV cache and the rotated tensors are stored.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_rope_b200 import build as star_build
from block_sparse_long_rope_b200 import star
from oracle import oracle as orc

from gpu_util import TOL_LSE, TOL_O, max_abs, rand_bf16, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    star_build.build()
    torch.cuda.init()


# ----------------------------------------------------------------------------- RoPE
@pytest.mark.parametrize("D,theta", [(64, 1e4), (128, 5e5)])
def test_rope_matches_oracle_at_far_positions(D, theta):
    S, H = 40, 3
    x = rand_bf16((2, S, H, D), seed=D)
    pos = torch.tensor([0, 1, 2, 3, 127, 128, 511, 4095, 4096, 16383, 65535, 65536, 131071,
                        131072, 262143, 524287, 524288, 1048575, 1048000, 999999] +
                       list(range(20)), dtype=torch.int32)
    y = torch.empty_like(x)
    star.star_rope(x, y, theta, pos=pos.cuda())
    torch.cuda.synchronize()
    ref = orc.rope(x.cpu(), pos.numpy().astype(np.int64), theta)
    got = to64(y)
    assert max_abs(got, ref) <= TOL_O
    # RoPE runs in fp64 and rounds once: the result is the correctly rounded
    # bf16 of the exact rotation, i.e. bit-identical to the oracle's rounding
    exact = orc.round_bf16(ref)
    np.testing.assert_array_equal(got, exact)


def test_rope_strided_and_in_place():
    B, S, H, D = 2, 33, 4, 128
    x = rand_bf16((B, S, H, D), seed=5)
    # head-major output [B, H, S, D] viewed as [B, S, H, D]
    ybuf = torch.empty((B, H, S, D), dtype=torch.bfloat16, device="cuda")
    y = ybuf.permute(0, 2, 1, 3)
    star.star_rope(x, y, 5e5, pos0=1000)
    xi = x.clone()
    star.star_rope(xi, xi, 5e5, pos0=1000)
    torch.cuda.synchronize()
    ref = orc.rope(x.cpu(), np.arange(1000, 1000 + S), 5e5, round_out=True)
    np.testing.assert_array_equal(to64(y), ref)
    assert torch.equal(xi, y.contiguous())


# ----------------------------------------------------------------------------- index math
@pytest.mark.parametrize("L,b,a", [(2048, 512, 512), (1000, 300, 100), (777, 256, 0), (64, 1, 1),
                                   (500, 1024, 0), (131072, 32768, 32768)])
def test_debug_index_is_bit_exact(L, b, a):
    blk, pos, rng = star.star_debug_index(L, b, a)
    torch.cuda.synchronize()
    oblk, orng = orc.phase1_ranges(L, b, a)
    np.testing.assert_array_equal(blk.cpu().numpy(), oblk)
    np.testing.assert_array_equal(pos.cpu().numpy(), np.arange(L))
    np.testing.assert_array_equal(rng.cpu().numpy(), orng)


# ----------------------------------------------------------------------------- LSE merge
@pytest.mark.parametrize("D", [64, 128])
def test_lse_merge_kernel(D):
    B, Hq, S, T = 2, 3, 5, 7
    g = torch.Generator().manual_seed(D)
    po = torch.randn(B, Hq, S, T, D, generator=g)
    pl = torch.randn(B, Hq, S, T, generator=g) * 3
    pl[0, 0, 1, :] = -float("inf")  # an empty split
    pl[1, 2, :, 3] = -float("inf")
    pl[1, 2, 4, 3] = 0.25            # only one live split for this row
    o = torch.empty(B, T, Hq, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, T, device="cuda")
    star.star_lse_merge(po.cuda(), pl.cuda(), o, lse)
    torch.cuda.synchronize()
    R = B * Hq * T
    po_r = po.permute(0, 1, 3, 2, 4).reshape(R, S, D).double().numpy()
    pl_r = pl.permute(0, 1, 3, 2).reshape(R, S).double().numpy()
    ro, rl = orc.lse_merge(po_r, pl_r)
    got_o = to64(o).transpose(0, 2, 1, 3).reshape(R, D)
    assert max_abs(got_o, ro) <= TOL_O
    assert max_abs(to64(lse).reshape(R), rl) <= TOL_LSE


# ----------------------------------------------------------------------------- bounded waits
def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait on a barrier nothing arrives on gives up after its limit and
    the host reads STAR_ERR_DEVICE_TIMEOUT; afterwards the context still runs
    kernels (a RoPE call checks out) and the status word reads clean."""
    from block_sparse_long_rope_b200 import _abi

    ws = star.alloc_workspace(256)
    star.star_debug_wait_probe(ws, seconds=0.05)
    with pytest.raises(_abi.StarError) as ei:
        star.star_device_status(ws)
    assert ei.value.name == "STAR_ERR_DEVICE_TIMEOUT"
    star.star_device_status(ws)  # read-back cleared the word
    x = rand_bf16((1, 4, 2, 64), seed=3)
    y = torch.empty_like(x)
    star.star_rope(x, y, 1e4)
    torch.cuda.synchronize()
    ref = orc.rope(x.cpu(), np.arange(4), 1e4, round_out=True)
    np.testing.assert_array_equal(to64(y), ref)
