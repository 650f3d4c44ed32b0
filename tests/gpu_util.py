"""Shared helpers of the GPU parity tests (tests only)."""
import numpy as np
import torch

TOL_O = 2e-2     # max-abs on bf16 outputs (and fp32 partial outputs)
TOL_LSE = 1e-3   # max-abs on fp32 LSE


def rand_bf16(shape, seed, scale=1.0, device="cuda"):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16).to(device)


def to64(t):
    return t.detach().float().cpu().double().numpy()


def max_abs(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    if a.size == 0:
        return 0.0
    return float(np.max(np.abs(a - b)))


def sample_rows(L, b, rng, extra=16):
    """Rows at every block start/end, 128-row tile edges around them, the
    first and last rows, plus random rows."""
    rows = {0, L - 1}
    n = -(-L // b)
    for i in range(n):
        s, e = i * b, min((i + 1) * b, L)
        for r in (s, s + 1, s + 127, s + 128, s + 255, e - 129, e - 128, e - 2, e - 1):
            if s <= r < e:
                rows.add(r)
    rows.update(int(x) for x in rng.integers(0, L, size=extra))
    return np.array(sorted(rows), dtype=np.int64)
