"""Seeded synthetic inputs (no arithmetic of the method lives here).

Every tensor is i.i.d. N(0, 1) drawn in fp32 from a seeded torch.Generator
and cast to bf16 (round to nearest even), as a QKV projection of a
Llama-shaped attention layer would emit it: Q [B, S, Hq, D] and
K, V [B, S, Hkv, D], token-major. The pages evaluate on RULER, BABILong and
InfiniteBench with trained Llama-3.1 weights; neither is available here, so
these shapes stand in for those layers.

Seed of one sequence's tensor = 1000 * config_index + 10 * sequence_index
+ tensor_id, with tensor_id q=0, k=1, v=2 (context) and q=3, k=4, v=5 (the
Phase-2 tokens). Each batch row is an independent sequence.
"""
import torch

TENSOR_ID = {"q": 0, "k": 1, "v": 2, "q2": 3, "k2": 4, "v2": 5}


def seed_for(config_index: int, seq_index: int, tensor_id: int) -> int:
    return 1000 * config_index + 10 * seq_index + tensor_id


def randn_bf16(shape, seed: int, device="cpu", scale: float = 1.0) -> torch.Tensor:
    """N(0, scale^2) samples drawn in fp32 on `device`, rounded to bf16."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(torch.bfloat16)


def make_tensor(name: str, B: int, S: int, H: int, D: int, config_index: int, device="cpu",
                scale: float = 1.0) -> torch.Tensor:
    """[B, S, H, D] bf16, one independent seed per sequence."""
    tid = TENSOR_ID[name]
    out = torch.empty((B, S, H, D), dtype=torch.bfloat16, device=device)
    for b in range(B):
        out[b] = randn_bf16((S, H, D), seed_for(config_index, b, tid), device=device, scale=scale)
    return out


def make_context(B, L, Hq, Hkv, D, config_index, device="cpu", q_scale=1.0):
    """Pre-RoPE context q[B,L,Hq,D], k/v[B,L,Hkv,D]."""
    q = make_tensor("q", B, L, Hq, D, config_index, device, q_scale)
    k = make_tensor("k", B, L, Hkv, D, config_index, device)
    v = make_tensor("v", B, L, Hkv, D, config_index, device)
    return q, k, v


def make_new_tokens(B, T, Hq, Hkv, D, config_index, device="cpu"):
    """Pre-RoPE q/k/v of the Phase-2 tokens (query chunk followed by decode
    tokens), [B, T, H, D]."""
    q = make_tensor("q2", B, T, Hq, D, config_index, device)
    k = make_tensor("k2", B, T, Hkv, D, config_index, device)
    v = make_tensor("v2", B, T, Hkv, D, config_index, device)
    return q, k, v


# ---- decoder stack (random, untrained weights) --------------------------------
STACK_ID = {"x": 0, "x2": 1, "gamma": 2, "wq": 3, "wk": 4, "wv": 5, "wo": 6}


def stack_seed(config_index: int, layer: int, tensor_id: int) -> int:
    return 100000 + 1000 * config_index + 10 * layer + tensor_id


def make_hidden(B: int, S: int, dm: int, config_index: int, name: str = "x",
                device="cpu") -> torch.Tensor:
    """Hidden states [B, S, dm] bf16, N(0, 1), drawn on the CPU (the same
    values on every device); name 'x' for the context, 'x2' for the
    Phase-2 tokens."""
    x = randn_bf16((B, S, dm), stack_seed(config_index, 999, STACK_ID[name]))
    return x.to(device)


def make_stack_weights(n_layers: int, dm: int, Hq: int, Hkv: int, D: int, config_index: int,
                       device="cpu"):
    """Per layer a dict: gamma [dm] ~ 1 + 0.1 N(0, 1); wq [Hq*D, dm], wk and
    wv [Hkv*D, dm] ~ N(0, 1/dm); wo [dm, Hq*D] ~ N(0, 1/(Hq*D)). bf16, drawn
    on the CPU."""
    layers = []
    for l in range(n_layers):
        s = lambda name: stack_seed(config_index, l, STACK_ID[name])  # noqa: E731
        g = torch.Generator().manual_seed(s("gamma"))
        gamma = (1.0 + 0.1 * torch.randn(dm, generator=g)).to(torch.bfloat16)
        layers.append({
            "gamma": gamma.to(device),
            "wq": randn_bf16((Hq * D, dm), s("wq"), scale=dm ** -0.5).to(device),
            "wk": randn_bf16((Hkv * D, dm), s("wk"), scale=dm ** -0.5).to(device),
            "wv": randn_bf16((Hkv * D, dm), s("wv"), scale=dm ** -0.5).to(device),
            "wo": randn_bf16((dm, Hq * D), s("wo"), scale=(Hq * D) ** -0.5).to(device),
        })
    return layers
