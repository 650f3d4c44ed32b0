"""Micro-benchmark of the library's projection GEMM on one GPU.

    python -m block_sparse_long_rope_b200.gemm_bench            # the shapes table
    python -m block_sparse_long_rope_b200.gemm_bench --once plain|rope|cache

The table times `star_linear` (y = x w^T, bf16 in and out, fp32 accumulation),
`star_linear_rope` writing rotated heads token-major and into a head-major
cache, and torch.matmul (cuBLAS) on the same operands, with CUDA events over
20 calls after 3 warm-up calls; it prints one JSON line per shape.
`--once` makes a single call of one form on 16384 x 4096 x 4096 and exits,
for a profiler to capture.
"""
import argparse
import json

SHAPES = [(16384, 4096, 4096), (16384, 1024, 4096), (4096, 4096, 4096), (65536, 4096, 4096)]
HEAD_DIM = 128
THETA = 5.0e5


def _timeit(torch, fn, reps=20, warm=3):
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def _operands(torch, M, N, K, dev):
    g = torch.Generator(device=dev).manual_seed(M * 31 + N * 7 + K)
    x = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, device=dev, generator=g) * K ** -0.5).to(torch.bfloat16)
    return x, w


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--once", choices=["plain", "rope", "cache"], default=None)
    args = ap.parse_args(argv)

    import torch

    from . import star

    dev = torch.device("cuda")
    ws = star.alloc_workspace(star.star_linear_rope_workspace_bytes(max(s[0] for s in SHAPES),
                                                                    HEAD_DIM, True))
    if args.once:
        M, N, K = SHAPES[0]
        x, w = _operands(torch, M, N, K, dev)
        if args.once == "plain":
            y = torch.empty(M, N, device=dev, dtype=torch.bfloat16)
            star.star_linear(x, w, y, workspace=ws)
        elif args.once == "rope":
            y = torch.empty(M, N, device=dev, dtype=torch.bfloat16)
            star.star_linear_rope(x, w, y, HEAD_DIM, True, M, 0, THETA, 0, ws)
        else:
            kc = torch.empty(1, N // HEAD_DIM, M + 8, HEAD_DIM, device=dev, dtype=torch.bfloat16)
            star.star_linear_rope(x, w, kc, HEAD_DIM, True, M, 0, THETA, M + 8, ws)
        torch.cuda.synchronize()
        star.star_device_status(ws)
        print(json.dumps({"once": args.once, "shape": [M, N, K]}))
        return

    for (M, N, K) in SHAPES:
        x, w = _operands(torch, M, N, K, dev)
        y = torch.empty(M, N, device=dev, dtype=torch.bfloat16)
        flops = 2.0 * M * N * K
        t_star = _timeit(torch, lambda: star.star_linear(x, w, y, workspace=ws))
        t_cublas = _timeit(torch, lambda: torch.matmul(x, w.t(), out=y))
        r = {"shape": [M, N, K], "star_linear_ms": t_star, "star_linear_tflops": flops / t_star / 1e9,
             "torch_matmul_ms": t_cublas, "torch_matmul_tflops": flops / t_cublas / 1e9}
        if N % HEAD_DIM == 0:
            kc = torch.empty(1, N // HEAD_DIM, M + 8, HEAD_DIM, device=dev, dtype=torch.bfloat16)
            t_cache = _timeit(torch, lambda: star.star_linear_rope(x, w, kc, HEAD_DIM, True, M, 0, THETA,
                                                                   M + 8, ws))
            t_tok = _timeit(torch, lambda: star.star_linear_rope(x, w, y, HEAD_DIM, True, M, 0, THETA, 0, ws))
            r.update({"star_linear_rope_cache_ms": t_cache, "star_linear_rope_ms": t_tok})
        star.star_device_status(ws)
        print(json.dumps({k: (round(v, 4) if isinstance(v, float) else v) for k, v in r.items()}), flush=True)


if __name__ == "__main__":
    main()
