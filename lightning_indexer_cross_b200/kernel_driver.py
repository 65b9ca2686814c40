"""Run one kernel family of the hot path on a fixed workload shape, for
profiling (e.g. under ``ncu -k regex:<kernel> -s <warm-up launches> -c 1``)
and quick timing.

    python -m lightning_indexer_cross_b200.kernel_driver --kernel indexer --shape stack --iters 3

Shapes: ``stack`` (one layer of the 78-layer stack: B=32 queries sharing
N=131072 keys, H_I=64, d_I=128, k=2048, H=128), ``single`` (B=8 queries with
their own caches, N=131072), ``long`` (B=4, N=1048576; ``--fp8`` for e4m3
keys). Every call runs ``--warmup`` untimed launches first, then ``--iters``
timed ones, and prints the mean time per call (CUDA events).
"""
from __future__ import annotations

import argparse

import torch

from . import ops
from . import workloads as W

SHAPES = {
    "stack": dict(B=32, N=131072, shared=True),
    "single": dict(B=8, N=131072, shared=False),
    "long": dict(B=4, N=1048576, shared=False),
}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", choices=["indexer", "topk", "mla"], required=True)
    ap.add_argument("--shape", choices=list(SHAPES), default="stack")
    ap.add_argument("--fp8", action="store_true")
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--iters", type=int, default=3)
    args = ap.parse_args()
    sh = SHAPES[args.shape]
    dev = torch.device("cuda:0")
    B, N, shared = sh["B"], sh["N"], sh["shared"]
    H_I, d_I, K, H = 64, 128, 2048, 128
    q, w, k, ks, _ = W.indexer_case(B, N, H_I, d_I, shared=shared, fp8=args.fp8, seed=5, device=dev)
    scores = ops.indexer_score(q, w, k, ks)
    idx = ops.topk(scores, K)
    torch.cuda.synchronize()
    if args.kernel == "indexer":
        ws = ops.new_workspace(256, dev)
        fn = lambda: ops.indexer_score(q, w, k, ks, scores=scores, workspace=ws)
    elif args.kernel == "topk":
        from . import _abi
        ws = ops.new_workspace(_abi.ic_topk_workspace_size(B, N, K), dev)
        fn = lambda: ops.topk(scores, K, idx=idx, workspace=ws)
    else:
        from . import _abi
        g = torch.Generator(device=dev).manual_seed(6)
        qa = torch.randn((B, H, W.D_QK), generator=g, device=dev).to(torch.bfloat16)
        kv = torch.randn((1 if shared else B, N, W.D_QK), generator=g, device=dev).to(torch.bfloat16)
        sink = torch.randn((H,), generator=g, device=dev) * 0.5
        gate = torch.randn((B, H, W.D_LATENT), generator=g, device=dev).to(torch.bfloat16)
        out = torch.empty((B, H, W.D_LATENT), dtype=torch.bfloat16, device=dev)
        ws = ops.new_workspace(_abi.ic_sparse_mla_workspace_size(B, H, K), dev)
        fn = lambda: ops.sparse_mla_decode(qa, kv, idx, sink, gate, out=out, want_lse=False, workspace=ws)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    print(f"{args.kernel} {args.shape}{' fp8' if args.fp8 else ''}: {e0.elapsed_time(e1) * 1000 / args.iters:.2f} us/call")


if __name__ == "__main__":
    main()
