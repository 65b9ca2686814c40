"""Context-parallel decode on CPU ranks (gloo): the cached tokens split over
2 and 3 ranks, each rank running the per-shard steps with the float64 oracle
in place of the CUDA kernels, the candidates and partial outputs exchanged
with all-gathers exactly as the NCCL path does. The merged indices must equal
the single-rank oracle's top-k over the whole cache (bit for bit as sets),
and the merged outputs the single-rank oracle's attention, on an F/S stack
with a shared cache, with per-query caches, and with causal limits that
leave some ranks without a valid token for some rows."""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleSteps:
    """The four per-rank steps of the context-parallel path, in float64 with
    the oracle (the GPU path runs the library's kernels instead)."""

    def local_candidates(self, q_idx, w, k_shard, k_scale, n_valid_local, topk, offset):
        import oracle
        fp8 = k_shard.dtype == torch.uint8
        sc = oracle.indexer_scores(q_idx, w, k_shard, k_scale, n_valid_local, keys_are_e4m3=fp8)
        idx = oracle.topk_indices(sc, topk, n_valid_local)
        cs = np.where(idx >= 0, np.take_along_axis(sc, np.maximum(idx, 0), axis=1), -np.inf)
        ci = np.where(idx >= 0, idx + offset, -1)
        return torch.from_numpy(cs), torch.from_numpy(ci)

    def merge(self, g_score, g_idx, topk, lo, hi):
        # k best of the gathered candidates: score descending, then global
        # position ascending; padding (-1) last
        G, B, kin = g_score.shape
        s = g_score.permute(1, 0, 2).reshape(B, G * kin).numpy()
        gi = g_idx.permute(1, 0, 2).reshape(B, G * kin).numpy()
        out = np.full((B, topk), -1, dtype=np.int64)
        for b in range(B):
            keep = gi[b] >= 0
            order = np.lexsort((gi[b][keep], -s[b][keep]))
            sel = gi[b][keep][order][:topk]
            out[b, :len(sel)] = sel
        loc = np.where((out >= lo) & (out < hi), out - lo, -1)
        return torch.from_numpy(out), torch.from_numpy(loc)

    def attend(self, q, kv_shard, idx_local, sm_scale):
        import oracle
        H = q.shape[1]
        # a sink of -1e300 contributes exactly 0 in float64: no sink term
        o, lse = oracle.sparse_mla(q, kv_shard, idx_local, np.full(H, -1e300), None, sm_scale)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def combine(self, g_out, g_lse, sink, gate, out_dtype):
        o, l = g_out.numpy(), g_lse.numpy()          # [G,B,H,512], [G,B,H]
        s = sink.double().numpy()
        M = np.maximum(s[None, :], l.max(axis=0))    # [B,H]
        wgt = np.exp(l - M[None])                    # [G,B,H]
        den = np.exp(s[None, :] - M) + wgt.sum(axis=0)
        out = (wgt[..., None] * o).sum(axis=0) / den[..., None]
        if gate is not None:
            out = out / (1.0 + np.exp(-gate.double().numpy()))
        return torch.from_numpy(out)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shard(t, lo, hi):
    return None if t is None else t[:, lo:hi]


def _worker(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import dataclasses
    import torch.distributed as dist

    import oracle
    from lightning_indexer_cross_b200 import workloads as W
    from lightning_indexer_cross_b200.context_parallel import ContextParallelDecode

    dist.init_process_group("gloo", rank=rank, world_size=world)
    res = "no result"
    try:
        n_valid = None
        if case == "stack_shared":
            wl = W.stack("cpu", seed=5, L=6, B=3, N=3001, H_I=8, d_I=64, topk=128, H=8, schedule="FFSFSS")
        elif case == "per_query_fp8":
            wl = W.long_context("cpu", seed=6, N=4099, B=2, H_I=8, d_I=64, topk=200, H=8, fp8=True, n_planted=8)
        else:  # causal: rows whose limit leaves the last ranks empty
            wl = W.stack("cpu", seed=7, L=2, B=4, N=2000, H_I=4, d_I=64, topk=100, H=8, schedule="FS")
            n_valid = torch.tensor([2000, 700, 150, 1], dtype=torch.int64)
        cp = ContextParallelDecode(wl.N, steps=OracleSteps(), sm_scale=wl.sm_scale)
        shards = [dataclasses.replace(lay, k_idx=_shard(lay.k_idx, cp.lo, cp.hi),
                                      k_scale=_shard(lay.k_scale, cp.lo, cp.hi),
                                      kv=_shard(lay.kv, cp.lo, cp.hi)) for lay in wl.layers]
        outs, traces = cp.layer_stack(shards, wl.schedule, wl.topk, n_valid=n_valid)
        res = None
        if rank == 0:
            ref = oracle.layer_stack(wl.layers, wl.schedule, wl.topk, n_valid=n_valid, sm_scale=wl.sm_scale,
                                     k_fp8=wl.k_fp8)
            worst = 0.0
            for l in range(wl.L):
                for b in range(wl.B):
                    got = set(traces[l][b].tolist()) - {-1}
                    exp = set(ref["idx"][l][b].tolist()) - {-1}
                    assert got == exp, (case, l, b)
                    assert int((traces[l][b] == -1).sum()) == int((ref["idx"][l][b] == -1).sum())
                r = ref["out"][l]
                err = np.abs(outs[l].numpy() - r).max() / max(np.abs(r).max(), 1e-300)
                worst = max(worst, float(err))
            res = worst
        else:
            res = 0.0
    except Exception as e:  # reported to the parent instead of a silent exit
        res = f"{type(e).__name__}: {e}"
    finally:
        q.put((rank, res))
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [(2, "stack_shared"), (3, "per_query_fp8"), (3, "causal")])
def test_context_parallel_equals_single_rank_oracle(world, case):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = dict(q.get(timeout=300) for _ in ps)
    for p in ps:
        p.join(timeout=60)
    assert all(not isinstance(v, str) for v in res.values()), res
    assert all(p.exitcode == 0 for p in ps)
    assert res[0] <= 1e-12, res[0]


def test_shard_bounds_cover_every_position_once():
    sys.path.insert(0, ROOT)
    from lightning_indexer_cross_b200.context_parallel import SHARD_ALIGN, local_limits, shard_bounds
    for N, G in [(100, 3), (1048576, 8), (7 * 16, 7), (131072, 2), (4099, 3)]:
        b = [shard_bounds(N, G, r) for r in range(G)]
        assert b[0][0] == 0 and b[-1][1] == N
        assert all(b[r][1] == b[r + 1][0] for r in range(G - 1))
        assert all(lo % SHARD_ALIGN == 0 and hi > lo for lo, hi in b)
        sizes = [hi - lo for lo, hi in b]
        assert max(sizes) - min(sizes) < 2 * SHARD_ALIGN
    with pytest.raises(ValueError):
        shard_bounds(40, 4, 0)
    nv = torch.tensor([0, 5, 10, 15])
    assert local_limits(nv, 5, 10).tolist() == [0, 0, 5, 5]
