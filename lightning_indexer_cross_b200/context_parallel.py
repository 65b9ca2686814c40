"""Context-parallel decode: the N cached tokens of every layer split over the
ranks of a torch.distributed process group, one GPU per rank, NCCL between
them.

Rank r holds the contiguous shard [lo_r, hi_r) of the token positions of the
indexer key cache and of the latent cache. The long-context decode is bound
by the indexer's pass over the whole cached past (Hy4 IndexCache explainer,
TL;DR and Jargon "Sparse attention"); split this way, each rank scores only
its shard. Per F layer:

1. every rank scores its shard and keeps its local top-k
   (``ic_indexer_score``, ``ic_topk``) and turns it into (score, global
   position) candidates (``ic_cp_candidates``);
2. one all-gather of the candidates ([G, B, k] scores and positions);
3. every rank selects the same global top-k from them
   (``ic_cp_merge_topk``, ties toward the lower global position): the k best
   tokens of a row are among the k best of their own shard, so the result is
   the single-GPU selection.

Per layer (F and S alike; S layers reuse the last F layer's selection):

4. every rank attends over the selected rows it owns, without the sink
   (``ic_sparse_mla_decode`` with sink -inf, fp32 output and lse);
5. one all-gather of the partial outputs and their lse;
6. ``ic_cp_combine`` merges them, adds e^{sink} once and applies the gate.

The exchanges are NCCL all-gathers of B*k*8 bytes (candidates) and
B*H*(512+1)*4 bytes (partials) per rank; no step reads another GPU's memory
directly. The compute steps go through the library's kernels (``CudaSteps``);
the class takes any object with the same four methods, which is how the
multi-rank logic is tested on CPU ranks.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import torch

D_QK = 576
D_V = 512


# Shards start at multiples of this many tokens, so that every shard's view
# of a cache (and of the e4m3 key scales, 4 bytes a token) starts on a
# 16-byte boundary as the library requires.
SHARD_ALIGN = 16


def shard_bounds(N: int, world: int, rank: int) -> Tuple[int, int]:
    """Rank `rank`'s positions [lo, hi) of N tokens split into `world`
    contiguous shards, each starting at a multiple of SHARD_ALIGN; sizes
    differ by less than 2 * SHARD_ALIGN."""
    if world < 1 or not (0 <= rank < world) or N < world * SHARD_ALIGN:
        raise ValueError(f"cannot split {N} tokens over {world} ranks (rank {rank})")

    def start(r):
        return N if r == world else (N * r // world) // SHARD_ALIGN * SHARD_ALIGN

    return start(rank), start(rank + 1)


def local_limits(n_valid: Optional[torch.Tensor], lo: int, hi: int) -> Optional[torch.Tensor]:
    """Causal limits [B] in shard coordinates: min(max(n_valid - lo, 0), hi - lo)."""
    if n_valid is None:
        return None
    return (n_valid - lo).clamp(0, hi - lo).contiguous()


class CudaSteps:
    """The per-rank compute steps through the library's CUDA kernels."""

    def local_candidates(self, q_idx, w, k_shard, k_scale, n_valid_local, topk: int, offset: int):
        from . import ops
        scores = ops.indexer_score(q_idx, w, k_shard, k_scale, n_valid_local)
        idx = ops.topk(scores, topk, n_valid_local)
        return ops.cp_candidates(scores, idx, offset)

    def merge(self, g_score, g_idx, topk: int, lo: int, hi: int):
        from . import ops
        return ops.cp_merge_topk(g_score, g_idx, topk, lo, hi)

    def attend(self, q, kv_shard, idx_local, sm_scale: float):
        from . import ops
        H = q.shape[1]
        no_sink = torch.full((H,), float("-inf"), dtype=torch.float32, device=q.device)
        return ops.sparse_mla_decode(q, kv_shard, idx_local, no_sink, None, sm_scale=sm_scale,
                                     out_dtype=torch.float32, want_lse=True)

    def combine(self, g_out, g_lse, sink, gate, out_dtype):
        from . import ops
        out, _ = ops.cp_combine(g_out, g_lse, sink, gate, out_dtype=out_dtype)
        return out


class ContextParallelDecode:
    """One rank's side of the context-parallel decode of N cached tokens.

    ``group``: the process group (default: the world); ``steps``: the compute
    steps (default ``CudaSteps``). Inputs are this rank's shards: key caches
    [Bk, hi - lo, d_I] (and e4m3 scales [Bk, hi - lo]), latent caches
    [Bkv, hi - lo, 576]; queries, weights, sinks and gates are the same on
    every rank.
    """

    def __init__(self, N: int, group=None, steps=None, sm_scale: Optional[float] = None):
        import torch.distributed as dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.N = int(N)
        self.lo, self.hi = shard_bounds(self.N, self.world, self.rank)
        self.steps = steps if steps is not None else CudaSteps()
        self.sm_scale = float(sm_scale if sm_scale is not None else 1.0 / math.sqrt(D_QK))

    def _all_gather(self, x: torch.Tensor) -> torch.Tensor:
        import torch.distributed as dist
        x = x.contiguous()
        out = torch.empty((self.world * x.shape[0],) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
        dist.all_gather_into_tensor(out, x, group=self.group)
        return out.view((self.world,) + tuple(x.shape))

    def select(self, q_idx, w, k_shard, k_scale=None, n_valid=None, topk: int = 2048):
        """Global top-k of an F layer: (idx_global [B, k], idx_local [B, k]);
        every rank gets the same idx_global."""
        nvl = local_limits(n_valid, self.lo, self.hi)
        cs, ci = self.steps.local_candidates(q_idx, w, k_shard, k_scale, nvl, topk, self.lo)
        return self.steps.merge(self._all_gather(cs), self._all_gather(ci), topk, self.lo, self.hi)

    def attention(self, q, kv_shard, idx_local, sink, gate=None, out_dtype=torch.bfloat16):
        """The layer's attention output [B, H, 512] (the same on every rank)."""
        o, lse = self.steps.attend(q, kv_shard, idx_local, self.sm_scale)
        return self.steps.combine(self._all_gather(o), self._all_gather(lse), sink, gate, out_dtype)

    def layer_stack(self, layers: Sequence, schedule: str, topk: int, n_valid=None,
                    out_dtype=torch.bfloat16) -> Tuple[List[torch.Tensor], List[torch.Tensor]]:
        """The F/S decode step over sharded layers (objects with the fields
        of ``workloads.Layer``, caches already sharded): S layers reuse the
        last preceding F layer's selection. Returns the per-layer outputs and
        the per-layer global index buffers."""
        if not schedule or schedule[0] != "F" or any(c not in "FS" for c in schedule):
            raise ValueError("schedule must be F/S characters starting with F")
        outs, traces = [], []
        idx_g = idx_l = None
        for l, lay in enumerate(layers):
            if schedule[l] == "F":
                idx_g, idx_l = self.select(lay.q_idx, lay.w, lay.k_idx, lay.k_scale, n_valid, topk)
            outs.append(self.attention(lay.q, lay.kv, idx_l, lay.sink, lay.gate, out_dtype))
            traces.append(idx_g)
        return outs, traces
