"""Context-parallel decode kernels on one GPU: G ranks emulated one after the
other in one process (each rank's shard steps through the library's
kernels; the all-gathers are replaced by stacking the ranks' tensors, so no
kernel waits on another). The merged top-k must equal the single-GPU top-k
exactly (the shard scores are the same fp32 values), every emulated rank
must select the same set, and the merged attention must match the oracle on
that set within the attention tolerance."""
import numpy as np
import pytest
import torch

import oracle
from lightning_indexer_cross_b200 import workloads as W
from tests._helpers import ATTN_TOL, attn_row_error

pytestmark = pytest.mark.gpu


def _emulate(wl, G, n_valid=None, out_dtype=torch.float32):
    from lightning_indexer_cross_b200.context_parallel import CudaSteps, local_limits, shard_bounds
    steps = CudaSteps()
    bounds = [shard_bounds(wl.N, G, r) for r in range(G)]
    outs, traces, per_rank_sets = [], [], []
    idx_g = idx_loc = None
    for l, lay in enumerate(wl.layers):
        if wl.schedule[l] == "F":
            cands = []
            for lo, hi in bounds:
                ks = None if lay.k_scale is None else lay.k_scale[:, lo:hi]
                cands.append(steps.local_candidates(lay.q_idx, lay.w, lay.k_idx[:, lo:hi], ks,
                                                    local_limits(n_valid, lo, hi), wl.topk, lo))
            gs = torch.stack([c[0] for c in cands])
            gi = torch.stack([c[1] for c in cands])
            merged = [steps.merge(gs, gi, wl.topk, lo, hi) for lo, hi in bounds]
            idx_g = merged[0][0]
            idx_loc = [m[1] for m in merged]
            per_rank_sets.append([[set(r.tolist()) for r in m[0].cpu()] for m in merged])
        parts = [steps.attend(lay.q, lay.kv[:, lo:hi], idx_loc[r], wl.sm_scale) for r, (lo, hi) in enumerate(bounds)]
        go = torch.stack([p[0] for p in parts])
        gl = torch.stack([p[1] for p in parts])
        outs.append(steps.combine(go, gl, lay.sink, lay.gate, out_dtype))
        traces.append(idx_g)
    torch.cuda.synchronize()
    return outs, traces, per_rank_sets


def _check(wl, G, n_valid=None, out_dtype=torch.float32):
    from lightning_indexer_cross_b200 import ops
    outs, traces, per_rank = _emulate(wl, G, n_valid, out_dtype)
    # every emulated rank selected the same set
    for sets in per_rank:
        assert all(s == sets[0] for s in sets)
    # the single-GPU path over the whole cache selects exactly the same sets
    st = ops.stack_from_workload(wl, trace=True, out_dtype=out_dtype)
    st.step()
    torch.cuda.synchronize()
    assert st.device_status() == 0
    for l in range(wl.L):
        for b in range(wl.B):
            assert set(traces[l][b].tolist()) == set(st.trace[l, b].tolist()), (l, b)
        lay = wl.layers[l]
        ref, _ = oracle.sparse_mla(lay.q, lay.kv, traces[l], lay.sink, lay.gate, wl.sm_scale)
        err = attn_row_error(outs[l], ref)
        assert err <= ATTN_TOL[out_dtype], f"layer {l}: attention row error {err:.3e}"


@pytest.mark.parametrize("G", [2, 8])
def test_cp_shared_cache_stack(cuda_dev, G):
    wl = W.stack(cuda_dev, seed=31, L=5, B=6, N=40000, topk=2048, schedule="FFSFS")
    _check(wl, G, out_dtype=torch.bfloat16)


def test_cp_per_query_caches_e4m3(cuda_dev):
    wl = W.long_context(cuda_dev, seed=32, N=60000, B=3, fp8=True, n_planted=16)
    _check(wl, 3)


def test_cp_causal_rows_with_empty_shards(cuda_dev):
    """Causal limits that leave the later ranks no valid token for some
    rows (their partial is empty: lse = -inf, weight 0), and a row with
    fewer valid tokens than k (padding)."""
    wl = W.stack(cuda_dev, seed=33, L=2, B=4, N=30000, topk=1024, schedule="FS")
    wl.n_valid = torch.tensor([30000, 9000, 700, 1], dtype=torch.int64, device=cuda_dev)
    _check(wl, 4, n_valid=wl.n_valid)
