"""The reuse diagnostic on a B200: ic_index_overlap against the oracle's set
overlap (exact: it is integer work), and the per-S-layer overlap of a small
stack against the GPU's own top-k sets and the oracle's."""
import numpy as np
import pytest
import torch

import oracle
from lightning_indexer_cross_b200 import workloads as W
from tests._helpers import index_sets_match

pytestmark = pytest.mark.gpu


def _ops():
    from lightning_indexer_cross_b200 import ops
    return ops


def _rows(g, B, k, N, dev, pad, junk):
    rows = torch.stack([torch.randperm(N, generator=g, device=dev)[:k] for _ in range(B)]).to(torch.int32)
    m = torch.rand((B, k), generator=g, device=dev)
    rows[m < pad] = -1
    rows[(m >= pad) & (m < pad + junk)] = N + 3  # outside [0, N): ignored
    return rows


@pytest.mark.parametrize("B,k,N,pad,junk,share", [
    (1, 1, 1, 0.0, 0.0, 1.0),
    (3, 2048, 131072, 0.0, 0.0, 0.5),
    (5, 777, 20000, 0.2, 0.05, 0.3),
    (2, 4096, 1048576, 0.1, 0.0, 0.9),
    (4, 1000, 1851392, 0.0, 0.01, 0.5),   # the largest N (one bit per position in shared memory)
    (33, 513, 3000, 0.3, 0.1, 0.0),
])
def test_index_overlap_equals_the_oracle(cuda_dev, B, k, N, pad, junk, share):
    g = torch.Generator(device=cuda_dev).manual_seed(B * 1000 + k)
    a = _rows(g, B, k, N, cuda_dev, pad, junk)
    b = _rows(g, B, k, N, cuda_dev, pad, junk)
    # b takes a share of a's entries (shuffled), so the overlaps are not all ~k^2/N
    n_sh = int(share * k)
    if n_sh:
        b[:, :n_sh] = a[:, torch.randperm(k, generator=g, device=cuda_dev)[:n_sh]]
    got = _ops().index_overlap(a, b, N)
    torch.cuda.synchronize()
    want = oracle.index_overlap(a.cpu().numpy(), b.cpu().numpy(), N)
    assert got.cpu().numpy().tolist() == want.tolist()


def test_reuse_overlap_of_a_small_stack(cuda_dev):
    """Schedule F S F S S over one shared cache per layer; keys shared across
    layers so that the overlaps are large and informative."""
    wl = W.stack(device=cuda_dev, seed=9, L=5, B=6, N=6000, H_I=64, d_I=128, topk=256, H=8,
                 schedule="FSFSS", gate=False, s_indexers=True, layer_keys="shared")
    ops = _ops()
    got = ops.reuse_overlap(wl.layers, wl.schedule, wl.topk)
    torch.cuda.synchronize()
    assert sorted(got) == [1, 3, 4]
    own = {l: ops.indexer_topk(lay.q_idx, lay.w, lay.k_idx, wl.topk).cpu().numpy()
           for l, lay in enumerate(wl.layers)}
    scores = {l: oracle.indexer_scores(lay.q_idx, lay.w, lay.k_idx) for l, lay in enumerate(wl.layers)}
    ref_sets = {l: oracle.topk_indices(sc, wl.topk) for l, sc in scores.items()}
    for l in scores:
        ok, msg = index_sets_match(own[l], ref_sets[l], scores[l], wl.topk)
        assert ok, msg
    ref = oracle.reuse_overlap(wl.layers, wl.schedule, wl.topk)
    for l, f in {1: 0, 3: 2, 4: 2}.items():
        # exactly the overlap of the GPU's own top-k sets
        exact = [len(set(own[f][b].tolist()) & set(own[l][b].tolist())) for b in range(wl.B)]
        assert got[l].cpu().numpy().tolist() == exact
        # and the oracle's, up to the entries the GPU's sets trade at near-ties
        slack = [len(set(own[f][b].tolist()) ^ set(ref_sets[f][b].tolist()))
                 + len(set(own[l][b].tolist()) ^ set(ref_sets[l][b].tolist())) for b in range(wl.B)]
        assert all(abs(e - r) <= sl for e, r, sl in zip(exact, ref[l].tolist(), slack))
