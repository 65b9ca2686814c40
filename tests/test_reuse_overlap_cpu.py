"""The reuse diagnostic's oracle (per-row overlap of two index sets and the
per-S-layer overlap of the reused index with the layer's own top-k), pinned
against set algebra it must obey, and the stack recipe's diagnostic options
(which must leave the stack's own inputs unchanged). CPU only."""
import numpy as np
import pytest
import torch

import oracle
from lightning_indexer_cross_b200 import workloads as W


def _rows(rng, B, k, N, pad=0.0, junk=0.0):
    out = np.empty((B, k), dtype=np.int64)
    for r in range(B):
        out[r] = rng.choice(N, k, replace=False)
        m = rng.random(k)
        out[r][m < pad] = -1
        out[r][(m >= pad) & (m < pad + junk)] = N + 7  # outside [0, N): ignored
    return out


def test_overlap_of_a_set_with_itself_counts_its_valid_entries():
    rng = np.random.default_rng(0)
    a = _rows(rng, 4, 300, 5000, pad=0.2, junk=0.05)
    got = oracle.index_overlap(a, a, 5000)
    want = [(row >= 0).sum() - (row == 5007).sum() for row in a]
    assert got.tolist() == want


def test_overlap_of_disjoint_sets_is_zero_and_is_symmetric_for_distinct_rows():
    a = np.arange(0, 200).reshape(1, 200)
    b = np.arange(200, 400).reshape(1, 200)
    assert oracle.index_overlap(a, b, 1000).tolist() == [0]
    rng = np.random.default_rng(1)
    x, y = _rows(rng, 6, 250, 3000, pad=0.1), _rows(rng, 6, 250, 3000, pad=0.1)
    assert oracle.index_overlap(x, y, 3000).tolist() == oracle.index_overlap(y, x, 3000).tolist()


def test_overlap_equals_numpy_intersection_sizes_and_ignores_order():
    rng = np.random.default_rng(2)
    N = 4000
    a, b = _rows(rng, 8, 400, N, pad=0.15, junk=0.03), _rows(rng, 8, 400, N, pad=0.15, junk=0.03)
    want = [np.intersect1d(a[r][(a[r] >= 0) & (a[r] < N)], b[r][(b[r] >= 0) & (b[r] < N)]).size for r in range(8)]
    assert oracle.index_overlap(a, b, N).tolist() == want
    perm = rng.permutation(400)
    assert oracle.index_overlap(a[:, perm], b[:, ::-1], N).tolist() == want


def _tiny_stack(schedule, **kw):
    return W.stack(device="cpu", seed=5, L=len(schedule), B=2, N=600, H_I=4, d_I=64, topk=40, H=8,
                   schedule=schedule, gate=False, **kw)


def test_reuse_overlap_is_complete_when_every_layer_scores_like_its_f_layer():
    """rho = 1 and keys shared across layers give an S layer the F layer's
    queries and keys; with the F layer's weights too, its own top-k is the
    reused one: full recall."""
    wl = _tiny_stack("FSS", rho=1.0, s_indexers=True, layer_keys="shared")
    for l in (1, 2):
        wl.layers[l].w = wl.layers[0].w
        assert torch.equal(wl.layers[l].q_idx, wl.layers[0].q_idx)
        assert wl.layers[l].k_idx is wl.layers[0].k_idx
    got = oracle.reuse_overlap(wl.layers, wl.schedule, wl.topk)
    assert sorted(got) == [1, 2]
    for l in (1, 2):
        assert got[l].tolist() == [wl.topk] * wl.B


def test_reuse_overlap_matches_the_oracle_topk_sets_and_skips_layers_without_indexers():
    wl = _tiny_stack("FSFSS", s_indexers=True)
    got = oracle.reuse_overlap(wl.layers, wl.schedule, wl.topk)
    own = {l: oracle.topk_indices(oracle.indexer_scores(lay.q_idx, lay.w, lay.k_idx), wl.topk)
           for l, lay in enumerate(wl.layers)}
    assert sorted(got) == [1, 3, 4]
    for l, gov in ((1, 0), (3, 2), (4, 2)):
        want = [len(set(own[gov][b].tolist()) & set(own[l][b].tolist())) for b in range(wl.B)]
        assert got[l].tolist() == want
    plain = _tiny_stack("FSFSS")
    assert oracle.reuse_overlap(plain.layers, plain.schedule, plain.topk) == {}


def test_diagnostic_options_leave_the_stacks_own_inputs_unchanged():
    base = _tiny_stack("FFSSF")
    diag = _tiny_stack("FFSSF", s_indexers=True)
    for l, c in enumerate("FFSSF"):
        a, b = base.layers[l], diag.layers[l]
        assert torch.equal(a.q, b.q) and torch.equal(a.kv, b.kv) and torch.equal(a.sink, b.sink)
        if c == "F":
            assert torch.equal(a.q_idx, b.q_idx) and torch.equal(a.w, b.w) and torch.equal(a.k_idx, b.k_idx)
        else:
            assert a.q_idx is None and b.q_idx is not None
