"""ic_topk_noalloc: top-k for callers that cannot allocate device memory
(graph captures that forbid cudaMalloc, engine plugins handed only their
input and output buffers). It must give the same index sets as ic_topk,
call after call, although every call reuses the same built-in scratch.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test."""
import ctypes

import pytest
import torch

from lightning_indexer_cross_b200 import workloads as W


def _abi():
    from lightning_indexer_cross_b200 import build
    build.build()
    from lightning_indexer_cross_b200 import _abi as a
    return a


def _sets(idx):
    return [set(r[r >= 0].tolist()) for r in idx.cpu()]


@pytest.mark.gpu
def test_noalloc_topk_matches_workspace_topk_on_consecutive_calls(cuda_dev):
    a = _abi()
    from lightning_indexer_cross_b200 import ops
    stream = ops._stream_ptr()
    cases = [
        # B, N, k, ties, -inf fraction, causal: two calls in a row with
        # different shapes, so the second starts from the first's leftovers
        (32, 131072, 2048, False, 0.0, False),
        (7, 50001, 300, True, 0.2, True),
    ]
    for B, N, k, ties, ninf, causal in cases:
        s = W.scores_case(B, N, seed=B * 1000 + k, ties=ties, neg_inf_frac=ninf, device=cuda_dev)
        nv = None
        if causal:
            g = torch.Generator(device=cuda_dev).manual_seed(B)
            nv = torch.randint(0, N + 1, (B,), generator=g, device=cuda_dev, dtype=torch.int64)
        ref = ops.topk(s, k, nv)
        got = torch.full((B, k), -7, dtype=torch.int32, device=cuda_dev)
        a.ic_topk_noalloc(ctypes.c_void_p(s.data_ptr()), B, N,
                          None if nv is None else ctypes.c_void_p(nv.data_ptr()), k,
                          ctypes.c_void_p(got.data_ptr()), stream)
        torch.cuda.synchronize()
        # the selected set is deterministic (ties go to the lower index): exact match
        assert _sets(got) == _sets(ref)
        assert torch.equal((got == -1).sum(1), (ref == -1).sum(1))


def test_noalloc_topk_rejects_more_rows_than_its_scratch_holds():
    a = _abi()
    fake = (ctypes.c_float * 64)()
    p = ctypes.c_void_p(ctypes.addressof(fake))
    rows = a.IC_TOPK_NOALLOC_MAX_ROWS + 1
    # refused on the host, before any CUDA call: runs without a GPU
    assert a._topk_noalloc(p, rows, 1000, None, 10, p, None) == a.IC_ERR_UNSUPPORTED
    assert a._topk_noalloc(p, 2, 1000, None, 0, p, None) == a.IC_ERR_INVALID_ARG
