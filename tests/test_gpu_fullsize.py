"""Parity at the five workloads' full sizes, through the same C-ABI calls the
benchmark makes (ic_layer_stack). The oracle checks sampled queries and
layers one by one; properties that hold at any size (S-layer byte identity,
planted-token recovery, index range and uniqueness) are checked everywhere.
Every test here needs a B200 and a few GB of device memory."""
import numpy as np
import pytest
import torch

import oracle
from lightning_indexer_cross_b200 import workloads as W
from tests._helpers import ATTN_TOL, attn_row_error, index_sets_match

pytestmark = pytest.mark.gpu


def _ops():
    from lightning_indexer_cross_b200 import ops
    return ops


def _run(wl, out_dtype=torch.bfloat16, rows_per_pass=0):
    st = _ops().stack_from_workload(wl, trace=True, out_dtype=out_dtype, rows_per_pass=rows_per_pass)
    st.step()
    torch.cuda.synchronize()
    assert st.device_status() == 0
    return st


def _check_layer(wl, st, l, rows, check_index=True, per_row=False):
    """Oracle indexer + top-k for `rows` of the layer governing l (unless
    check_index is False, e.g. for an S layer whose governing F layer was
    checked), and oracle attention of layer l on the GPU's own index set.
    per_row: the oracle takes one query at a time (a 1M-token key cache is
    1 GB in float64)."""
    gov = oracle.governing_full_layer(wl.schedule)[l]
    f = wl.layers[gov]
    lay = wl.layers[l]
    trace = st.trace[l].cpu().numpy()
    if check_index:
        groups = [[b] for b in rows] if per_row else [list(rows)]
        for rs in groups:
            nv = None if wl.n_valid is None else wl.n_valid[rs]
            kk = f.k_idx if f.k_idx.shape[0] == 1 else f.k_idx[rs]
            ks = None if f.k_scale is None else (f.k_scale if f.k_scale.shape[0] == 1 else f.k_scale[rs])
            sc = oracle.indexer_scores(f.q_idx[rs], f.w[rs], kk, ks, nv, keys_are_e4m3=wl.k_fp8)
            ref_idx = oracle.topk_indices(sc, wl.topk, nv)
            ok, msg = index_sets_match(trace[rs], ref_idx, sc, wl.topk, nv)
            assert ok, f"layer {gov}, rows {rs[:4]}...: {msg}"
    # gather only the selected rows before handing them to the float64 oracle
    # (a whole cache would not fit in host memory as float64)
    idx = torch.as_tensor(trace[rows], device=lay.kv.device, dtype=torch.int64)
    cache = lay.kv[0] if lay.kv.shape[0] == 1 else None
    sel = []
    for i, b in enumerate(rows):
        src = cache if cache is not None else lay.kv[b]
        sel.append(src[idx[i].clamp_min(0)])
    kv_sel = torch.stack(sel)                               # [R, k, 576]
    idx_sel = torch.where(idx >= 0, torch.arange(idx.shape[1], device=idx.device), -1)
    gate = None if lay.gate is None else lay.gate[rows]
    ref, _ = oracle.sparse_mla(lay.q[rows], kv_sel, idx_sel, lay.sink, gate, wl.sm_scale)
    err = attn_row_error(st.outs[l][rows], ref)
    assert err <= ATTN_TOL[st.outs[l].dtype], f"layer {l}: attention row error {err:.3e}"


def _check_indices_valid(wl, st):
    tr = st.trace
    nv = torch.full((wl.B,), wl.N, device=tr.device) if wl.n_valid is None else wl.n_valid
    assert bool(((tr >= -1) & (tr < nv.view(1, -1, 1))).all())
    srt = tr.sort(dim=2).values
    dup = (srt[:, :, 1:] == srt[:, :, :-1]) & (srt[:, :, 1:] >= 0)
    assert not bool(dup.any())


def test_single_f_layer_model_shape(cuda_dev):
    """N=131072, 8 queries with their own caches, 64x128 indexer, k=2048,
    128 heads, gate: every query checked."""
    wl = W.single_f(cuda_dev)
    st = _run(wl)
    _check_indices_valid(wl, st)
    _check_layer(wl, st, 0, list(range(wl.B)))


@pytest.mark.parametrize("fp8", [False, True])
def test_long_context_1m(cuda_dev, fp8):
    """N=1,048,576, 4 queries with their own caches, bf16 and e4m3 keys:
    planted tokens (+4 sigma) recovered for every query, every query against
    the oracle (indexer, top-k, attention)."""
    wl = W.long_context(cuda_dev, fp8=fp8)
    st = _run(wl)
    _check_indices_valid(wl, st)
    for b in range(wl.B):
        assert set(wl.planted[b].tolist()) <= set(st.trace[0, b].tolist())
    _check_layer(wl, st, 0, list(range(wl.B)), per_row=True)


def test_prefill_chunk_causal(cuda_dev):
    """2048 causal queries over 264192 tokens, scored and selected 128 rows
    at a time (a 135 MB score scratch instead of 2.16 GB): 64 rows against
    the oracle (the first and last rows, then evenly spaced ones)."""
    wl = W.prefill(cuda_dev)
    st = _run(wl, rows_per_pass=128)
    from lightning_indexer_cross_b200 import _abi
    # the F layer's scores and top-k scratch: 128 rows at a time
    assert _abi.ic_indexer_topk_workspace_size(wl.B, wl.N, wl.topk, 128) < wl.B * wl.N * 4 // 8
    _check_indices_valid(wl, st)
    rows = sorted(set([0, 1, 2046, 2047] + [int(x) for x in np.linspace(3, 2045, 60)]))
    assert len(rows) == 64
    _check_layer(wl, st, 0, rows)


def test_stack78_decode(cuda_dev):
    """The 78-layer F/S stack the benchmark runs (B=32, N=131072): every S
    layer byte-identical to its governing F layer; every query of four F
    layers (the first, two inner ones, the last) against the oracle's indexer
    and top-k and attention, and every query's attention on four S layers."""
    wl = W.stack(cuda_dev)
    st = _run(wl)
    _check_indices_valid(wl, st)
    gov = oracle.governing_full_layer(wl.schedule)
    tr = st.trace.cpu().numpy()
    for l in range(wl.L):
        assert tr[l].tobytes() == tr[gov[l]].tobytes(), f"layer {l}"
    f_layers = [l for l in range(wl.L) if wl.schedule[l] == "F"]
    s_layers = [l for l in range(wl.L) if wl.schedule[l] == "S"]
    rows = list(range(wl.B))
    for l in (f_layers[0], f_layers[7], f_layers[14], f_layers[-1]):
        _check_layer(wl, st, l, rows)
    for l in (s_layers[0], s_layers[len(s_layers) // 3], s_layers[2 * len(s_layers) // 3], s_layers[-1]):
        _check_layer(wl, st, l, rows, check_index=False)
