"""Torch-tensor front end of the C ABI.

PyTorch provides device memory and the stream; every step of the computation
runs in the library's CUDA kernels. Functions here check shapes/dtypes,
allocate outputs and workspaces with torch, and pass raw pointers through
``_abi``. They refuse CPU tensors: there is no CPU implementation.
"""
from __future__ import annotations

import ctypes
import math
from typing import List, Optional, Sequence

import torch

from . import _abi

D_QK = 576
D_V = 512


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream: Optional[torch.cuda.Stream] = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("lightning_indexer_cross_b200 ops need CUDA tensors (no CPU path exists)")


def _need_dense(*ts):
    """Tensors handed to the library as raw pointers are read with dense
    row-major strides."""
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("lightning_indexer_cross_b200 ops need contiguous tensors")


def _need_dense_rows(*ts):
    """Caches may sit apart by a batch stride (dim 0) but are dense within."""
    for t in ts:
        if t is None:
            continue
        if not t[0].is_contiguous() or (t.shape[0] > 1 and t.stride(0) < t[0].numel()):
            raise ValueError("lightning_indexer_cross_b200 ops need caches dense within each batch entry")


def new_workspace(nbytes: int, device) -> torch.Tensor:
    """Zeroed byte workspace (the status word must start at IC_OK)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def indexer_score(q: torch.Tensor, w: torch.Tensor, k: torch.Tensor, k_scale: Optional[torch.Tensor] = None,
                  n_valid: Optional[torch.Tensor] = None, scores: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """scores[b,s] = sum_h w[b,h] ReLU(q[b,h] . k[s]). k: [Bk,N,d_I] bf16 or uint8 (e4m3 codes)."""
    _need_cuda(q, w, k, k_scale, n_valid, scores)
    _need_dense(q, w, n_valid, scores)
    _need_dense_rows(k, k_scale)
    B, H_I, d_I = q.shape
    Bk, N, dk = k.shape
    assert dk == d_I and Bk in (1, B)
    fp8 = k.dtype == torch.uint8
    assert q.dtype == torch.bfloat16 and w.dtype == torch.float32
    assert k.dtype in (torch.bfloat16, torch.uint8)
    assert k_scale is None or (fp8 and k_scale.dtype == torch.float32 and k_scale.shape == (Bk, N))
    if scores is None:
        scores = torch.empty((B, N), dtype=torch.float32, device=q.device)
    assert scores.shape == (B, N) and scores.dtype == torch.float32
    if workspace is None:
        workspace = new_workspace(_abi.ic_indexer_workspace_size(), q.device)
    kbs = k.stride(0) if Bk > 1 else 0
    sbs = (k_scale.stride(0) if (k_scale is not None and k_scale.shape[0] > 1) else 0)
    _abi.ic_indexer_score(_ptr(q), _ptr(w), _ptr(k), _ptr(k_scale), _abi.IC_FP8_E4M3 if fp8 else _abi.IC_BF16,
                          B, H_I, d_I, N, kbs, sbs, _ptr(n_valid), _ptr(scores), _ptr(workspace),
                          workspace.numel(), _stream_ptr(stream))
    return scores


def indexer_topk(q: torch.Tensor, w: torch.Tensor, k: torch.Tensor, topk: int,
                 k_scale: Optional[torch.Tensor] = None, n_valid: Optional[torch.Tensor] = None,
                 rows_per_pass: int = 0, idx: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The indexer and the top-k in one call: idx [B, topk] int32, the scores kept in a workspace scratch of
    rows_per_pass rows (0 = all rows)."""
    _need_cuda(q, w, k, k_scale, n_valid, idx)
    _need_dense(q, w, n_valid, idx)
    _need_dense_rows(k, k_scale)
    B, H_I, d_I = q.shape
    Bk, N, dk = k.shape
    assert dk == d_I and Bk in (1, B) and q.dtype == torch.bfloat16 and w.dtype == torch.float32
    fp8 = k.dtype == torch.uint8
    assert k.dtype in (torch.bfloat16, torch.uint8)
    assert k_scale is None or (fp8 and k_scale.dtype == torch.float32 and k_scale.shape == (Bk, N))
    if idx is None:
        idx = torch.empty((B, topk), dtype=torch.int32, device=q.device)
    assert idx.shape == (B, topk) and idx.dtype == torch.int32
    if workspace is None:
        workspace = new_workspace(_abi.ic_indexer_topk_workspace_size(B, N, topk, rows_per_pass), q.device)
    kbs = k.stride(0) if Bk > 1 else 0
    sbs = k_scale.stride(0) if (k_scale is not None and k_scale.shape[0] > 1) else 0
    _abi.ic_indexer_topk(_ptr(q), _ptr(w), _ptr(k), _ptr(k_scale), _abi.IC_FP8_E4M3 if fp8 else _abi.IC_BF16,
                         B, H_I, d_I, N, kbs, sbs, _ptr(n_valid), topk, int(rows_per_pass), _ptr(idx),
                         _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    return idx


def topk(scores: torch.Tensor, k: int, n_valid: Optional[torch.Tensor] = None,
         idx: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _need_cuda(scores, n_valid, idx)
    _need_dense(scores, n_valid, idx)
    B, N = scores.shape
    assert scores.dtype == torch.float32
    if idx is None:
        idx = torch.empty((B, k), dtype=torch.int32, device=scores.device)
    assert idx.shape == (B, k) and idx.dtype == torch.int32
    if workspace is None:
        workspace = new_workspace(_abi.ic_topk_workspace_size(B, N, k), scores.device)
    _abi.ic_topk(_ptr(scores), B, N, _ptr(n_valid), k, _ptr(idx), _ptr(workspace), workspace.numel(),
                 _stream_ptr(stream))
    return idx


def sparse_mla_decode(q: torch.Tensor, kv: torch.Tensor, idx: torch.Tensor, sink: torch.Tensor,
                      gate: Optional[torch.Tensor] = None, sm_scale: Optional[float] = None,
                      out_dtype: torch.dtype = torch.bfloat16, out: Optional[torch.Tensor] = None,
                      lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                      workspace: Optional[torch.Tensor] = None, stream=None):
    _need_cuda(q, kv, idx, sink, gate, out, lse)
    _need_dense(q, idx, sink, gate, out, lse)
    _need_dense_rows(kv)
    B, H, D = q.shape
    Bkv, N, Dk = kv.shape
    assert D == D_QK and Dk == D_QK and Bkv in (1, B)
    assert q.dtype == torch.bfloat16 and kv.dtype == torch.bfloat16 and idx.dtype == torch.int32
    assert sink.shape == (H,) and sink.dtype == torch.float32
    assert gate is None or (gate.shape == (B, H, D_V) and gate.dtype == torch.bfloat16)
    k = idx.shape[1]
    assert idx.shape == (B, k)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D_QK)
    if out is None:
        out = torch.empty((B, H, D_V), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    assert out.shape == (B, H, D_V) and out.dtype in (torch.bfloat16, torch.float32)
    assert lse is None or (lse.shape == (B, H) and lse.dtype == torch.float32)
    if workspace is None:
        workspace = new_workspace(_abi.ic_sparse_mla_workspace_size(B, H, k), q.device)
    od = _abi.IC_F32 if out.dtype == torch.float32 else _abi.IC_BF16
    kvs = kv.stride(0) if Bkv > 1 else 0
    _abi.ic_sparse_mla_decode(_ptr(q), _ptr(kv), kvs, N, _ptr(idx), k, _ptr(sink), _ptr(gate), float(sm_scale),
                              B, H, od, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                              _stream_ptr(stream))
    return out, lse


def decompress_gate(o_latent: torch.Tensor, wv_b: torch.Tensor, gate: Optional[torch.Tensor] = None,
                    out_dtype: torch.dtype = torch.bfloat16, out: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out[b,h] = sigmoid(gate[b,h]) * (wv_b[h] @ o_latent[b,h]): o_latent [B,H,512] bf16 (ungated attention
    output), wv_b [H,128,512] bf16, gate [B,H,128] bf16 or None."""
    _need_cuda(o_latent, wv_b, gate, out)
    _need_dense(o_latent, wv_b, gate, out)
    B, H, K = o_latent.shape
    Hw, d_v, Kw = wv_b.shape
    assert K == D_V and Kw == D_V and Hw == H
    assert o_latent.dtype == torch.bfloat16 and wv_b.dtype == torch.bfloat16
    assert gate is None or (gate.shape == (B, H, d_v) and gate.dtype == torch.bfloat16)
    if out is None:
        out = torch.empty((B, H, d_v), dtype=out_dtype, device=o_latent.device)
    assert out.shape == (B, H, d_v) and out.dtype in (torch.bfloat16, torch.float32)
    if workspace is None:
        workspace = new_workspace(_abi.ic_decompress_gate_workspace_size(), o_latent.device)
    _abi.ic_decompress_gate(_ptr(o_latent), _ptr(wv_b), _ptr(gate), B, H, d_v,
                            _abi.IC_F32 if out.dtype == torch.float32 else _abi.IC_BF16, _ptr(out), _ptr(workspace),
                            workspace.numel(), _stream_ptr(stream))
    return out


def cache_append(k_raw: torch.Tensor, ln_gamma: torch.Tensor, ln_beta: torch.Tensor, kv_raw: torch.Tensor,
                 pos: torch.Tensor, key_cache: torch.Tensor, kv_cache: torch.Tensor,
                 key_scale: Optional[torch.Tensor] = None, ln_eps: float = 1e-6, rope_base: float = 10000.0,
                 q: Optional[torch.Tensor] = None, q_pos: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Append T new tokens: LayerNorm-with-bias of k_raw [T, d_I] into row pos[t] of key_cache (bf16, or
    uint8 e4m3 codes with per-token key_scale), kv_raw [T, 576] into kv_cache with its rotary dims
    [512, 576) rotated (interleaved pairs) to pos[t]; if q [B, H, 576] is given, its rotary dims are
    rotated in place to q_pos[b]. Caches are [C, N, ...] with C == 1 (one shared cache) or C == T (token t
    writes cache t). Returns the workspace (its status word records out-of-range rows)."""
    _need_cuda(k_raw, ln_gamma, ln_beta, kv_raw, pos, key_cache, kv_cache, key_scale, q, q_pos)
    _need_dense(k_raw, ln_gamma, ln_beta, kv_raw, pos, q, q_pos)
    _need_dense_rows(key_cache, kv_cache, key_scale)
    T, d_I = k_raw.shape
    C, N, dk = key_cache.shape
    assert k_raw.dtype == torch.bfloat16 and kv_raw.dtype == torch.bfloat16 and kv_cache.dtype == torch.bfloat16
    assert ln_gamma.dtype == torch.float32 and ln_beta.dtype == torch.float32 and pos.dtype == torch.int64
    assert dk == d_I and kv_raw.shape == (T, D_QK) and kv_cache.shape == (C, N, D_QK) and C in (1, T)
    fp8 = key_cache.dtype == torch.uint8
    assert key_cache.dtype in (torch.bfloat16, torch.uint8) and (key_scale is not None) == fp8
    B = H = 0
    if q is not None:
        B, H, D = q.shape
        assert D == D_QK and q.dtype == torch.bfloat16 and q_pos is not None and q_pos.dtype == torch.int64
    if workspace is None:
        workspace = new_workspace(_abi.ic_cache_append_workspace_size(), k_raw.device)
    kbs = key_cache.stride(0) if C > 1 else 0
    sbs = key_scale.stride(0) if (fp8 and C > 1) else 0
    kvbs = kv_cache.stride(0) if C > 1 else 0
    _abi.ic_cache_append(_ptr(k_raw), _ptr(ln_gamma), _ptr(ln_beta), ln_eps,
                         _abi.IC_FP8_E4M3 if fp8 else _abi.IC_BF16, _ptr(key_cache), _ptr(key_scale), kbs, sbs,
                         _ptr(kv_raw), _ptr(kv_cache), kvbs, _ptr(pos), T, d_I, N, rope_base, _ptr(q), _ptr(q_pos),
                         B, H, _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    return workspace


def cp_candidates(scores: torch.Tensor, idx: torch.Tensor, offset: int, cand_score: Optional[torch.Tensor] = None,
                  cand_idx: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None):
    """(score, global position) of each local top-k entry of a shard: scores [B, N_local] fp32, idx [B, k]
    int32 shard positions (-1 padding), offset = global position of the shard's first token."""
    _need_cuda(scores, idx, cand_score, cand_idx)
    _need_dense(scores, idx, cand_score, cand_idx)
    B, N_local = scores.shape
    k = idx.shape[1]
    assert scores.dtype == torch.float32 and idx.dtype == torch.int32 and idx.shape[0] == B
    if cand_score is None:
        cand_score = torch.empty((B, k), dtype=torch.float32, device=scores.device)
    if cand_idx is None:
        cand_idx = torch.empty((B, k), dtype=torch.int32, device=scores.device)
    assert cand_score.shape == (B, k) and cand_idx.shape == (B, k)
    assert cand_score.dtype == torch.float32 and cand_idx.dtype == torch.int32
    if workspace is None:
        workspace = new_workspace(_abi.ic_cp_workspace_size(), scores.device)
    _abi.ic_cp_candidates(_ptr(scores), _ptr(idx), B, N_local, k, int(offset), _ptr(cand_score), _ptr(cand_idx),
                          _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    return cand_score, cand_idx


def cp_merge_topk(cand_score: torch.Tensor, cand_idx: torch.Tensor, k: int, lo: int = 0, hi: int = 0,
                  idx_global: Optional[torch.Tensor] = None, idx_local: Optional[torch.Tensor] = None,
                  want_local: bool = True, stream=None):
    """Global top-k of the gathered candidates [G, B, kin] (fp32 scores, int32 global positions): ties toward
    the lower global position; also the positions inside the shard [lo, hi) (-1 elsewhere)."""
    _need_cuda(cand_score, cand_idx, idx_global, idx_local)
    _need_dense(cand_score, cand_idx, idx_global, idx_local)
    G, B, kin = cand_score.shape
    assert cand_idx.shape == (G, B, kin) and cand_score.dtype == torch.float32 and cand_idx.dtype == torch.int32
    if idx_global is None:
        idx_global = torch.empty((B, k), dtype=torch.int32, device=cand_score.device)
    if idx_local is None and want_local:
        idx_local = torch.empty((B, k), dtype=torch.int32, device=cand_score.device)
    assert idx_global.shape == (B, k) and (idx_local is None or idx_local.shape == (B, k))
    _abi.ic_cp_merge_topk(_ptr(cand_score), _ptr(cand_idx), B * kin, G, B, kin, k, int(lo), int(hi),
                          _ptr(idx_global), _ptr(idx_local), _stream_ptr(stream))
    return idx_global, idx_local


def cp_combine(part_out: torch.Tensor, part_lse: torch.Tensor, sink: torch.Tensor,
               gate: Optional[torch.Tensor] = None, out_dtype: torch.dtype = torch.bfloat16,
               out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, want_lse: bool = False,
               stream=None):
    """Merge the ranks' partial attention outputs part_out [G, B, H, 512] fp32 (normalised, no sink) and
    part_lse [G, B, H] fp32: the sink added once, then the gate [B, H, 512] bf16."""
    _need_cuda(part_out, part_lse, sink, gate, out, lse)
    _need_dense(part_out, part_lse, sink, gate, out, lse)
    G, B, H, D = part_out.shape
    assert D == D_V and part_lse.shape == (G, B, H) and part_out.dtype == torch.float32
    assert part_lse.dtype == torch.float32 and sink.shape == (H,) and sink.dtype == torch.float32
    assert gate is None or (gate.shape == (B, H, D_V) and gate.dtype == torch.bfloat16)
    if out is None:
        out = torch.empty((B, H, D_V), dtype=out_dtype, device=part_out.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=part_out.device)
    assert out.shape == (B, H, D_V) and out.dtype in (torch.bfloat16, torch.float32)
    _abi.ic_cp_combine(_ptr(part_out), B * H * D_V, _ptr(part_lse), B * H, G, B, H, _ptr(sink), _ptr(gate),
                       _abi.IC_F32 if out.dtype == torch.float32 else _abi.IC_BF16, _ptr(out), _ptr(lse),
                       _stream_ptr(stream))
    return out, lse


def index_overlap(a: torch.Tensor, b: torch.Tensor, N: int, count: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    """Per row, the number of valid entries of b ([B, k] int32) that occur in a: [B] int32."""
    _need_cuda(a, b, count)
    _need_dense(a, b, count)
    assert a.dim() == 2 and a.shape == b.shape and a.dtype == torch.int32 and b.dtype == torch.int32
    B, k = a.shape
    if count is None:
        count = torch.empty((B,), dtype=torch.int32, device=a.device)
    assert count.shape == (B,) and count.dtype == torch.int32
    _abi.ic_index_overlap(_ptr(a), _ptr(b), B, k, int(N), _ptr(count), _stream_ptr(stream))
    return count


def reuse_overlap(layers: Sequence, schedule: str, topk: int, n_valid: Optional[torch.Tensor] = None,
                  rows_per_pass: int = 0, stream=None) -> dict:
    """The reuse diagnostic of a layer stack: for every S layer that carries
    indexer inputs, the overlap (per query, [B] int32) of the index it reuses
    -- the last preceding F layer's top-k -- with the top-k of its own
    indexer; recall = overlap / topk. Layers without indexer inputs (the
    stack's S layers normally) are skipped."""
    own, last, ws = {}, None, None
    for l, c in enumerate(schedule):
        lay = layers[l]
        if lay.q_idx is None:
            if c == "F":
                raise ValueError(f"F layer {l} has no indexer inputs")
            continue
        B, N = lay.q_idx.shape[0], lay.k_idx.shape[1]
        if ws is None:
            ws = new_workspace(_abi.ic_indexer_topk_workspace_size(B, N, topk, rows_per_pass), lay.q_idx.device)
        idx = indexer_topk(lay.q_idx, lay.w, lay.k_idx, topk, lay.k_scale, n_valid, rows_per_pass, workspace=ws,
                           stream=stream)
        if c == "F":
            last = idx
        elif last is not None:
            own[l] = index_overlap(last, idx, N, stream=stream)
    return own


class LayerStack:
    """Holds the per-layer pointer table, the shape struct, the index buffer
    and the workspace of one decode stack, so that a step is one C call."""

    def __init__(self, layers: Sequence, schedule: str, B: int, N: int, H_I: int, d_I: int, topk: int, H: int,
                 k_fp8: bool = False, shared_keys: bool = True, shared_kv: bool = True,
                 n_valid: Optional[torch.Tensor] = None, sm_scale: Optional[float] = None,
                 out_dtype: torch.dtype = torch.bfloat16, trace: bool = False, device="cuda",
                 want_lse: bool = False, rows_per_pass: int = 0):
        self.L = len(schedule)
        self.schedule = schedule.encode()
        self.layers = layers
        self.B, self.topk, self.H = B, topk, H
        dev = torch.device(device)
        self.outs: List[torch.Tensor] = [torch.empty((B, H, D_V), dtype=out_dtype, device=dev)
                                         for _ in range(self.L)]
        self.lses = [torch.empty((B, H), dtype=torch.float32, device=dev) if want_lse else None
                     for _ in range(self.L)]
        first_f = next(l for l in layers if l.k_idx is not None)
        first_kv = layers[0].kv
        sh = _abi.ic_stack_shape_t()
        sh.B, sh.N, sh.H_I, sh.d_I = B, N, H_I, d_I
        sh.k_dtype = _abi.IC_FP8_E4M3 if k_fp8 else _abi.IC_BF16
        sh.topk, sh.H = topk, H
        sh.sm_scale = float(sm_scale if sm_scale is not None else 1.0 / math.sqrt(D_QK))
        sh.out_dtype = _abi.IC_F32 if out_dtype == torch.float32 else _abi.IC_BF16
        sh.k_batch_stride = 0 if (shared_keys or B == 1) else first_f.k_idx.stride(0)
        sh.scale_batch_stride = 0 if (shared_keys or B == 1 or first_f.k_scale is None) else first_f.k_scale.stride(0)
        sh.kv_batch_stride = 0 if (shared_kv or B == 1) else first_kv.stride(0)
        sh.n_valid = None if n_valid is None else n_valid.data_ptr()
        sh.rows_per_pass = int(rows_per_pass)
        self.n_valid = n_valid
        self.shape = sh
        table = (_abi.ic_layer_t * self.L)()
        for l, lay in enumerate(layers):
            t = table[l]
            if schedule[l] == "F":
                t.q_idx, t.w, t.k_idx = lay.q_idx.data_ptr(), lay.w.data_ptr(), lay.k_idx.data_ptr()
                t.k_scale = None if lay.k_scale is None else lay.k_scale.data_ptr()
            t.q, t.kv, t.sink = lay.q.data_ptr(), lay.kv.data_ptr(), lay.sink.data_ptr()
            t.gate = None if lay.gate is None else lay.gate.data_ptr()
            t.out = self.outs[l].data_ptr()
            t.lse = None if self.lses[l] is None else self.lses[l].data_ptr()
        self.table = table
        self.index_buf = torch.empty((B, topk), dtype=torch.int32, device=dev)
        self.trace = torch.empty((self.L, B, topk), dtype=torch.int32, device=dev) if trace else None
        self.ws = new_workspace(_abi.ic_layer_stack_workspace_size(sh), dev)

    def set_wait_events(self, events: Optional[Sequence] = None) -> None:
        """Per-layer ``torch.cuda.Event`` objects (or None entries) that each
        step waits on before the layer's first kernel, e.g. events recorded
        after that layer's inputs were copied on another stream. ``None``
        clears them. Each event is recorded once here so that it has a
        handle; the caller re-records it every step."""
        for l in range(self.L):
            e = None if events is None else events[l]
            if e is not None and not e.cuda_event:
                e.record()
            self.table[l].wait_event = None if e is None else e.cuda_event
        self._events = events  # keep the events alive while the table points at them

    def step(self, stream=None) -> int:
        """Enqueue one decode step; returns the number of kernels enqueued."""
        _abi.ic_layer_stack(self.table, self.L, self.schedule, self.shape, _ptr(self.index_buf), _ptr(self.trace),
                            _ptr(self.ws), self.ws.numel(), _stream_ptr(stream))
        return _abi.ic_last_launch_count()

    def device_status(self, stream=None) -> int:
        return _abi.ic_last_device_status(_ptr(self.ws), _stream_ptr(stream))


def stack_from_workload(wl, trace: bool = False, out_dtype=torch.bfloat16, want_lse: bool = False,
                        rows_per_pass: int = 0) -> LayerStack:
    return LayerStack(wl.layers, wl.schedule, wl.B, wl.N, wl.H_I, wl.d_I, wl.topk, wl.H, k_fp8=wl.k_fp8,
                      shared_keys=wl.shared_keys, shared_kv=wl.shared_kv, n_valid=wl.n_valid,
                      sm_scale=wl.sm_scale, out_dtype=out_dtype, trace=trace,
                      device=wl.layers[0].q.device, want_lse=want_lse, rows_per_pass=rows_per_pass)
