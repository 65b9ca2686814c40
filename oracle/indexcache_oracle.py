"""Float64 oracle of the IndexCache decode hot path (test infrastructure only).

What the path computes, and where each step comes from:

* Lightning indexer -- "a cheap indexer picks the handful of cached tokens
  each query will actually attend to" and "scores every cached position"
  (Hy4 IndexCache explainer, Q&A "What is IndexCache" and Jargon "Indexer").
  The pages name the indexer but print no formula; the score used here is the
  DeepSeek lightning-indexer form  score(s) = sum_h w_h * ReLU(q_h . k_s),
  with per-query head weights w and no extra 1/sqrt(d) factor (the inputs are
  pre-scaled).
* Top-k selection -- "keeping the k highest-scoring candidates" (explainer,
  Jargon "Top-k selection"); k = 2048 at model shape (porting issue on
  Hy4-preview, first paragraph: "RoPE-64, head 576, top-k 2048").
  Reading: ties are broken toward the lower token index; output order is not
  part of the result.
* IndexCache reuse -- later layers read the stored selection instead of
  rebuilding it (explainer, TL;DR and "The news"); shared-indexer layers reuse
  the last preceding full layer's top-k, pattern F F F S S S..., 21 full of 78
  (porting issue, "Indexer" bullet).
* DSA token-level sparse attention with the MLA shape -- each query attends to
  the individual selected tokens (explainer, Jargon "DSA"), rows of 576 =
  512 latent + 64 RoPE (porting issue, first paragraph), latent 512-d values.
* Learnable per-head sink, "softmax-denominator bias" (porting issue, sink
  bullet). Reading: a logit whose exponential joins the denominator,
  p_j = exp(z_j) / (exp(sink_h) + sum_j exp(z_j)); the sink is not scaled.
* Elementwise sigmoid gate multiplying the per-head attention output (porting
  issue, gate bullet). Reading: applied to the 512-d latent output,
  out = sigmoid(g) * o; gate = None means identity.

Precision: every input arrives already rounded to bf16 / e4m3 (the same bytes
the GPU reads) and is converted exactly to float64; all arithmetic is float64.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np


# ----------------------------------------------------------------------------
# fp8 e4m3 decoding (OCP 8-bit floating point, E4M3 variant): 1 sign bit,
# 4 exponent bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 NaN.
# ----------------------------------------------------------------------------
def decode_e4m3(codes) -> np.ndarray:
    """Decode e4m3 byte codes to float64, straight from the format definition."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = (1.0 + m / 8.0) * np.power(2.0, e - 7.0)
    subnormal = (m / 8.0) * 2.0 ** (1 - 7)
    mag = np.where(e == 0, subnormal, normal)
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def _f64(x) -> np.ndarray:
    """Exact conversion of a (possibly torch, possibly bf16) tensor to float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------
# Indexer
# ----------------------------------------------------------------------------
def indexer_scores(q, w, keys, key_scale=None, n_valid=None, keys_are_e4m3=False) -> np.ndarray:
    """score[b, s] = sum_h w[b,h] * max(0, sum_d q[b,h,d] * k[s,d]).

    q [B,H_I,d_I]; w [B,H_I]; keys [Bk,N,d_I] with Bk in {1, B} (1 = one cache
    shared by all queries); for e4m3 keys pass the uint8 codes with
    ``keys_are_e4m3=True`` and the per-token scale [Bk,N]: k[s,d] =
    decode(code[s,d]) * scale[s]. Positions s >= n_valid[b] are masked to -inf.
    The q.k contraction is one library matmul per query; ReLU, the head weights
    and the head sum follow the formula term by term.
    """
    q = _f64(q)
    w = _f64(w)
    if keys_are_e4m3:
        import torch
        codes = keys.detach().cpu().numpy() if isinstance(keys, torch.Tensor) else np.asarray(keys)
        k = decode_e4m3(codes)
        k = k * _f64(key_scale)[..., None]
    else:
        k = _f64(keys)
    B, H_I, d_I = q.shape
    Bk, N, _ = k.shape
    out = np.empty((B, N), dtype=np.float64)
    for b in range(B):
        kb = k[0 if Bk == 1 else b]            # [N, d_I]
        logits = q[b] @ kb.T                    # [H_I, N]  q_h . k_s
        relu = np.maximum(logits, 0.0)
        out[b] = w[b] @ relu                    # sum_h w_h * ReLU(.)
    if n_valid is not None:
        nv = np.asarray(_f64(n_valid), dtype=np.int64)
        for b in range(B):
            out[b, nv[b]:] = -np.inf
    return out


# ----------------------------------------------------------------------------
# Top-k
# ----------------------------------------------------------------------------
def topk_indices(scores, k: int, n_valid=None) -> np.ndarray:
    """The k highest scores of each row as token indices (int64 [B,k]).

    Rows are ranked by (score descending, index ascending) with a full sort;
    only positions < n_valid[b] compete. When fewer than k positions compete
    the row is padded with -1. Returned in rank order (rank order is not part
    of the result; comparisons are set-based).
    """
    s = _f64(scores)
    B, N = s.shape
    nv = np.full(B, N, dtype=np.int64) if n_valid is None else np.asarray(_f64(n_valid), dtype=np.int64)
    out = np.full((B, k), -1, dtype=np.int64)
    for b in range(B):
        n = int(min(max(nv[b], 0), N))
        # lexsort sorts by the last key first: primary -score, secondary index
        order = np.lexsort((np.arange(n), -s[b, :n]))
        take = order[:k]
        out[b, :len(take)] = take
    return out


# ----------------------------------------------------------------------------
# Sparse MLA attention with sink and gate
# ----------------------------------------------------------------------------
def _sigmoid(x):
    # exp(-x) overflows to inf for x < -709; 1 / (1 + inf) = 0 is then the exact limit
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def sparse_mla(q, kv, idx, sink, gate=None, sm_scale: Optional[float] = None, d_v: int = 512):
    """Attention of each query over only its selected rows.

    For query b, head h and selected tokens j (idx[b,j] >= 0):
      z_j   = sm_scale * sum_{d<576} q[b,h,d] * kv[idx_j, d]
      p_j   = exp(z_j) / (exp(sink_h) + sum_j exp(z_j))
      o     = sum_j p_j * kv[idx_j, 0:512]
      out   = sigmoid(gate[b,h]) * o          (gate None: out = o)
      lse   = log(exp(sink_h) + sum_j exp(z_j))
    kv is [Bkv,N,576] with Bkv in {1, B}. Returns (out [B,H,512], lse [B,H]).
    The max is subtracted before exponentiating (exact in real arithmetic).
    """
    q = _f64(q)
    kv = _f64(kv)
    idx = np.asarray(_f64(idx), dtype=np.int64)
    sink = _f64(sink)
    g = None if gate is None else _f64(gate)
    B, H, D = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    Bkv = kv.shape[0]
    out = np.zeros((B, H, d_v), dtype=np.float64)
    lse = np.zeros((B, H), dtype=np.float64)
    for b in range(B):
        sel = idx[b][idx[b] >= 0]
        rows = kv[0 if Bkv == 1 else b][sel]               # [k', 576]
        z = sm_scale * (q[b] @ rows.T)                      # [H, k']
        m = np.maximum(sink, z.max(axis=1) if z.shape[1] else -np.inf)  # [H]
        e = np.exp(z - m[:, None])
        den = np.exp(sink - m) + e.sum(axis=1)
        o = (e @ rows[:, :d_v]) / den[:, None]
        if g is not None:
            o = o * _sigmoid(g[b])
        out[b] = o
        lse[b] = m + np.log(den)
    return out, lse


def dense_sink_attention(q, kv, sink, gate=None, sm_scale: Optional[float] = None, d_v: int = 512):
    """Dense (full) attention of each query over every cached row, with the
    sink as one extra logit column whose value row is zero (explainer, scheme
    table: dense attention attends to every earlier token). Written as a
    softmax over the augmented logit matrix [sink | z]; independent of
    ``sparse_mla``'s gather-and-sum formulation."""
    q = _f64(q)
    kv = _f64(kv)
    sink = _f64(sink)
    g = None if gate is None else _f64(gate)
    B, H, D = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    Bkv, N, _ = kv.shape
    out = np.zeros((B, H, d_v))
    for b in range(B):
        K = kv[0 if Bkv == 1 else b]
        z = sm_scale * np.einsum("hd,nd->hn", q[b], K)
        aug = np.concatenate([sink[:, None], z], axis=1)          # [H, 1+N]
        aug = aug - aug.max(axis=1, keepdims=True)
        p = np.exp(aug)
        p = p / p.sum(axis=1, keepdims=True)
        V = np.concatenate([np.zeros((1, d_v)), K[:, :d_v]], axis=0)  # sink row is zero
        o = p @ V
        if g is not None:
            o = o * _sigmoid(g[b])
        out[b] = o
    return out


# ----------------------------------------------------------------------------
# IndexCache layer schedule
# ----------------------------------------------------------------------------
def validate_schedule(schedule: str) -> None:
    """A schedule is a string over {F, S}. Reading: it must start with F,
    because an S layer reuses "the last preceding full layer" (porting issue,
    indexer bullet), which does not exist for a leading S."""
    if not isinstance(schedule, str) or len(schedule) == 0:
        raise ValueError("schedule must be a non-empty string")
    bad = set(schedule) - {"F", "S"}
    if bad:
        raise ValueError(f"schedule has characters other than F/S: {sorted(bad)}")
    if schedule[0] != "F":
        raise ValueError("schedule must start with an F layer")


def governing_full_layer(schedule: str) -> List[int]:
    """For each layer, the index of the F layer whose top-k it uses."""
    validate_schedule(schedule)
    gov, last = [], -1
    for l, c in enumerate(schedule):
        if c == "F":
            last = l
        gov.append(last)
    return gov


def layer_stack(layers: Sequence, schedule: str, topk: int, n_valid=None,
                sm_scale: Optional[float] = None, k_fp8: bool = False) -> Dict:
    """Run the decode stack layer by layer following the F/S schedule.

    F layer: scores = indexer(q_idx, w, k_idx); idx = topk(scores) and the
    shared index buffer is overwritten. S layer: idx is the buffer as the last
    preceding F layer left it. Every layer then runs sparse MLA over idx.
    Returns per-layer index copies (so S-layer identity can be checked), the
    outputs, lse, and the number of indexer scores evaluated.
    """
    gov = governing_full_layer(schedule)
    idx_buf = None
    idx_per_layer, outs, lses = [], [], []
    n_scores = 0
    for l, c in enumerate(schedule):
        lay = layers[l]
        if c == "F":
            sc = indexer_scores(lay.q_idx, lay.w, lay.k_idx, lay.k_scale, n_valid,
                                keys_are_e4m3=k_fp8)
            B = sc.shape[0]
            nv = np.full(B, sc.shape[1]) if n_valid is None else np.asarray(_f64(n_valid), dtype=np.int64)
            n_scores += int(np.minimum(nv, sc.shape[1]).sum())
            idx_buf = topk_indices(sc, topk, n_valid)
        assert gov[l] >= 0
        idx_per_layer.append(idx_buf.copy())
        o, lse = sparse_mla(lay.q, lay.kv, idx_buf, lay.sink, lay.gate, sm_scale)
        outs.append(o)
        lses.append(lse)
    return {"idx": idx_per_layer, "out": outs, "lse": lses, "n_scores": n_scores,
            "governing": gov}


# ----------------------------------------------------------------------------
# Reuse diagnostic
# ----------------------------------------------------------------------------
def index_overlap(a, b, N: int) -> np.ndarray:
    """Per row, how many valid entries of b (in [0, N); -1 padding and
    anything else ignored) occur among the valid entries of a. Reuse is free
    only where nearby layers want the same tokens (Hy4 IndexCache explainer,
    the bet that sparse selections are largely shared between nearby layers);
    with a = the reused index and b = a layer's own top-k this counts what
    the reuse keeps (Bai et al. record: cross-layer reuse is not exact
    equality to each layer's own selection)."""
    a = np.asarray(_f64(a), dtype=np.int64)
    b = np.asarray(_f64(b), dtype=np.int64)
    out = np.zeros(a.shape[0], dtype=np.int64)
    for r in range(a.shape[0]):
        have = {int(x) for x in a[r] if 0 <= x < N}
        out[r] = sum(1 for x in b[r] if 0 <= x < N and int(x) in have)
    return out


def reuse_overlap(layers: Sequence, schedule: str, topk: int, n_valid=None, k_fp8: bool = False) -> Dict[int, np.ndarray]:
    """For each S layer that carries indexer inputs: index_overlap of the
    index it reuses (the last preceding F layer's top-k) with the top-k of
    its own indexer scores, per query."""
    gov = governing_full_layer(schedule)
    own = {}
    for l, c in enumerate(schedule):
        lay = layers[l]
        if lay.q_idx is None:
            continue
        sc = indexer_scores(lay.q_idx, lay.w, lay.k_idx, lay.k_scale, n_valid, keys_are_e4m3=k_fp8)
        own[l] = topk_indices(sc, topk, n_valid)
    N = layers[0].k_idx.shape[1]
    return {l: index_overlap(own[gov[l]], own[l], N) for l, c in enumerate(schedule) if c == "S" and l in own}

