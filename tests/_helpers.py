"""Comparison helpers for the parity tests (test infrastructure)."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances. Index sets: the GPU set may differ from the oracle's only in
# tokens whose oracle score lies within 1e-3 (relative) of the oracle's k-th
# score. Attention: max |gpu - ref| / max |ref| per (query, head) row,
# 2e-2 for bf16 outputs, 5e-3 for fp32 outputs.
TOPK_REL = 1e-3
ATTN_TOL = {torch.bfloat16: 2e-2, torch.float32: 5e-3}
# Indexer scores (no stated tolerance): the kernel accumulates bf16 products
# in fp32 over d_I terms, then sums H_I fp32 terms; against the float64 value
# the error is far below 1e-4 of the row's largest |score|.
SCORE_TOL = 1e-4


def index_sets_match(gpu_idx, ref_idx, ref_scores, k, n_valid=None):
    """Check one or more rows of top-k indices against the oracle's.

    Returns (ok, message). gpu_idx/ref_idx [B,k] (any order, -1 padded),
    ref_scores [B,N] float64 oracle scores.
    """
    g = np.asarray(gpu_idx.cpu() if isinstance(gpu_idx, torch.Tensor) else gpu_idx, dtype=np.int64)
    r = np.asarray(ref_idx, dtype=np.int64)
    s = np.asarray(ref_scores, dtype=np.float64)
    N = s.shape[1]
    nv = (np.full(g.shape[0], N) if n_valid is None else
          np.asarray(n_valid.cpu() if isinstance(n_valid, torch.Tensor) else n_valid, dtype=np.int64))
    for b in range(g.shape[0]):
        gv = g[b][g[b] >= 0]
        rv = r[b][r[b] >= 0]
        if np.any(g[b] < -1) or np.any(gv >= min(nv[b], N)):
            return False, f"row {b}: index outside [-1, n_valid)"
        if len(gv) != len(set(gv.tolist())):
            return False, f"row {b}: duplicate indices"
        if len(gv) != len(rv):
            return False, f"row {b}: {len(gv)} valid indices vs {len(rv)}"
        if len(rv) == 0:
            continue
        if nv[b] <= k:  # every valid position must be selected
            if set(gv.tolist()) != set(rv.tolist()):
                return False, f"row {b}: n_valid <= k but sets differ"
            continue
        t = s[b, rv].min()  # oracle's k-th score
        diff = set(gv.tolist()) ^ set(rv.tolist())
        if not diff:
            continue
        d = np.array(sorted(diff))
        if np.any(d >= s.shape[1]) or np.any(d < 0):
            return False, f"row {b}: out-of-range index"
        if t == 0:
            near = s[b, d] == 0
        else:
            near = np.abs(s[b, d] - t) <= TOPK_REL * abs(t)
        if not np.all(near):
            bad = d[~near][:5]
            return False, f"row {b}: {len(d)} differing tokens, not near k-th score: {bad} (t={t})"
    return True, ""


def attn_row_error(gpu_out, ref_out):
    """max |gpu - ref| / max |ref| per (b, h) row; returns the worst value."""
    g = gpu_out.float().cpu().numpy().astype(np.float64)
    r = np.asarray(ref_out, dtype=np.float64)
    num = np.abs(g - r).max(axis=-1)
    den = np.abs(r).max(axis=-1)
    den = np.where(den == 0, 1.0, den)
    return float((num / den).max())
