"""Float64 oracle of the decompressed-space output gate (test infrastructure
only).

Porting issue on Hy4-preview, "hy_v4 deltas" gate bullet: the elementwise
sigmoid gate (linear_gate) multiplies the *decompressed* per-head attention
output, i.e. after the per-head value up-projection wv_b and before o_proj,
so a backend that folds wv_b into o_proj gates in the wrong space. The decode
path's attention produces the 512-d latent output of each head; this step
takes that (ungated) latent output to the head's value space and gates it
there:

    v[b, h, :]   = wv_b[h] @ o_latent[b, h, :]        wv_b [H, d_v, 512]
    out[b, h, :] = sigmoid(g[b, h, :]) * v[b, h, :]   g    [B, H, d_v]

The weight layout (out x in per head) and d_v are parameters; the pages give
neither (reading: d_v = 128 per head, synthetic weights).
"""
from __future__ import annotations

import numpy as np

from .indexcache_oracle import _f64


def _sigmoid(x):
    # exp(-x) overflows to inf for x < -709; 1 / (1 + inf) = 0 is then the exact limit
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def decompress(o_latent, wv_b) -> np.ndarray:
    """v[b,h,:] = wv_b[h] @ o_latent[b,h,:] (one matrix-vector product per head)."""
    o = _f64(o_latent)
    w = _f64(wv_b)
    B, H, K = o.shape
    assert w.shape[0] == H and w.shape[2] == K
    v = np.empty((B, H, w.shape[1]))
    for h in range(H):
        v[:, h, :] = o[:, h, :] @ w[h].T
    return v


def decompressed_gate(o_latent, wv_b, gate=None) -> np.ndarray:
    """sigmoid(gate) * (wv_b @ o_latent) per head; gate None means identity."""
    v = decompress(o_latent, wv_b)
    if gate is None:
        return v
    return _sigmoid(_f64(gate)) * v
