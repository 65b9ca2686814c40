"""Float64 oracle of the cache-append step (test infrastructure only).

The step that runs once per new token, just before the decode hot path: the
token's indexer key and its latent attention row are written into the two
caches, and the query's RoPE dims are rotated to its position.

Where each piece comes from (porting issue on Hy4-preview, "hy_v4 deltas"
bullets):

* "Indexer" bullet: the indexer key goes through a LayerNorm with bias, whose
  eps is the model's RMSNorm eps. The eps value is not printed; it is a
  parameter here (reading: 1e-6 by default).
* "RoPE is interleaved" bullet (is_neox_style=False): the rotated pairs are
  adjacent dims (2i, 2i+1), not the two halves. The pages name the MLA shape
  "RoPE-64, head 576" (first paragraph): the rotated dims are the last 64 of
  each 576-d row, [512, 576), of both the cached latent row and the query.
  The frequency base is not printed; reading: theta_i = base^(-2i/64) with
  base 10000 by default, angle = position * theta_i.
* fp8 keys: the e4m3 key cache with one fp32 scale per token. Reading: the
  scale is max|y| / 448 over the token's normalised key (1 when that max is
  0), codes = round-to-nearest-even of y / scale on the OCP E4M3 grid,
  saturating to +-448.

Precision: inputs are the exact bf16 bytes converted to float64; all
arithmetic is float64. Results are returned unrounded (the caches store bf16
or e4m3; tests judge the stored value against these exact ones).
"""
from __future__ import annotations

import math

import numpy as np

from .indexcache_oracle import _f64, decode_e4m3

E4M3_MAX = 448.0


def layernorm_bias(x, gamma, beta, eps: float) -> np.ndarray:
    """LayerNorm over the last axis with affine weight and bias:
    y = (x - mean(x)) / sqrt(mean((x - mean(x))^2) + eps) * gamma + beta
    (population variance, as LayerNorm defines it)."""
    x = _f64(x)
    g = _f64(gamma)
    b = _f64(beta)
    mu = x.mean(axis=-1, keepdims=True)
    d = x - mu
    var = (d * d).mean(axis=-1, keepdims=True)
    return d / np.sqrt(var + eps) * g + b


def _e4m3_grid():
    """The 127 non-negative finite E4M3 values with their codes, ascending."""
    codes = np.arange(0, 127, dtype=np.uint8)  # 0x00 .. 0x7E (0x7F is NaN)
    return codes, decode_e4m3(codes)


def encode_e4m3(x) -> np.ndarray:
    """Nearest E4M3 code of each value: ties go to the code with an even
    mantissa, magnitudes above 448 saturate to 448, the sign bit follows the
    sign of x (so negative values that round to zero give 0x80), NaN gives
    0x7F. Brute force over the grid, straight from the format definition."""
    x = np.asarray(x, dtype=np.float64)
    codes, vals = _e4m3_grid()
    out = np.empty(x.shape, dtype=np.uint8)
    flat_x = x.reshape(-1)
    flat_o = out.reshape(-1)
    for n, v in enumerate(flat_x):
        if math.isnan(v):
            flat_o[n] = 0x7F
            continue
        a = min(abs(v), E4M3_MAX)
        dist = np.abs(vals - a)
        best = np.flatnonzero(dist == dist.min())
        if len(best) > 1:  # exactly half way: the even mantissa wins
            best = [c for c in best if (codes[c] & 1) == 0]
        c = int(codes[best[0]])
        if math.copysign(1.0, v) < 0:
            c |= 0x80
        flat_o[n] = c
    return out


def rope_interleaved(x, pos, base: float = 10000.0) -> np.ndarray:
    """Rotate adjacent pairs (2i, 2i+1) of the last axis by pos * theta_i,
    theta_i = base^(-2i/d):  (a, b) -> (a cos - b sin, a sin + b cos).
    `pos` broadcasts against the leading axes of x."""
    x = _f64(x)
    d = x.shape[-1]
    assert d % 2 == 0
    i = np.arange(d // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def quantize_key_e4m3(y):
    """Per-token e4m3 quantisation of normalised keys y [T, d]: returns
    (codes [T, d] uint8, scale [T] float64) with scale = max|y| / 448 (1 for an
    all-zero row) and codes = encode_e4m3(y / scale)."""
    y = _f64(y)
    amax = np.abs(y).max(axis=-1)
    scale = np.where(amax > 0, amax / E4M3_MAX, 1.0)
    return encode_e4m3(y / scale[:, None]), scale


def cache_append(k_raw, gamma, beta, eps, kv_raw, pos, base=10000.0, d_v=512):
    """The whole step for T new tokens. Returns a dict with
    key  [T, d_I]  LayerNorm-with-bias of k_raw (exact),
    kv   [T, 576]  kv_raw with dims [d_v, 576) rotated to pos (exact),
    and, for the e4m3 cache, codes [T, d_I] / scale [T] of `key`."""
    key = layernorm_bias(k_raw, gamma, beta, eps)
    kv = _f64(kv_raw).copy()
    kv[:, d_v:] = rope_interleaved(kv[:, d_v:], np.asarray(pos), base)
    codes, scale = quantize_key_e4m3(key)
    return {"key": key, "kv": kv, "codes": codes, "scale": scale}


def rope_query(q, pos, base=10000.0, d_v=512):
    """Queries [B, H, 576] with dims [d_v, 576) rotated to pos[b] (exact)."""
    q = _f64(q).copy()
    q[:, :, d_v:] = rope_interleaved(q[:, :, d_v:], np.asarray(pos)[:, None], base)
    return q
