"""Pins of the cache-append oracle (LayerNorm with bias, e4m3 encoding,
interleaved RoPE) against library routines, closed forms and invariants.
CPU only."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import cache_append_oracle as A


def _rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------ LayerNorm
def test_layernorm_matches_torch_layer_norm():
    r = _rng(0)
    x = r.standard_normal((6, 128)) * 3 + 0.7
    g = r.standard_normal(128)
    b = r.standard_normal(128)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (128,), torch.from_numpy(g),
                                         torch.from_numpy(b), eps=1e-6).numpy()
    np.testing.assert_allclose(A.layernorm_bias(x, g, b, 1e-6), ref, rtol=1e-12, atol=1e-12)


def test_layernorm_unit_affine_gives_zero_mean_unit_variance():
    x = _rng(1).standard_normal((4, 64)) * 5 - 2
    y = A.layernorm_bias(x, np.ones(64), np.zeros(64), 0.0)
    np.testing.assert_allclose(y.mean(axis=-1), 0.0, atol=1e-12)
    np.testing.assert_allclose((y * y).mean(axis=-1), 1.0, rtol=1e-12)


def test_layernorm_affine_and_eps():
    x = _rng(2).standard_normal((3, 32))
    n = A.layernorm_bias(x, np.ones(32), np.zeros(32), 0.5)
    var = x.var(axis=-1, keepdims=True)
    np.testing.assert_allclose(n, (x - x.mean(axis=-1, keepdims=True)) / np.sqrt(var + 0.5), rtol=1e-12)
    g, b = np.full(32, 2.0), np.full(32, -3.0)
    np.testing.assert_allclose(A.layernorm_bias(x, g, b, 0.5), 2.0 * n - 3.0, rtol=1e-12)


def test_layernorm_constant_row_gives_the_bias():
    b = _rng(3).standard_normal(16)
    y = A.layernorm_bias(np.full((2, 16), 7.25), _rng(4).standard_normal(16), b, 1e-6)
    np.testing.assert_array_equal(y, np.broadcast_to(b, (2, 16)))


# ------------------------------------------------------------ e4m3 encoding
def test_e4m3_encode_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    np.testing.assert_array_equal(A.encode_e4m3(oracle.decode_e4m3(codes)), codes)


def test_e4m3_encode_matches_torch_cast_in_range():
    r = _rng(5)
    # random magnitudes over the whole exponent range plus every midpoint
    # between adjacent codes (the ties)
    x = np.concatenate([r.uniform(-448, 448, 4000),
                        np.exp2(r.uniform(-12, 8.8, 4000)) * r.choice([-1, 1], 4000)])
    vals = oracle.decode_e4m3(np.arange(0, 127, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2
    x = np.concatenate([x, mids, -mids]).astype(np.float32)  # all exactly representable in fp32
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(A.encode_e4m3(x.astype(np.float64)), ref)


def test_e4m3_encode_saturates_and_keeps_signs():
    np.testing.assert_array_equal(A.encode_e4m3([448.0, 460.0, 1000.0, 1e30, -500.0, math.inf, -math.inf]),
                                  [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7E, 0xFE])
    np.testing.assert_array_equal(A.encode_e4m3([0.0, -0.0, -1e-9, math.nan]), [0x00, 0x80, 0x80, 0x7F])


def test_e4m3_encode_is_monotone():
    x = np.linspace(-448, 448, 20001)
    v = oracle.decode_e4m3(A.encode_e4m3(x))
    assert np.all(np.diff(v) >= 0)
    # and within half a grid step of the input
    vals = oracle.decode_e4m3(np.arange(0, 127, dtype=np.uint8))
    j = np.clip(np.searchsorted(vals, np.abs(x), side="right") - 1, 0, len(vals) - 2)
    step = vals[j + 1] - vals[j]  # spacing of the grid interval holding |x|
    assert np.all(np.abs(v - x) <= step / 2 + 1e-12)


def test_key_quantisation_scale_and_extremes():
    y = _rng(6).standard_normal((5, 128))
    codes, scale = A.quantize_key_e4m3(y)
    np.testing.assert_allclose(scale, np.abs(y).max(axis=-1) / 448.0, rtol=1e-15)
    # the largest element of each row lands exactly on +-448
    am = np.abs(y).argmax(axis=-1)
    np.testing.assert_array_equal(codes[np.arange(5), am] & 0x7F, 0x7E)
    # decoded keys are within half a step (relative 1/16) of the exact ones
    back = oracle.decode_e4m3(codes) * scale[:, None]
    assert np.all(np.abs(back - y) <= np.maximum(np.abs(y) / 16, 2.0 ** -9 * scale[:, None]) + 1e-15)
    z_codes, z_scale = A.quantize_key_e4m3(np.zeros((1, 8)))
    np.testing.assert_array_equal(z_codes, 0)
    assert z_scale[0] == 1.0


# ------------------------------------------------------------ interleaved RoPE
def test_rope_matches_complex_rotation():
    r = _rng(7)
    x = r.standard_normal((9, 64))
    pos = r.integers(0, 1 << 20, 9)
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * np.outer(pos, 10000.0 ** (-np.arange(32) / 32.0)))
    out = A.rope_interleaved(x, pos)
    np.testing.assert_allclose(out[:, 0::2], z.real, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(out[:, 1::2], z.imag, rtol=1e-9, atol=1e-9)


def test_rope_position_zero_is_identity_and_pairs_keep_their_norm():
    x = _rng(8).standard_normal((3, 64))
    np.testing.assert_array_equal(A.rope_interleaved(x, np.zeros(3)), x)
    y = A.rope_interleaved(x, np.array([5, 1000, 131071]))
    np.testing.assert_allclose(np.hypot(y[:, 0::2], y[:, 1::2]), np.hypot(x[:, 0::2], x[:, 1::2]), rtol=1e-12)


def test_rope_first_pair_closed_form_and_adjacent_pairing():
    e1 = np.zeros(64)
    e1[1] = 1.0  # dim 1 pairs with dim 0 (interleaved), not with dim 33 (halves)
    y = A.rope_interleaved(e1[None], np.array([3]))[0]
    assert abs(y[0] + math.sin(3.0)) < 1e-15 and abs(y[1] - math.cos(3.0)) < 1e-15
    assert np.count_nonzero(y) == 2
    e62 = np.zeros(64)
    e62[62] = 1.0  # last pair: theta = base^(-62/64)
    y = A.rope_interleaved(e62[None], np.array([7]), base=500.0)[0]
    ang = 7 * 500.0 ** (-62 / 64)
    assert abs(y[62] - math.cos(ang)) < 1e-14 and abs(y[63] - math.sin(ang)) < 1e-14


def test_rope_scores_depend_only_on_relative_position():
    r = _rng(9)
    q, k = r.standard_normal(64), r.standard_normal(64)
    def s(p, t):
        return A.rope_interleaved(q[None], np.array([p]))[0] @ A.rope_interleaved(k[None], np.array([t]))[0]
    for p, t, sh in [(10, 3, 100), (5000, 4000, 77777), (0, 131071, 12)]:
        assert abs(s(p, t) - s(p + sh, t + sh)) < 1e-9 * max(1.0, abs(s(p, t)))


# ------------------------------------------------------------ the whole step
def test_cache_append_composes_the_pieces():
    r = _rng(10)
    T = 4
    k_raw = r.standard_normal((T, 128))
    g, b = r.standard_normal(128), r.standard_normal(128)
    kv_raw = r.standard_normal((T, 576))
    pos = np.array([0, 1, 4095, 131071])
    res = A.cache_append(k_raw, g, b, 1e-6, kv_raw, pos)
    np.testing.assert_array_equal(res["key"], A.layernorm_bias(k_raw, g, b, 1e-6))
    np.testing.assert_array_equal(res["kv"][:, :512], kv_raw[:, :512])  # latent dims untouched
    np.testing.assert_array_equal(res["kv"][0], kv_raw[0])              # position 0: no rotation
    np.testing.assert_allclose(res["kv"][:, 512:], A.rope_interleaved(kv_raw[:, 512:], pos))
    codes, scale = A.quantize_key_e4m3(res["key"])
    np.testing.assert_array_equal(res["codes"], codes)
    np.testing.assert_array_equal(res["scale"], scale)
    q = r.standard_normal((T, 8, 576))
    qr = A.rope_query(q, pos)
    np.testing.assert_array_equal(qr[:, :, :512], q[:, :, :512])
    np.testing.assert_allclose(qr[2, 5, 512:], A.rope_interleaved(q[2, 5, 512:][None], np.array([4095]))[0])
