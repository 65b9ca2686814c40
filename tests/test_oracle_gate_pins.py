"""Pins of the decompressed-space gate oracle against brute force, library
routines and closed forms. CPU only."""
import numpy as np
import scipy.special
import torch

import oracle
from oracle import gate_oracle as G


def _rng(seed):
    return np.random.default_rng(seed)


def test_decompress_matches_python_loops():
    r = _rng(0)
    o = r.standard_normal((2, 3, 5))
    w = r.standard_normal((3, 4, 5))
    v = G.decompress(o, w)
    for b in range(2):
        for h in range(3):
            for d in range(4):
                assert abs(v[b, h, d] - sum(w[h, d, k] * o[b, h, k] for k in range(5))) < 1e-12


def test_decompress_matches_torch_einsum():
    r = _rng(1)
    o = r.standard_normal((4, 8, 512))
    w = r.standard_normal((8, 128, 512)) / 22.6
    ref = torch.einsum("bhk,hdk->bhd", torch.from_numpy(o), torch.from_numpy(w)).numpy()
    np.testing.assert_allclose(G.decompress(o, w), ref, rtol=1e-12, atol=1e-12)


def test_gate_is_scipy_expit_times_values():
    r = _rng(2)
    o = r.standard_normal((3, 4, 16))
    w = r.standard_normal((4, 8, 16))
    g = r.standard_normal((3, 4, 8)) * 3
    np.testing.assert_allclose(G.decompressed_gate(o, w, g), scipy.special.expit(g) * G.decompress(o, w),
                               rtol=1e-13)
    np.testing.assert_array_equal(G.decompressed_gate(o, w, None), G.decompress(o, w))
    np.testing.assert_allclose(G.decompressed_gate(o, w, np.zeros((3, 4, 8))), G.decompress(o, w) / 2, rtol=1e-15)
    np.testing.assert_allclose(G.decompressed_gate(o, w, np.full((3, 4, 8), 50.0)), G.decompress(o, w), rtol=1e-15)


def test_identity_projection_reduces_to_the_latent_gate():
    # with wv_b = I the decompressed gate is the decode path's latent gate
    r = _rng(3)
    B, H, K = 2, 3, 512
    q = r.standard_normal((B, H, 576))
    kv = r.standard_normal((1, 40, 576))
    idx = np.stack([r.permutation(40)[:16] for _ in range(B)]).astype(np.int32)
    sink = r.standard_normal(H) * 0.5
    g = r.standard_normal((B, H, K))
    o_lat, _ = oracle.sparse_mla(q, kv, idx, sink, None)
    gated, _ = oracle.sparse_mla(q, kv, idx, sink, g)
    eye = np.broadcast_to(np.eye(K), (H, K, K))
    np.testing.assert_allclose(G.decompressed_gate(o_lat, eye, g), gated, rtol=1e-12, atol=1e-14)


def test_gate_commutes_with_the_projection_only_when_constant_per_head():
    r = _rng(4)
    o = r.standard_normal((2, 3, 64))
    w = r.standard_normal((3, 16, 64))
    c = r.standard_normal((2, 3, 1))
    # a gate constant over a head's dims is a scalar: either space gives the same
    const_dec = G.decompressed_gate(o, w, np.broadcast_to(c, (2, 3, 16)))
    const_lat = G.decompress(scipy.special.expit(np.broadcast_to(c, (2, 3, 64))) * o, w)
    np.testing.assert_allclose(const_dec, const_lat, rtol=1e-12)
    # a gate that varies over dims does not commute: gating the latent and
    # then projecting (what an absorbed backend does) is a different result
    g = r.standard_normal((2, 3, 16)) * 2
    g_lat = r.standard_normal((2, 3, 64)) * 2
    assert np.abs(G.decompressed_gate(o, w, g) - G.decompress(scipy.special.expit(g_lat) * o, w)).max() > 0.1
