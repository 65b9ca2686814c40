"""Pins of the float64 oracle against things other than itself.

Each test checks the oracle against brute force on tiny inputs, a closed form,
a library routine, or a figure printed on the pages, so that a plausible slip
in the oracle (a dropped term, a wrong sign or index, a transposed operand)
fails at least one of them. CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import indexcache_oracle as O
from lightning_indexer_cross_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- e4m3 decode
def test_e4m3_decode_matches_torch_cast_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.decode_e4m3(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


@pytest.mark.parametrize("code,value", [
    (0x38, 1.0), (0xB8, -1.0), (0x7E, 448.0), (0x08, 2.0 ** -6), (0x01, 2.0 ** -9),
    (0x07, 7 * 2.0 ** -9), (0x3C, 1.5), (0x00, 0.0),
])
def test_e4m3_decode_known_values(code, value):
    # OCP 8-bit floating point spec, E4M3: bias 7, max normal 448, min normal
    # 2^-6, min subnormal 2^-9.
    assert O.decode_e4m3([code])[0] == value


# ---------------------------------------------------------------- indexer
def _brute_scores(q, w, k):
    B, H, D = len(q), len(q[0]), len(q[0][0])
    N = len(k[0])
    out = [[0.0] * N for _ in range(B)]
    for b in range(B):
        for s in range(N):
            tot = 0.0
            for h in range(H):
                dot = 0.0
                for d in range(D):
                    dot += q[b][h][d] * k[b if len(k) > 1 else 0][s][d]
                tot += w[b][h] * (dot if dot > 0 else 0.0)
            out[b][s] = tot
    return out


@pytest.mark.parametrize("shared", [False, True])
def test_indexer_matches_brute_force(shared):
    rng = np.random.default_rng(0)
    B, H, D, N = 2, 3, 5, 7
    q = rng.standard_normal((B, H, D))
    w = rng.standard_normal((B, H))  # signed weights too
    k = rng.standard_normal((1 if shared else B, N, D))
    ref = np.array(_brute_scores(q.tolist(), w.tolist(), k.tolist()))
    got = O.indexer_scores(q, w, k)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_indexer_single_head_single_dim_closed_form():
    q = np.array([[[0.75]]])
    w = np.array([[2.0]])
    k = np.array([[[-1.0], [0.0], [0.5], [4.0]]])
    got = O.indexer_scores(q, w, k)[0]
    assert list(got) == [0.0, 0.0, 2.0 * 0.375, 2.0 * 3.0]


def test_indexer_linear_in_w_and_relu_kills_negative():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((2, 4, 8))
    k = rng.standard_normal((2, 50, 8))
    w1, w2 = rng.random((2, 4)), rng.random((2, 4))
    s = O.indexer_scores(q, w1 + w2, k)
    np.testing.assert_allclose(s, O.indexer_scores(q, w1, k) + O.indexer_scores(q, w2, k), rtol=1e-12)
    # flipping every key sign swaps which heads pass the ReLU:
    # s(k) + s(-k) = sum_h w_h |q_h . k|
    s_neg = O.indexer_scores(q, w1, -k)
    absdot = np.einsum("bh,bhn->bn", w1, np.abs(np.einsum("bhd,bnd->bhn", q, k)))
    np.testing.assert_allclose(O.indexer_scores(q, w1, k) + s_neg, absdot, rtol=1e-12)


def test_indexer_fp8_path_equals_plain_path_on_representable_keys():
    rng = np.random.default_rng(2)
    codes = rng.integers(0, 256, size=(1, 40, 16), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38  # drop NaN codes
    vals = O.decode_e4m3(codes)
    q = rng.standard_normal((3, 4, 16))
    w = rng.random((3, 4))
    ones = np.ones((1, 40))
    a = O.indexer_scores(q, w, torch.from_numpy(codes), ones, keys_are_e4m3=True)
    b = O.indexer_scores(q, w, vals)
    np.testing.assert_array_equal(a, b)
    # positive per-token scale factors out of the head sum
    sc = rng.random((1, 40)) + 0.1
    c = O.indexer_scores(q, w, torch.from_numpy(codes), sc, keys_are_e4m3=True)
    np.testing.assert_allclose(c, b * sc, rtol=1e-12)


def test_indexer_causal_mask():
    rng = np.random.default_rng(3)
    q, w, k = rng.standard_normal((3, 2, 4)), rng.random((3, 2)), rng.standard_normal((1, 10, 4))
    s = O.indexer_scores(q, w, k, n_valid=np.array([10, 4, 0]))
    assert np.all(np.isfinite(s[0]))
    assert np.all(np.isfinite(s[1, :4])) and np.all(s[1, 4:] == -np.inf)
    assert np.all(s[2] == -np.inf)


# ---------------------------------------------------------------- top-k
def test_topk_matches_python_sorted():
    rng = np.random.default_rng(4)
    s = rng.standard_normal((3, 200))
    got = O.topk_indices(s, 17)
    for b in range(3):
        ref = sorted(range(200), key=lambda i: (-s[b, i], i))[:17]
        assert list(got[b]) == ref


def test_topk_ties_go_to_lower_index():
    s = np.array([[1.0, 3.0, 3.0, 2.0, 3.0, 3.0]])
    assert list(O.topk_indices(s, 3)[0]) == [1, 2, 4]
    assert list(O.topk_indices(np.zeros((1, 10)), 4)[0]) == [0, 1, 2, 3]


def test_topk_pads_when_fewer_valid_than_k():
    s = np.arange(10, dtype=np.float64)[None].repeat(2, 0)
    got = O.topk_indices(s, 6, n_valid=np.array([3, 10]))
    assert sorted(got[0][:3]) == [0, 1, 2] and list(got[0][3:]) == [-1, -1, -1]
    assert list(got[1]) == [9, 8, 7, 6, 5, 4]


def test_topk_permutation_invariance():
    rng = np.random.default_rng(5)
    s = rng.standard_normal((1, 500))
    perm = rng.permutation(500)
    a = set(O.topk_indices(s, 50)[0])
    b = set(perm[O.topk_indices(s[:, perm], 50)[0]])
    assert a == b


def test_topk_neg_inf_ranked_last():
    s = np.array([[-np.inf, 0.5, -np.inf, -3.0]])
    assert list(O.topk_indices(s, 3)[0]) == [1, 3, 0]


# ---------------------------------------------------------------- planted tokens
def _planted_z(s_row, planted):
    """z-scores of the planted positions against the unplanted scores."""
    mask = np.ones(s_row.shape[0], bool)
    mask[planted] = False
    return (s_row[planted] - s_row[mask].mean()) / s_row[mask].std()


def test_planted_tokens_recovered_tiny_workload():
    """Tiny recipe: planted keys "aligned to q, score +4 sigma". The oracle's
    scores put every planted token at 3.9..4.1 standard deviations above the
    mean of the 4088 unplanted ones, and top-256 keeps all 8."""
    wl = W.tiny("cpu")
    lay = wl.layers[0]
    s = O.indexer_scores(lay.q_idx, lay.w, lay.k_idx)
    planted = wl.planted[0].numpy()
    z = _planted_z(s[0], planted)
    assert np.all((z >= 3.9) & (z <= 4.1)), z
    top = set(O.topk_indices(s, wl.topk)[0])
    assert set(planted) <= top


def test_planted_tokens_long_context_recipe_small():
    """The long-context recipe at a reduced N, bf16 and e4m3 keys: planted
    z-scores in [3.9, 4.1] (for e4m3 on the stored, quantised keys) and
    every planted token recovered."""
    for fp8 in (False, True):
        wl = W.long_context("cpu", N=32768, B=2, H=8, fp8=fp8, n_planted=16)
        lay = wl.layers[0]
        s = O.indexer_scores(lay.q_idx, lay.w, lay.k_idx, lay.k_scale, keys_are_e4m3=fp8)
        for b in range(wl.B):
            z = _planted_z(s[b], wl.planted[b].numpy())
            assert np.all((z >= 3.9) & (z <= 4.1)), (fp8, b, z)
            top = set(O.topk_indices(s[b:b + 1], wl.topk)[0])
            assert set(wl.planted[b].numpy()) <= top


def test_planting_moments_match_the_oracle_scores_of_random_keys():
    """The closed-form mean and standard deviation used to place planted keys
    agree with the oracle's scores of 65536 keys drawn from the recipe's
    distribution (no planted keys), within sampling error."""
    q, w, k, _, _ = W.indexer_case(3, 65536, 64, 128, seed=77)
    s = O.indexer_scores(q, w, k)
    mu, sd = W.unplanted_score_moments(q, w, 1.0 / np.sqrt(128))
    for b in range(3):
        assert abs(s[b].mean() - float(mu[b])) <= 0.02 * float(sd[b])
        assert abs(s[b].std() / float(sd[b]) - 1.0) <= 0.02


# ---------------------------------------------------------------- sparse MLA
def _rand_attn(rng, B=2, H=3, N=40, D=576, Bkv=None):
    Bkv = B if Bkv is None else Bkv
    q = rng.standard_normal((B, H, D))
    kv = rng.standard_normal((Bkv, N, D))
    sink = 0.5 * rng.standard_normal(H)
    return q, kv, sink


def test_sparse_with_every_token_equals_dense():
    rng = np.random.default_rng(6)
    q, kv, sink = _rand_attn(rng, B=2, H=4, N=33)
    gate = rng.standard_normal((2, 4, 512))
    idx = np.stack([rng.permutation(33), rng.permutation(33)])
    a, _ = O.sparse_mla(q, kv, idx, sink, gate, 0.05)
    b = O.dense_sink_attention(q, kv, sink, gate, 0.05)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-13)


def test_sparse_equal_rows_closed_form():
    # every selected row equal: o = v * S / (e^sink + S), S = sum_j e^{z_j}
    rng = np.random.default_rng(7)
    row = rng.standard_normal(576)
    kv = np.tile(row, (1, 20, 1))
    q = rng.standard_normal((1, 2, 576))
    sink = np.array([0.3, -0.7])
    idx = np.arange(0, 20, 2)[None]
    out, _ = O.sparse_mla(q, kv, idx, sink, None, 0.04)
    z = 0.04 * q[0] @ row                      # same logit for all 10 rows
    S = 10 * np.exp(z)
    exp = row[None, :512] * (S / (np.exp(sink) + S))[:, None]
    np.testing.assert_allclose(out[0], exp, rtol=1e-12)


def test_sparse_zero_query_closed_form():
    # q = 0: every logit is 0, o = mean(V) * k / (k + e^sink)
    rng = np.random.default_rng(8)
    kv = rng.standard_normal((1, 30, 576))
    q = np.zeros((1, 3, 576))
    sink = np.array([0.0, 1.0, -2.0])
    idx = np.array([[3, 7, 11, 29, 0]])
    out, lse = O.sparse_mla(q, kv, idx, sink)
    mean = kv[0, idx[0], :512].mean(axis=0)
    for h in range(3):
        np.testing.assert_allclose(out[0, h], mean * 5 / (5 + np.exp(sink[h])), rtol=1e-12)
        assert lse[0, h] == pytest.approx(math.log(5 + math.exp(sink[h])), rel=1e-13)


def test_sparse_sink_to_minus_infinity_is_plain_softmax():
    rng = np.random.default_rng(9)
    q, kv, _ = _rand_attn(rng, B=1, H=2, N=25)
    idx = rng.permutation(25)[:12][None]
    out, _ = O.sparse_mla(q, kv, idx, np.array([-np.inf, -1e300]), None, 0.05)
    z = 0.05 * q[0] @ kv[0, idx[0]].T
    ref = scipy.special.softmax(z, axis=1) @ kv[0, idx[0], :512]
    np.testing.assert_allclose(out[0], ref, rtol=1e-11)


def test_sparse_gate_limits():
    rng = np.random.default_rng(10)
    q, kv, sink = _rand_attn(rng, B=1, H=2, N=25)
    idx = rng.permutation(25)[:9][None]
    base, _ = O.sparse_mla(q, kv, idx, sink, None)
    big, _ = O.sparse_mla(q, kv, idx, sink, np.full((1, 2, 512), 800.0))
    half, _ = O.sparse_mla(q, kv, idx, sink, np.zeros((1, 2, 512)))
    neg, _ = O.sparse_mla(q, kv, idx, sink, np.full((1, 2, 512), -800.0))
    np.testing.assert_array_equal(big, base)
    np.testing.assert_allclose(half, 0.5 * base, rtol=1e-15)
    assert np.abs(neg).max() < 1e-300
    g = rng.standard_normal((1, 2, 512))
    gated, _ = O.sparse_mla(q, kv, idx, sink, g)
    np.testing.assert_allclose(gated, base * scipy.special.expit(g), rtol=1e-13)


def test_sparse_lse_matches_scipy_logsumexp():
    rng = np.random.default_rng(11)
    q, kv, sink = _rand_attn(rng, B=2, H=3, N=30)
    idx = np.stack([rng.permutation(30)[:10] for _ in range(2)])
    _, lse = O.sparse_mla(q, kv, idx, sink, None, 0.07)
    for b in range(2):
        z = 0.07 * q[b] @ kv[b, idx[b]].T
        ref = scipy.special.logsumexp(np.concatenate([sink[:, None], z], axis=1), axis=1)
        np.testing.assert_allclose(lse[b], ref, rtol=1e-13)


def test_sparse_matches_brute_force_loops():
    rng = np.random.default_rng(12)
    B, H, N, k = 2, 2, 12, 5
    q, kv, sink = _rand_attn(rng, B=B, H=H, N=N, Bkv=1)
    gate = rng.standard_normal((B, H, 512))
    idx = np.stack([rng.permutation(N)[:k] for _ in range(B)])
    out, _ = O.sparse_mla(q, kv, idx, sink, gate, 0.1)
    for b in range(B):
        for h in range(H):
            zs = []
            for j in idx[b]:
                zs.append(0.1 * sum(q[b, h, d] * kv[0, j, d] for d in range(576)))
            den = math.exp(sink[h]) + sum(math.exp(z) for z in zs)
            for d in (0, 1, 255, 511):
                o = sum(math.exp(z) * kv[0, j, d] for z, j in zip(zs, idx[b])) / den
                o *= 1.0 / (1.0 + math.exp(-gate[b, h, d]))
                assert out[b, h, d] == pytest.approx(o, rel=1e-10, abs=1e-13)


def test_sparse_padding_is_skipped():
    rng = np.random.default_rng(13)
    q, kv, sink = _rand_attn(rng, B=1, H=2, N=20)
    idx = np.array([[4, 9, 13, -1, -1]])
    a, la = O.sparse_mla(q, kv, idx, sink)
    b, lb = O.sparse_mla(q, kv, idx[:, :3], sink)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(la, lb)
    # all padding: output 0, lse = sink
    c, lc = O.sparse_mla(q, kv, np.full((1, 4), -1), sink)
    assert np.all(c == 0) and np.allclose(lc[0], sink)


def test_sparse_rope_dims_enter_logits_not_values():
    rng = np.random.default_rng(14)
    q, kv, sink = _rand_attn(rng, B=1, H=2, N=16)
    idx = np.arange(16)[None]
    a, _ = O.sparse_mla(q, kv, idx, sink)
    kv2 = kv.copy()
    kv2[..., 512:] *= 3.0  # changes logits only
    b, _ = O.sparse_mla(q, kv2, idx, sink)
    assert np.abs(a - b).max() > 1e-3
    q3 = q.copy()
    q3[..., 512:] = 0.0
    kv3 = kv.copy()
    kv3[..., 512:] = 123.0  # no effect once the query's RoPE part is 0
    c1, _ = O.sparse_mla(q3, kv, idx, sink)
    c2, _ = O.sparse_mla(q3, kv3, idx, sink)
    np.testing.assert_allclose(c1, c2, rtol=1e-12)


# ---------------------------------------------------------------- schedule / stack
def test_schedule_validation():
    for bad in ["", "SFF", "FXS", "fss"]:
        with pytest.raises(ValueError):
            O.validate_schedule(bad)
    assert O.governing_full_layer("FSSFSF") == [0, 0, 0, 3, 3, 5]


def test_golden_counting_figures():
    g = json.load(open(os.path.join(GOLDEN, "counting_figures.json")))
    L, N = g["layers"], g["context_tokens"]
    all_f = "F" * L
    once = "F" + "S" * (L - 1)
    every6 = W.every_nth_schedule(L, g["refresh_period"])
    assert all_f.count("F") * N == g["scores_per_token_indexer_every_layer"]
    assert once.count("F") * N == g["scores_per_token_index_built_once"]
    assert all_f.count("F") // once.count("F") == g["cut_if_built_once"]
    assert every6.count("F") == g["cut_if_refreshed_every_6_layers"]
    hy4 = W.hy4_schedule(L, g["hy4_full_layers"])
    assert hy4.count("F") == g["hy4_full_layers"]
    assert hy4.startswith(g["hy4_schedule_prefix"])
    assert g["mla_head_dim"] == W.D_QK and g["mla_rope_dim"] == W.D_ROPE


def _small_stack(schedule, B=2, N=300, seed=5):
    return W.stack("cpu", seed=seed, L=len(schedule), B=B, N=N, H_I=4, d_I=16, topk=32, H=2,
                   schedule=schedule, gate=True)


def test_stack_s_layers_reuse_governing_index_bytewise():
    sched = "FFSSFSSS"
    wl = _small_stack(sched)
    r = O.layer_stack(wl.layers, sched, wl.topk)
    gov = O.governing_full_layer(sched)
    for l in range(len(sched)):
        assert np.array_equal(r["idx"][l], r["idx"][gov[l]])
        assert r["idx"][l].tobytes() == r["idx"][gov[l]].tobytes()
    # each F layer's index is its own top-k (not the previous one's)
    s4 = O.indexer_scores(wl.layers[4].q_idx, wl.layers[4].w, wl.layers[4].k_idx)
    assert np.array_equal(r["idx"][4], O.topk_indices(s4, wl.topk))
    # an S layer's attention equals attention over the governing F layer's index
    o6, _ = O.sparse_mla(wl.layers[6].q, wl.layers[6].kv, r["idx"][4], wl.layers[6].sink,
                         wl.layers[6].gate)
    np.testing.assert_array_equal(r["out"][6], o6)


@pytest.mark.parametrize("sched", ["FSSS", "FFFF", "F" + "S" * 11, W.every_nth_schedule(12, 6)])
def test_stack_counting_identity(sched):
    B, N = 2, 200
    wl = _small_stack(sched, B=B, N=N)
    r = O.layer_stack(wl.layers, sched, wl.topk)
    assert r["n_scores"] == sched.count("F") * N * B


def test_stack_counting_identity_causal():
    sched = "FSF"
    wl = _small_stack(sched, B=3, N=100)
    nv = np.array([100, 37, 0])
    r = O.layer_stack(wl.layers, sched, 8, n_valid=nv)
    assert r["n_scores"] == 2 * (100 + 37 + 0)
    assert np.all(r["idx"][0][2] == -1)


def test_workload_recipes_are_deterministic():
    a = W.tiny("cpu")
    b = W.tiny("cpu")
    for la, lb in zip(a.layers, b.layers):
        assert torch.equal(la.q, lb.q) and torch.equal(la.kv, lb.kv)
    assert torch.equal(a.layers[0].k_idx, b.layers[0].k_idx)
