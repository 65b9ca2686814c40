"""GPU parity of the cache-append step (ic_cache_append) against the float64
oracle: LayerNorm-with-bias keys (bf16 or e4m3 + scale), interleaved RoPE on
the latent rows and the queries, untouched rows, out-of-range rows.

Stored values are judged against the exact (float64) ones: a bf16 value must
be a correct rounding of the exact value (within half a unit in the last
place, with a hair of slack for the kernel's fp32 arithmetic); an e4m3 code
must equal the oracle's encoding of the exact quotient, except where that
quotient lies within 1e-5 (relative) of the midpoint between two adjacent
grid values, where either neighbour is a correct rounding."""
import numpy as np
import pytest
import torch

import oracle
from oracle import cache_append_oracle as A
from lightning_indexer_cross_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _ops():
    from lightning_indexer_cross_b200 import ops
    return ops


def _f64(t):
    return t.detach().cpu().to(torch.float64).numpy()


def assert_bf16_rounding_of(got: torch.Tensor, exact: np.ndarray, what: str):
    g = _f64(got)
    mag = np.abs(exact)
    ulp = np.where(mag > 0, np.exp2(np.floor(np.log2(np.maximum(mag, 1e-300))) - 7), 0.0)
    err = np.abs(g - exact)
    bad = err > 0.5 * ulp * (1 + 2.0 ** -10) + 1e-30
    assert not bad.any(), f"{what}: {bad.sum()} values are not a rounding of the exact ones " \
                          f"(worst {err[bad].max():.3e} at |x| {mag[bad][err[bad].argmax()]:.3e})"


def assert_e4m3_codes(got_codes: np.ndarray, quotient: np.ndarray, what: str):
    exp = A.encode_e4m3(quotient)
    diff = got_codes != exp
    if diff.any():
        a = oracle.decode_e4m3(got_codes[diff])
        b = oracle.decode_e4m3(exp[diff])
        v = quotient[diff]
        ok = np.abs(v - (a + b) / 2) <= 1e-5 * np.maximum(np.abs(v), 2.0 ** -9)
        assert ok.all(), f"{what}: {int((~ok).sum())} codes differ from the correct rounding"


def _run_and_check(case, fp8, eps=1e-6, base=10000.0):
    c = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in case.items()}
    before = {k: (v.clone() if isinstance(v, torch.Tensor) else None) for k, v in c.items()}
    ws = _ops().cache_append(c["k_raw"], c["gamma"], c["beta"], c["kv_raw"], c["pos"], c["key_cache"],
                             c["kv_cache"], key_scale=c["key_scale"], ln_eps=eps, rope_base=base, q=c["q"],
                             q_pos=c["q_pos"])
    torch.cuda.synchronize()
    from lightning_indexer_cross_b200 import _abi
    assert _abi.ic_last_device_status(_ops()._ptr(ws), _ops()._stream_ptr()) == _abi.IC_OK
    ref = A.cache_append(c["k_raw"], c["gamma"], c["beta"], eps, c["kv_raw"], _f64(c["pos"]).astype(np.int64),
                         base=base)
    T = c["k_raw"].shape[0]
    C = c["key_cache"].shape[0]
    pos = c["pos"].cpu().numpy()
    cache_of = np.arange(T) if C > 1 else np.zeros(T, dtype=np.int64)
    # rows that were not written keep their bytes
    written = torch.zeros(c["key_cache"].shape[:2], dtype=torch.bool)
    written[torch.from_numpy(cache_of), torch.from_numpy(pos)] = True
    keep = ~written.to(c["key_cache"].device)
    assert torch.equal(c["key_cache"][keep].view(torch.uint8), before["key_cache"][keep].view(torch.uint8))
    assert torch.equal(c["kv_cache"][keep].view(torch.uint8), before["kv_cache"][keep].view(torch.uint8))
    if fp8:
        assert torch.equal(c["key_scale"][keep], before["key_scale"][keep])
    rows = (torch.from_numpy(cache_of).to(c["key_cache"].device), c["pos"])
    # latent dims: a byte copy; rotary dims: a rounding of the exact rotation
    kv_rows = c["kv_cache"][rows]
    assert torch.equal(kv_rows[:, :512].view(torch.uint8), c["kv_raw"][:, :512].view(torch.uint8))
    assert_bf16_rounding_of(kv_rows[:, 512:], ref["kv"][:, 512:], "rotary dims of the latent rows")
    # keys
    if not fp8:
        assert_bf16_rounding_of(c["key_cache"][rows], ref["key"], "normalised keys")
    else:
        scale = c["key_scale"][rows].double().cpu().numpy()
        np.testing.assert_allclose(scale, ref["scale"], rtol=1e-5)
        codes = c["key_cache"][rows].cpu().numpy()
        assert_e4m3_codes(codes, ref["key"] / ref["scale"][:, None], "e4m3 keys")
    # queries
    if c["q"] is not None:
        qref = A.rope_query(before["q"], _f64(c["q_pos"]).astype(np.int64), base=base)
        assert torch.equal(c["q"][:, :, :512].view(torch.uint8), before["q"][:, :, :512].view(torch.uint8))
        assert_bf16_rounding_of(c["q"][:, :, 512:], qref[:, :, 512:], "rotary dims of the queries")


@pytest.mark.parametrize("d_I", [64, 128])
@pytest.mark.parametrize("per_token", [False, True])
@pytest.mark.parametrize("fp8", [False, True])
def test_cache_append_matches_oracle(cuda_dev, d_I, per_token, fp8):
    T = 16 if per_token else 200
    case = W.append_case(T, 4096, d_I, per_token=per_token, fp8=fp8, seed=50 + d_I + 2 * per_token + fp8,
                         device=cuda_dev)
    _run_and_check(case, fp8)


def test_cache_append_rotates_queries_and_takes_eps_and_base(cuda_dev):
    case = W.append_case(3, 131072, 128, per_token=False, fp8=False, B=6, H=128, seed=61, device=cuda_dev)
    _run_and_check(case, False, eps=0.25, base=500.0)


def test_cache_append_single_token_decode_shape(cuda_dev):
    # one new token per query, 32 per-query caches, e4m3 keys, queries rotated
    case = W.append_case(32, 2048, 128, per_token=True, fp8=True, B=32, H=128, seed=62, device=cuda_dev)
    _run_and_check(case, True)


def test_cache_append_constant_key_gives_the_bias(cuda_dev):
    case = W.append_case(4, 64, 128, seed=63, device=cuda_dev)
    case["k_raw"][:] = 3.0
    c = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in case.items()}
    _ops().cache_append(c["k_raw"], c["gamma"], c["beta"], c["kv_raw"], c["pos"], c["key_cache"], c["kv_cache"])
    torch.cuda.synchronize()
    got = c["key_cache"][0, c["pos"]]
    assert torch.equal(got, c["beta"].to(torch.bfloat16).expand_as(got))


def test_cache_append_out_of_range_row_is_reported_and_skipped(cuda_dev):
    from lightning_indexer_cross_b200 import _abi
    case = W.append_case(5, 300, 128, seed=64, device=cuda_dev)
    bad = case["pos"].clone()
    bad[2] = 300  # == N
    kc, kvc = case["key_cache"].clone(), case["kv_cache"].clone()
    ws = _ops().cache_append(case["k_raw"], case["gamma"], case["beta"], case["kv_raw"], bad, kc, kvc)
    assert _abi.ic_last_device_status(_ops()._ptr(ws), _ops()._stream_ptr()) == _abi.IC_ERR_BAD_INDEX
    good_rows = {int(r) for i, r in enumerate(bad.tolist()) if i != 2}
    kv_changed = (kvc != case["kv_cache"]).any(dim=-1)[0].nonzero().flatten().tolist()
    key_changed = (kc.view(torch.uint8) != case["key_cache"].view(torch.uint8)).any(dim=-1)[0]
    assert set(kv_changed) == good_rows
    assert set(key_changed.nonzero().flatten().tolist()) == good_rows
