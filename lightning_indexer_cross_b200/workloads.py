"""Seeded synthetic inputs for the IndexCache decode path.

This module is the one place that draws random inputs. Both the float64
oracle (under ``oracle/``) and the CUDA path read the tensors it returns, so
both sides see identical bytes: values are drawn in fp32, rounded once to
bf16 (round-to-nearest-even) or quantised once to fp8 e4m3, and never
re-rounded afterwards.

It holds none of the method's arithmetic (no indexer scores, no top-k, no
attention). The only derived quantities are input-construction steps:

* bf16 rounding (``torch.Tensor.to(torch.bfloat16)``, RNE);
* per-token fp8 e4m3 quantisation of indexer keys with scale
  ``max|k_s| / 448`` (the cache-append step that precedes the hot path);
* planted keys (the "planted relevant tokens" of the tiny and 1M-context
  workloads, "aligned to q, score +4 sigma"): a key c * u along
  u = unit(sum_h w_h q_h) of its query, its length c chosen so that its
  score is mu + 4 sigma of the score distribution of the unplanted keys.
  The recipe is stated in terms of the score, so this step evaluates two
  things about it in closed form: the score of a key along u (linear in c:
  c * sum_{h: q_h.u > 0} w_h q_h.u) and the population mean and standard
  deviation of the score of a key drawn N(0, sigma_k^2 I), from the Gaussian
  moments of ReLU (the first-order arc-cosine kernel: for jointly Gaussian
  X, Y with standard deviations s_x, s_y and correlation cos t,
  E[ReLU(X) ReLU(Y)] = s_x s_y (sin t + (pi - t) cos t) / (2 pi)). No score
  of any drawn key is computed here.

Workload shapes follow the five configurations of the IndexCache decode study
(Hy4 IndexCache explainer, "Where the saving actually lands": 78 layers and a
1M-token context; porting issue on Hy4-preview, indexer bullet: 21 full layers
of 78 starting F F F S S S; MLA shape RoPE-64, head 576, top-k 2048).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch

D_LATENT = 512  # latent value width of an MLA row
D_ROPE = 64     # rotary part of an MLA row
D_QK = D_LATENT + D_ROPE  # 576: the head dim of the MLA query/key


# Planted keys score this many standard deviations above the mean of the
# unplanted scores ("score +4 sigma").
PLANT_Z = 4.0


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, g, device, scale=1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x


def _rand(shape, g, device, scale=1.0) -> torch.Tensor:
    x = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x


def quantize_e4m3_rows(k: torch.Tensor):
    """Per-token (last-dim row) fp8 e4m3 quantisation.

    Returns ``(codes uint8 [..., d], scale fp32 [...])`` with
    ``scale = max|k| / 448`` and ``codes = e4m3(k / scale)`` rounded to
    nearest even by torch's cast. A row of zeros gets scale 0 and zero codes.
    """
    amax = k.abs().amax(dim=-1)
    scale = (amax / 448.0).to(torch.float32)
    safe = torch.where(scale > 0, scale, torch.ones_like(scale))
    codes = (k / safe.unsqueeze(-1)).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale


def planted_direction(q: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
    """Unit vector along sum_h w_h q_h for each query: q [B,H,d], w [B,H] -> [B,d]."""
    u = (w.float().unsqueeze(-1) * q.float()).sum(dim=1)
    return u / u.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def unplanted_score_moments(q: torch.Tensor, w: torch.Tensor, sigma_k: float):
    """Population mean and standard deviation of sum_h w_h ReLU(q_h . k) for
    k ~ N(0, sigma_k^2 I), per query, in float64: q [B,H,d], w [B,H] ->
    (mu [B], sd [B]). X_h = q_h . k are jointly Gaussian with covariance
    sigma_k^2 q_h . q_g; E[ReLU(X_h)] = s_h / sqrt(2 pi) and the second
    moments are the first-order arc-cosine kernel."""
    qd = q.double().cpu()
    wd = w.double().cpu()
    nrm = qd.norm(dim=-1)                                   # [B,H]
    sh = sigma_k * nrm
    mu = (wd * sh).sum(-1) / math.sqrt(2 * math.pi)
    cos = (qd @ qd.transpose(1, 2)) / (nrm.unsqueeze(-1) * nrm.unsqueeze(-2)).clamp_min(1e-300)
    t = torch.arccos(cos.clamp(-1.0, 1.0))
    m2 = sh.unsqueeze(-1) * sh.unsqueeze(-2) * (torch.sin(t) + (math.pi - t) * torch.cos(t)) / (2 * math.pi)
    e2 = torch.einsum("bh,bhg,bg->b", wd, m2, wd)
    return mu, (e2 - mu * mu).clamp_min(0.0).sqrt()


def schedule_from_f_positions(L: int, f_positions) -> str:
    s = ["S"] * L
    for p in f_positions:
        s[int(p)] = "F"
    return "".join(s)


def hy4_schedule(L: int = 78, n_full: int = 21, seed: int = 2) -> str:
    """The 78-layer F/S pattern: F at 0,1,2, S at 3,4,5, the remaining F
    positions drawn without replacement from layers 6..L-1 with a seeded
    ``numpy.random.default_rng``."""
    rng = np.random.default_rng(seed)
    rest = rng.choice(np.arange(6, L), n_full - 3, replace=False)
    return schedule_from_f_positions(L, [0, 1, 2] + sorted(int(x) for x in rest))


def every_nth_schedule(L: int, n: int) -> str:
    """Refresh the index every n layers: F at 0, n, 2n, ..."""
    return "".join("F" if l % n == 0 else "S" for l in range(L))


@dataclasses.dataclass
class Layer:
    """One layer's inputs. Indexer fields are None on S layers."""
    q_idx: Optional[torch.Tensor] = None    # [B,H_I,d_I] bf16
    w: Optional[torch.Tensor] = None        # [B,H_I] fp32
    k_idx: Optional[torch.Tensor] = None    # [Bk,N,d_I] bf16 or uint8 (e4m3 codes)
    k_scale: Optional[torch.Tensor] = None  # [Bk,N] fp32 (fp8 keys only)
    q: Optional[torch.Tensor] = None        # [B,H,576] bf16
    kv: Optional[torch.Tensor] = None       # [Bkv,N,576] bf16
    sink: Optional[torch.Tensor] = None     # [H] fp32
    gate: Optional[torch.Tensor] = None     # [B,H,512] bf16 or None


@dataclasses.dataclass
class Workload:
    name: str
    B: int
    N: int
    H_I: int
    d_I: int
    topk: int
    H: int
    schedule: str
    layers: List[Layer]
    k_fp8: bool = False
    shared_keys: bool = False     # one indexer key cache for all B queries
    shared_kv: bool = False       # one latent KV cache for all B queries
    n_valid: Optional[torch.Tensor] = None  # [B] int64, causal limit
    planted: Optional[torch.Tensor] = None  # [B,P] int64 planted positions
    sm_scale: float = 1.0 / math.sqrt(D_QK)
    seed: int = 0

    @property
    def L(self) -> int:
        return len(self.schedule)


def _indexer_inputs(B, N, H_I, d_I, Bk, g, device, key_scale, w_scale):
    q = _randn((B, H_I, d_I), g, device, 1.0 / math.sqrt(d_I)).to(torch.bfloat16)
    w = _rand((B, H_I), g, device, w_scale)
    k = _randn((Bk, N, d_I), g, device, key_scale)
    return q, w, k


def _plant(k_f32, q, w, positions, sigma_k, z=PLANT_Z, e4m3=False):
    """Overwrite the keys at ``positions`` [Bk,P] of query b's cache with
    c_b * d_b, d_b along unit(sum_h w_h q_h), c_b such that the planted score
    is mu_b + z sd_b of the unplanted scores (population moments). For e4m3
    keys d_b is the direction as the per-token quantisation stores it (its
    codes do not depend on c_b, the scale is c_b times the unit key's), so
    the target holds for the stored bytes, not only before quantisation."""
    u = planted_direction(q, w)  # [B,d] float32
    mu, sd = unplanted_score_moments(q, w, sigma_k)
    qd, wd = q.double().cpu(), w.double().cpu()
    for b in range(positions.shape[0]):
        d = u[b].double().cpu()
        if e4m3:
            codes, scale = quantize_e4m3_rows(u[b:b + 1].cpu())
            d = codes.view(torch.float8_e4m3fn).double()[0] * float(scale[0])
        per_unit = (wd[b] * torch.relu(qd[b] @ d)).sum()  # score of the key d
        c = float((mu[b] + z * sd[b]) / per_unit)
        k_f32[b, positions[b]] = (c * d).to(torch.float32).to(k_f32.device).unsqueeze(0)
    return k_f32


def _attn_inputs(B, N, H, Bkv, g, device, gate: bool):
    q = _randn((B, H, D_QK), g, device).to(torch.bfloat16)
    kv = _randn((Bkv, N, D_QK), g, device).to(torch.bfloat16)
    sink = _randn((H,), g, device, 0.5)
    gt = _randn((B, H, D_LATENT), g, device).to(torch.bfloat16) if gate else None
    return q, kv, sink, gt




def tiny(device="cpu", seed: int = 0) -> Workload:
    """4-layer stack F S S S, N=4096, B=1, H_I=4, d_I=64, k=256, H=8, 8 planted."""
    B, N, H_I, d_I, H, K = 1, 4096, 4, 64, 8, 256
    g = _gen(seed, device)
    q_i, w, k = _indexer_inputs(B, N, H_I, d_I, B, g, device, 1.0 / math.sqrt(d_I), 0.25)
    rng = np.random.default_rng(seed)
    pos = torch.as_tensor(np.sort(rng.choice(N, 8, replace=False)), dtype=torch.int64).view(1, 8)
    k = _plant(k, q_i, w, pos.to(device), 1.0 / math.sqrt(d_I)).to(torch.bfloat16)
    layers = []
    for l in range(4):
        q, kv, sink, _ = _attn_inputs(B, N, H, B, g, device, gate=False)
        lay = Layer(q=q, kv=kv, sink=sink)
        if l == 0:
            lay.q_idx, lay.w, lay.k_idx = q_i, w, k
        layers.append(lay)
    return Workload("tiny_stack4_N4096", B, N, H_I, d_I, K, H, "FSSS", layers,
                    planted=pos, seed=seed)


def single_f(device="cpu", seed: int = 1, N: int = 131072, B: int = 8, H_I: int = 64,
             d_I: int = 128, topk: int = 2048, H: int = 128, gate: bool = True,
             shared: bool = False) -> Workload:
    """One F layer at model shape: per-query caches (default) or one shared cache."""
    g = _gen(seed, device)
    Bk = 1 if shared else B
    q_i, w, k = _indexer_inputs(B, N, H_I, d_I, Bk, g, device, 1.0 / math.sqrt(d_I), 1.0 / H_I)
    q, kv, sink, gt = _attn_inputs(B, N, H, Bk, g, device, gate)
    lay = Layer(q_idx=q_i, w=w, k_idx=k.to(torch.bfloat16), q=q, kv=kv, sink=sink, gate=gt)
    return Workload(f"single_F_B{B}_N{N}", B, N, H_I, d_I, topk, H, "F", [lay],
                    shared_keys=shared, shared_kv=shared, seed=seed)


def stack(device="cpu", seed: int = 2, L: int = 78, n_full: int = 21, B: int = 32,
          N: int = 131072, H_I: int = 64, d_I: int = 128, topk: int = 2048, H: int = 128,
          rho: float = 0.8, schedule: Optional[str] = None, gate: bool = True,
          s_indexers: bool = False, layer_keys: str = "per_layer") -> Workload:
    """The 78-layer F/S decode stack: one key cache and one KV cache per layer,
    shared by all B queries; keys independent per layer; indexer and attention
    queries correlated across layers, q_l = rho q_{l-1} + sqrt(1-rho^2) eps_l.

    For the reuse diagnostic only: s_indexers also gives every S layer the
    indexer inputs it would have (its query from the same correlated chain,
    weights and keys from a second generator, so the stack's own inputs are
    unchanged); layer_keys="shared" makes every layer's indexer keys those of
    layer 0 (the draws of the others are still made and then dropped)."""
    assert layer_keys in ("per_layer", "shared")
    sched = schedule if schedule is not None else hy4_schedule(L, n_full, seed)
    assert len(sched) == L
    g = _gen(seed, device)
    g2 = _gen(seed + 7919, device) if s_indexers else None
    c = math.sqrt(1.0 - rho * rho)
    qi_prev = q_prev = None
    keys0 = None
    layers = []
    for l in range(L):
        eps_i = _randn((B, H_I, d_I), g, device, 1.0 / math.sqrt(d_I))
        eps_q = _randn((B, H, D_QK), g, device)
        qi_f = eps_i if qi_prev is None else rho * qi_prev + c * eps_i
        q_f = eps_q if q_prev is None else rho * q_prev + c * eps_q
        qi_prev, q_prev = qi_f, q_f
        lay = Layer(q=q_f.to(torch.bfloat16))
        lay.kv = _randn((1, N, D_QK), g, device).to(torch.bfloat16)
        lay.sink = _randn((H,), g, device, 0.5)
        lay.gate = _randn((B, H, D_LATENT), g, device).to(torch.bfloat16) if gate else None
        if sched[l] == "F":
            lay.q_idx = qi_f.to(torch.bfloat16)
            lay.w = _rand((B, H_I), g, device, 1.0 / H_I)
            lay.k_idx = _randn((1, N, d_I), g, device, 1.0 / math.sqrt(d_I)).to(torch.bfloat16)
        elif s_indexers:
            lay.q_idx = qi_f.to(torch.bfloat16)
            lay.w = _rand((B, H_I), g2, device, 1.0 / H_I)
            lay.k_idx = _randn((1, N, d_I), g2, device, 1.0 / math.sqrt(d_I)).to(torch.bfloat16)
        if layer_keys == "shared" and lay.k_idx is not None:
            keys0 = lay.k_idx if keys0 is None else keys0
            lay.k_idx = keys0
        layers.append(lay)
    return Workload(f"stack{L}_B{B}_N{N}", B, N, H_I, d_I, topk, H, sched, layers,
                    shared_keys=True, shared_kv=True, seed=seed)


def long_context(device="cpu", seed: int = 3, N: int = 1048576, B: int = 4, H_I: int = 64,
                 d_I: int = 128, topk: int = 2048, H: int = 128, fp8: bool = False,
                 n_planted: int = 64) -> Workload:
    """1M-context decode, per-query caches, planted tokens at evenly spaced
    positions floor((i + 1/2) N / P); keys bf16 or fp8 e4m3 with per-token scale.
    Both key variants come from the same fp32 draw."""
    g = _gen(seed, device)
    q_i, w, k = _indexer_inputs(B, N, H_I, d_I, B, g, device, 1.0 / math.sqrt(d_I), 1.0 / H_I)
    pos = torch.tensor([int((i + 0.5) * N / n_planted) for i in range(n_planted)],
                       dtype=torch.int64).repeat(B, 1)
    k = _plant(k, q_i, w, pos.to(device), 1.0 / math.sqrt(d_I), e4m3=fp8)
    q, kv, sink, _ = _attn_inputs(B, N, H, B, g, device, gate=False)
    lay = Layer(q_idx=q_i, w=w, q=q, kv=kv, sink=sink)
    if fp8:
        lay.k_idx, lay.k_scale = quantize_e4m3_rows(k)
    else:
        lay.k_idx = k.to(torch.bfloat16)
    return Workload(f"long_ctx_B{B}_N{N}_{'fp8' if fp8 else 'bf16'}", B, N, H_I, d_I, topk, H, "F",
                    [lay], k_fp8=fp8, planted=pos, seed=seed)


def prefill(device="cpu", seed: int = 4, P: int = 262144, C: int = 2048, H_I: int = 64,
            d_I: int = 128, topk: int = 2048, H: int = 128) -> Workload:
    """Chunked prefill: C causal queries at positions P..P+C-1 over one shared
    cache of P + C tokens; query i sees tokens 0..P+i."""
    N = P + C
    g = _gen(seed, device)
    q_i, w, k = _indexer_inputs(C, N, H_I, d_I, 1, g, device, 1.0 / math.sqrt(d_I), 1.0 / H_I)
    q, kv, sink, _ = _attn_inputs(C, N, H, 1, g, device, gate=False)
    lay = Layer(q_idx=q_i, w=w, k_idx=k.to(torch.bfloat16), q=q, kv=kv, sink=sink)
    n_valid = torch.arange(P + 1, P + C + 1, dtype=torch.int64, device=device)
    return Workload(f"prefill_C{C}_P{P}", C, N, H_I, d_I, topk, H, "F", [lay],
                    shared_keys=True, shared_kv=True, n_valid=n_valid, seed=seed)


def indexer_case(B, N, H_I, d_I, shared=False, fp8=False, causal=False, seed=11, device="cpu"):
    """A bare indexer input set (used by unit tests)."""
    g = _gen(seed, device)
    Bk = 1 if shared else B
    q, w, k = _indexer_inputs(B, N, H_I, d_I, Bk, g, device, 1.0 / math.sqrt(d_I), 1.0 / H_I)
    if fp8:
        codes, scale = quantize_e4m3_rows(k)
        kk, ks = codes, scale
    else:
        kk, ks = k.to(torch.bfloat16), None
    n_valid = None
    if causal:
        n_valid = torch.randint(0, N + 1, (B,), generator=g, device=device, dtype=torch.int64)
        n_valid[0] = N
    return q, w, kk, ks, n_valid


def scores_case(B, N, seed=12, ties=False, neg_inf_frac=0.0, device="cpu"):
    """Random fp32 score rows for top-k tests; optional heavy ties and -inf."""
    g = _gen(seed, device)
    s = torch.randn((B, N), generator=g, device=device, dtype=torch.float32)
    if ties:
        s = torch.round(s * 4.0) / 4.0  # few distinct values, many exact ties
    if neg_inf_frac > 0:
        m = torch.rand((B, N), generator=g, device=device) < neg_inf_frac
        s[m] = float("-inf")
    return s


def attention_case(B, N, H, k, shared=False, gate=True, n_invalid=0, seed=13, device="cpu"):
    """Bare sparse-MLA inputs: q, kv, idx (distinct per row, -1 padding at the
    end of each row when n_invalid > 0), sink, gate."""
    g = _gen(seed, device)
    Bkv = 1 if shared else B
    q, kv, sink, gt = _attn_inputs(B, N, H, Bkv, g, device, gate)
    idx = torch.empty((B, k), dtype=torch.int32, device=device)
    for b in range(B):
        perm = torch.randperm(N, generator=g, device=device)[:k]
        idx[b] = perm.to(torch.int32)
        if n_invalid:
            idx[b, k - n_invalid:] = -1
    return q, kv, idx, sink, gt


def append_case(T, N, d_I, per_token=False, fp8=False, B=0, H=128, seed=14, device="cpu"):
    """Inputs of the cache-append step: T new tokens' raw indexer keys
    [T, d_I] bf16 (mean offset and spread so the norm has work to do),
    LayerNorm weight ~ 1 + N(0, 0.1) and bias ~ N(0, 0.1) fp32, raw latent
    rows [T, 576] bf16, destination rows (distinct for one shared cache;
    0 and N-1 always among them), caches [C, N, ...] pre-filled with random
    bytes (C = T per-token caches, else 1), and optionally queries
    [B, H, 576] bf16 with positions q_pos [B] (0, 1, N-1 and 1000003 first)."""
    g = _gen(seed, device)
    k_raw = (_randn((T, d_I), g, device, 2.0) + 0.5).to(torch.bfloat16)
    gamma = 1.0 + _randn((d_I,), g, device, 0.1)
    beta = _randn((d_I,), g, device, 0.1)
    kv_raw = _randn((T, D_QK), g, device).to(torch.bfloat16)
    if per_token:
        pos = torch.randint(0, N, (T,), generator=g, device=device)
        pos[0] = 0
        if T > 1:
            pos[T - 1] = N - 1
    else:  # distinct rows: 0, T - 2 others from [1, N - 2], N - 1
        assert T <= N and (T == 1 or N >= 2)
        mid = torch.randperm(max(N - 2, 0), generator=g, device=device)[:max(T - 2, 0)] + 1
        ends = [torch.zeros(1, dtype=mid.dtype, device=device)]
        pos = torch.cat(ends + ([mid, torch.full((1,), N - 1, dtype=mid.dtype, device=device)] if T > 1 else []))
    pos = pos.to(torch.int64)
    C = T if per_token else 1
    kc_bytes = torch.randint(0, 256, (C, N, d_I * (1 if fp8 else 2)), generator=g, device=device, dtype=torch.uint8)
    key_cache = kc_bytes if fp8 else kc_bytes.view(torch.bfloat16)
    # finite bf16 filler for the latent cache (random bytes could be NaN)
    kv_cache = _randn((C, N, D_QK), g, device).to(torch.bfloat16)
    key_scale = _rand((C, N), g, device) if fp8 else None
    q = q_pos = None
    if B:
        q = _randn((B, H, D_QK), g, device).to(torch.bfloat16)
        q_pos = torch.randint(0, 1 << 20, (B,), generator=g, device=device).to(torch.int64)
        for i, v in enumerate([0, 1, N - 1, 1000003][:B]):
            q_pos[i] = v
    return dict(k_raw=k_raw, gamma=gamma, beta=beta, kv_raw=kv_raw, pos=pos, key_cache=key_cache,
                kv_cache=kv_cache, key_scale=key_scale, q=q, q_pos=q_pos)


def gate_case(B, H, d_v=128, gate=True, seed=15, device="cpu"):
    """Inputs of the decompressed-space gate: ungated latent attention
    outputs [B, H, 512] bf16 ~ N(0, 1), per-head up-projections
    [H, d_v, 512] bf16 ~ N(0, 1)/sqrt(512) (synthetic weights), gate logits
    [B, H, d_v] bf16 ~ N(0, 1) or None."""
    g = _gen(seed, device)
    o = _randn((B, H, D_LATENT), g, device).to(torch.bfloat16)
    w = _randn((H, d_v, D_LATENT), g, device, 1.0 / math.sqrt(D_LATENT)).to(torch.bfloat16)
    gl = _randn((B, H, d_v), g, device).to(torch.bfloat16) if gate else None
    return o, w, gl
