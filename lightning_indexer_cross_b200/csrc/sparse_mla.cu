// Sparse MLA decode attention with a per-head sink and a sigmoid output gate
// on sm_100a tensor cores.
//
// For query b, head h, selected rows j (Hy4 IndexCache explainer, Jargon
// "DSA": token-level selection; Hy4-preview porting issue: head 576 = 512
// latent + 64 RoPE, per-head "softmax-denominator bias", sigmoid gate):
//   z_j = sm_scale * q[b,h,:] . kv[idx_j, :]            (576-d)
//   o   = sum_j e^{z_j} kv[idx_j, :512] / (e^{sink_h} + sum_j e^{z_j})
//   out = sigmoid(gate[b,h,:]) * o
//
// Main kernel: persistent, one CTA per SM; a work unit is (split of TS <= 256
// selected rows, query, block of 128 heads). Tensor memory holds 512 fp32
// columns per lane, and the 128 x 512 output alone fills it, so its two
// 256-column halves swap roles from one unit to the next. With A the half
// the unit's logits use and B the other:
//   QK   S[128 heads x TS] = Q . KV^T over 9 slices of 64 dims (tcgen05,
//        M = 128 heads, N = TS rows) into half A;
//   soft the epilogue warps read S (one head per TMEM lane), write
//        P = 2^{z log2e - ref} as bf16 into shared memory in the K-major
//        layout of an MMA A operand;
//   PV   O[:, 0:256] = P . V[:, 0:256] into half B, then
//        O[:, 256:512] = P . V[:, 256:512] into half A (S is dead by then);
//        V rows are the same gathered rows, read again as an MN-major B
//        operand (64 rows x 256 dims per stage).
// Each unit writes a normalised partial (m, l, O / l): O / l as 32-head x
// 128-byte tiles staged in swizzled shared memory and written by TMA stores.
// Half B is read out while the MMAs of half A run, and the next unit's
// logits go into it (its A is this unit's B), so the next QK does not wait
// for the whole output to be read out. The combine kernel merges the splits,
// adds e^{sink} once to the denominator, applies the gate and writes out /
// lse.
//
// Warp roles (16 warps): 0-10 gather every stage of every unit (one ring of
// three stages), 11 issues the MMAs, 12-15 run the softmax and the output.
// Gathers are cp.async (16 B, zero fill for -1 rows) into 128-byte-swizzled
// stages; the gathering threads fence the async proxy before signalling the
// MMA. Each unit's row indices are loaded one unit ahead.
#include "common.cuh"
#include "kernels.h"

namespace ic {

namespace {

constexpr int kD = 576;
constexpr int kDv = 512;
constexpr int kHeads = 128;      // heads per CTA (MMA M)
constexpr int kQKChunks = kD / 64;
// 16 warps (so at most 128 registers per thread): warps 0-10 gather, warp 11
// issues the MMAs, warps 12-15 run the softmax and the output (one per TMEM
// lane quadrant, quadrant = warp % 4). (Measured on B200: a CTA's random
// 16-byte gathers scale with the threads issuing them, about 51 GB/s from 224
// threads and 66 GB/s from 512.)
constexpr int kGatherWarps = 11;
constexpr int kGather = kGatherWarps * 32;
constexpr int kMmaWarp = 11;
constexpr int kEpiWarp0 = 12;
constexpr int kThreads = 512;
constexpr int kStages = 3;
constexpr float kLog2e = 1.4426950408889634f;

template <int TS>
struct MlaCfg {
  static constexpr int kQKStage = kHeads * 128 + TS * 128;
  static constexpr int kPVStage = 64 * 256 * 2;
  static constexpr int kStageBytes = kQKStage > kPVStage ? kQKStage : kPVStage;
  static constexpr int kPBytes = kHeads * TS * 2;
  // output tiles (4 KB) per epilogue warp, staged in the P buffer
  static constexpr int kOutSlots = kPBytes / (4 * 4096) < 4 ? kPBytes / (4 * 4096) : 4;
  static constexpr int kOffStages = 0;
  static constexpr int kOffP = kStages * kStageBytes;
  // one 4 KB output tile per epilogue warp for the first output half (the P
  // buffer is still being read by the second half's MMAs)
  static constexpr int kOffTiles = kOffP + kPBytes;
  static constexpr int kOffIdx = kOffTiles + 4 * 4096;    // [2][TS] selected rows, double-buffered
  static constexpr int kOffMask = kOffIdx + 2 * TS * 4;   // [2][TS / 32] validity bits
  static constexpr int kOffBar = kOffMask + 2 * (TS / 32) * 4;
  // full[kStages], empty[kStages], s_full, p_ready, o1_full, o2_full, o1_free, o2_free, retire,
  // idx_ready[2], idx_free[2]
  static constexpr int kNumBars = 2 * kStages + 11;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  // dynamic shared memory starts 1024-byte aligned (checked at entry)
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr int kNumSt = kQKChunks + 2 * (TS / 64);
  static_assert(kOutSlots >= 1, "at least one output tile per warp");
  static_assert(kOffBar % 8 == 0, "mbarrier alignment");
  static_assert(kOffTiles % 1024 == 0, "swizzled tiles 1024-byte aligned");
  static_assert(kSmemBytes <= 232448, "fits one CTA per SM");
};

// PV stage p (64 selected rows x 256 latent dims) gathered by NT threads:
// copy i is 16-byte chunk i % 8 of (row, 64-dim block) pair i / 8; thread gt
// takes i = gt + NT n, so its chunk column is fixed.
template <int TS, int NT>
IC_DEV void gather_pv_stage(uint32_t base_u, const int32_t* idx_s, const __nv_bfloat16* kvb,
                            const __nv_bfloat16* zero_src, int gt, int p) {
  constexpr int kRowStep = NT / 8;
  constexpr int kNP = (64 * 32 + NT - 1) / NT;
  static_assert(NT % 8 == 0, "chunk column fixed per thread");
  const int cc = gt & 7, q0 = gt >> 3;
  const int jh = p / (TS / 64), tc = p % (TS / 64);
  int tok[kNP];
#pragma unroll
  for (int n = 0; n < kNP; ++n) {
    const int q = q0 + kRowStep * n;  // (row in chunk) * 4 + 64-dim block
    tok[n] = q < 256 ? idx_s[tc * 64 + (q >> 2)] : -1;
  }
#pragma unroll
  for (int n = 0; n < kNP; ++n) {
    const int q = q0 + kRowStep * n;
    if (q < 256) {
      const int j = q >> 2, bb = q & 3;
      const __nv_bfloat16* src =
          tok[n] >= 0 ? kvb + static_cast<int64_t>(tok[n]) * kD + jh * 256 + bb * 64 + cc * 8 : zero_src;
      cp_async16(base_u + bb * 8192 + sw128_offset(j, cc), src, tok[n] >= 0 ? 16u : 0u);
    }
  }
}

// Work unit u -> (token split, query, head block); splits of one query are
// adjacent, so the CTAs working at one time share each query's Q rows in L2.
struct Unit {
  int sp, b, hb;
};
IC_DEV Unit unit_of(const MlaArgs& a, int u) {
  Unit w;
  w.sp = u % a.splits;
  const int r = u / a.splits;
  w.b = r % a.B;
  w.hb = r / a.B;
  return w;
}

// Persistent: CTA c takes units c, c + ctas, c + 2 ctas, ... The gather warps
// run continuously through the units' stages (a ring of kStages shared-memory
// stages); the output of unit i (TMEM -> swizzled tiles -> TMA stores)
// overlaps the QK gathers and MMAs of unit i + 1.
template <int TS>
__global__ void __launch_bounds__(kThreads, 1) sparse_mla_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                   const __grid_constant__ CUtensorMap omap,
                                                                   const MlaArgs a) {
  using C = MlaCfg<TS>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzled layouts need a 1024-byte-aligned base; the layout leaves no
  // room to align it here, so a misaligned window is reported, not used
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) record_status(a.status, IC_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* stages = smem + C::kOffStages;
  uint8_t* ps = smem + C::kOffP;
  uint8_t* tiles1 = smem + C::kOffTiles;
  int32_t* idx_s = reinterpret_cast<int32_t*>(smem + C::kOffIdx);
  uint32_t* vmask = reinterpret_cast<uint32_t*>(smem + C::kOffMask);  // bit j of word w: row 32w+j valid
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = full + kStages;
  uint64_t* s_full = empty + kStages;  // S of the current unit in TMEM (half A)
  uint64_t* p_ready = s_full + 1;      // P in shared memory, S read
  uint64_t* o1_full = p_ready + 1;     // output dims [0, 256) in TMEM half B
  uint64_t* o2_full = o1_full + 1;     // output dims [256, 512) in TMEM half A
  uint64_t* o1_free = o2_full + 1;     // half B read out
  uint64_t* o2_free = o1_free + 1;     // half A read out
  uint64_t* retire = o2_free + 1;      // every MMA of this CTA retired
  uint64_t* idx_ready = retire + 1;    // [2] selected rows of a unit in shared memory
  uint64_t* idx_free = idx_ready + 2;  // [2] the softmax is done with a unit's validity bits
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&omap);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], kGather);
      mbar_init(&empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_ready, 128);  // the four epilogue warps
    mbar_init(o1_full, 1);
    mbar_init(o2_full, 1);
    mbar_init(o1_free, 128);
    mbar_init(o2_free, 128);
    mbar_init(retire, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&idx_ready[i], kGather);
      mbar_init(&idx_free[i], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  pdl_wait();
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp < kGatherWarps) {
    // ------------------------------------------------------------ gather warps
    // QK stage c: the 64-dim slice c of the unit's 128-head Q block by one TMA
    // load, and slice c of every selected row by cp.async. PV stage: 64
    // selected rows x 256 latent dims by cp.async. Rows land in
    // 128-byte-swizzled operand layouts; -1 slots are zero-filled (their
    // logits are masked). (Measured on B200: random 16-byte gathers of one
    // SM scale with the number of threads issuing them and the bytes in
    // flight, about 33 GB/s from 96 threads and 62 GB/s from 256, while
    // tile::gather4 and per-row bulk copies are limited by their issue rate.)
    const int gt = threadIdx.x;
    constexpr int kQRowStep = kGather / 8;
    constexpr int kNQ = (TS + kQRowStep - 1) / kQRowStep;
    const int gcc = gt & 7, gq0 = gt >> 3;
    // Thread gt holds rows gt and gt + kGather of a unit's selection in
    // registers; the next unit's are loaded one unit ahead.
    auto load_rows = [&](int u, int (&v)[2]) {
      const Unit w = unit_of(a, u);
      const int tok0 = w.sp * TS;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = gt + e * kGather;
        int x = -1;
        if (j < TS && tok0 + j < a.k) {
          x = a.idx[static_cast<int64_t>(w.b) * a.k + tok0 + j];
          if (x < -1 || static_cast<int64_t>(x) >= a.N) {  // anything outside [0, N) counts as -1
            record_status(a.status, IC_ERR_BAD_INDEX);
            x = -1;
          }
        }
        v[e] = x;
      }
    };
    int cur[2], nxt[2] = {-1, -1};
    if (blockIdx.x < a.units) load_rows(blockIdx.x, cur);
    bool ok = true;
    int g = 0;  // global stage counter
    for (int i = 0, u = blockIdx.x; u < a.units && ok; ++i, u += a.ctas) {
      const Unit w = unit_of(a, u);
      int32_t* ids = idx_s + (i & 1) * TS;
      uint32_t* vm = vmask + (i & 1) * (TS / 32);
      // the softmax of unit i - 2 is done with this buffer's validity bits
      if (i >= 2 && !mbar_wait(&idx_free[i & 1], static_cast<uint32_t>(((i >> 1) - 1) & 1), abort_flag, a.status, a.wait_ns)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j0 = warp * 32 + e * kGather;  // warp-uniform
        if (j0 < TS) {
          ids[j0 + lane] = cur[e];
          const uint32_t bal = __ballot_sync(0xffffffffu, cur[e] >= 0);
          if (lane == 0) vm[j0 >> 5] = bal;
        }
      }
      mbar_arrive(&idx_ready[i & 1]);
      if (u + a.ctas < a.units) load_rows(u + a.ctas, nxt);
      if (!mbar_wait(&idx_ready[i & 1], static_cast<uint32_t>((i >> 1) & 1), abort_flag, a.status, a.wait_ns)) {
        ok = false;
        break;
      }
      int qk_tok[kNQ];  // this thread's QK rows, the same in all nine QK stages
#pragma unroll
      for (int n = 0; n < kNQ; ++n) {
        const int j = gq0 + kQRowStep * n;
        qk_tok[n] = j < TS ? ids[j] : -1;
      }
      const __nv_bfloat16* kvb = a.kv + static_cast<int64_t>(w.b) * a.kv_batch_stride;
      for (int s = 0; s < C::kNumSt; ++s, ++g) {
        const int st = g % kStages;
        if (!mbar_wait(&empty[st], static_cast<uint32_t>((g / kStages) & 1) ^ 1u, abort_flag, a.status, a.wait_ns)) {
          ok = false;
          break;
        }
        uint8_t* base = stages + st * C::kStageBytes;
        const uint32_t base_u = smem_u32(base);
        if (s < kQKChunks) {
          // rows past the last query read zeros; rows of a neighbouring query
          // are never written out. The Q bytes are booked before thread 0's
          // own arrival can complete the phase.
          if (gt == 0) {
            mbar_expect_tx(&full[st], kHeads * 128);
            tma_load_2d(base, &qmap, &full[st], s * 64, w.b * a.H + w.hb * kHeads);
          }
          const uint32_t kv_u = base_u + kHeads * 128;
#pragma unroll
          for (int n = 0; n < kNQ; ++n) {
            const int j = gq0 + kQRowStep * n;
            if (j < TS) {
              const int tok = qk_tok[n];
              const __nv_bfloat16* src = tok >= 0 ? kvb + static_cast<int64_t>(tok) * kD + s * 64 + gcc * 8 : a.kv;
              // a row's slices are read one stage apart: a 256-byte DRAM fetch
              // brings the next slice into L2 with this one
              cp_async16_l2_256(kv_u + sw128_offset(j, gcc), src, tok >= 0 ? 16u : 0u);
            }
          }
        } else {
          gather_pv_stage<TS, kGather>(base_u, ids, kvb, a.kv, gt, s - kQKChunks);
        }
        // this thread's arrival on the stage happens when its copies have
        // landed; the MMA thread fences the async proxy after its wait
        cp_async_arrive_noinc(&full[st]);
      }
      cur[0] = nxt[0];
      cur[1] = nxt[1];
    }
    // land everything still in flight (also on the abort path)
    cp_async_wait_all();
    if (!ok && gt == 0) {
      // wind down: Q loads of QK stages still pending must land (bounded waits)
      for (int r = (g > kStages ? g - kStages : 0); r < g; ++r)
        if (r % C::kNumSt < kQKChunks) mbar_drain(&full[r % kStages], static_cast<uint32_t>((r / kStages) & 1));
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, TS, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
      const uint32_t p_addr = smem_u32(ps);
      bool ok = true;
      int g = 0;
      for (int i = 0, u = blockIdx.x; u < a.units && ok; ++i, u += a.ctas) {
        // TMEM halves: S and output dims [256, 512) in half A, output dims
        // [0, 256) in half B; the next unit's A is this unit's B, read out
        // first, while this unit's second output half is still being formed
        const uint32_t col_a = (i & 1) ? 256u : 0u, col_b = 256u - col_a;
        if (i > 0 && !mbar_wait(o1_free, static_cast<uint32_t>((i - 1) & 1), abort_flag, a.status, a.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int s = 0; s < kQKChunks; ++s, ++g) {
          const int st = g % kStages;
          if (!mbar_wait(&full[st], (g / kStages) & 1, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t base = smem_u32(stages + st * C::kStageBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem_base + col_a, sw128_desc(base + kk * 32, 16, 1024),
                        sw128_desc(base + kHeads * 128 + kk * 32, 16, 1024), idesc_qk, (s | kk) != 0);
          mma_commit(&empty[st]);
        }
        if (!ok) break;
        mma_commit(s_full);
        if (!mbar_wait(p_ready, static_cast<uint32_t>(i & 1), abort_flag, a.status, a.wait_ns)) { ok = false; break; }
        // half B held the previous unit's second output half
        if (i > 0 && !mbar_wait(o2_free, static_cast<uint32_t>((i - 1) & 1), abort_flag, a.status, a.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int s = kQKChunks; s < C::kNumSt; ++s, ++g) {
          const int st = g % kStages;
          if (!mbar_wait(&full[st], (g / kStages) & 1, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
          fence_proxy_async_smem();
          tc_fence_after();
          const int p = s - kQKChunks;
          const int jh = p / (TS / 64), tc = p % (TS / 64);
          const uint32_t d_tmem = tmem_base + (jh == 0 ? col_b : col_a);
          const uint32_t base = smem_u32(stages + st * C::kStageBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(d_tmem, sw128_desc(p_addr + tc * (kHeads * 128) + kk * 32, 16, 1024),
                        sw128_desc(base + kk * 2048, 8192, 1024), idesc_pv, (tc | kk) != 0);
          mma_commit(&empty[st]);
          if (p == TS / 64 - 1) mma_commit(o1_full);
        }
        if (!ok) break;
        mma_commit(o2_full);
      }
      // every MMA issued has retired before TMEM is released
      mma_commit(retire);
      mbar_drain(retire, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax + output
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // head row within the block
    const uint32_t tlane = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    const float c2 = a.sm_scale * kLog2e;
    uint8_t* tiles = ps + quad * (C::kOutSlots * 4096);
    bool ok = true;
    for (int i = 0, u = blockIdx.x; u < a.units && ok; ++i, u += a.ctas) {
      const Unit w = unit_of(a, u);
      const uint32_t col_a = (i & 1) ? 256u : 0u, col_b = 256u - col_a;
      const uint32_t taddr = tlane + col_a;  // S (and later output dims [256, 512))
      const uint32_t* vm = vmask + (i & 1) * (TS / 32);
      ok = mbar_wait(&idx_ready[i & 1], static_cast<uint32_t>((i >> 1) & 1), abort_flag, a.status, a.wait_ns) &&
           mbar_wait(s_full, static_cast<uint32_t>(i & 1), abort_flag, a.status, a.wait_ns);
      __syncwarp();  // tcgen05.ld is warp-collective
      if (!ok) break;
      tc_fence_after();
      constexpr int kChunks = TS / 32;  // even: TS is a multiple of 64
      uint32_t rb0[32], rb1[32];
      // The exponent reference is the max over the first 32-column chunk's
      // valid entries (one TMEM load), not the row max: P = 2^(z log2e - ref)
      // then exceeds 1 by at most 2^(row max - ref), and the row max is
      // tracked on the way. Only if they differ by more than kSafe (log2
      // units; P stays finite in bf16 and fp32 far beyond, and no valid entry
      // underflows) is the pass redone with the row max. The partial's (m, l)
      // use the same reference.
      constexpr float kSafe = 64.f;
      float mp[4];
      auto chunk_max = [&](const uint32_t (&rv)[32], uint32_t vmw) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float x = ((vmw >> j) & 1u) ? __uint_as_float(rv[j]) : -INFINITY;
          mp[j & 3] = fmaxf(mp[j & 3], x);
        }
      };
      tmem_ld32_issue(taddr, rb0);
      tmem_ld_wait(rb0);
      mp[0] = mp[1] = mp[2] = mp[3] = -INFINITY;
      chunk_max(rb0, vm[0]);
      const float m0 = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
      float mxe = m0 == -INFINITY ? 0.f : m0 * c2;
      float lp[4];
      // P = 2^(z log2e - mxe) as bf16 into the A-operand layout; row sum of
      // the rounded values; running row max
      auto p_chunk = [&](const uint32_t (&rv)[32], uint32_t vmw, int c0) {
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float x0 = ((vmw >> j) & 1u) ? __uint_as_float(rv[j]) : -INFINITY;
          const float x1 = ((vmw >> (j + 1)) & 1u) ? __uint_as_float(rv[j + 1]) : -INFINITY;
          mp[(j >> 1) & 3] = fmaxf(mp[(j >> 1) & 3], fmaxf(x0, x1));
          const __nv_bfloat162 pb =
              __floats2bfloat162_rn(ex2_approx(fmaf(x0, c2, -mxe)), ex2_approx(fmaf(x1, c2, -mxe)));
          lp[(j >> 1) & 3] += __low2float(pb) + __high2float(pb);
          pk[j >> 1] = *reinterpret_cast<const uint32_t*>(&pb);
        }
        const uint32_t blk = smem_u32(ps + (c0 >> 6) * (kHeads * 128));
        const int ch0 = (c0 & 63) >> 3;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          st_shared_v4(blk + sw128_offset(r, ch0 + q4),
                       make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]));
      };
      float m = -INFINITY;
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {  // the second pass only if some row needs it (warp-uniform)
        lp[0] = lp[1] = lp[2] = lp[3] = 0.f;
        mp[0] = mp[1] = mp[2] = mp[3] = -INFINITY;
        if (pass > 0) {
          tmem_ld32_issue(taddr, rb0);
          tmem_ld_wait(rb0);
        }
#pragma unroll 1
        for (int c = 0; c < kChunks; c += 2) {
          tmem_ld32_issue(taddr + (c + 1) * 32, rb1);
          p_chunk(rb0, vm[c], c * 32);
          tmem_ld_wait(rb1);
          if (c + 2 < kChunks) tmem_ld32_issue(taddr + (c + 2) * 32, rb0);
          p_chunk(rb1, vm[c + 1], (c + 1) * 32);
          if (c + 2 < kChunks) tmem_ld_wait(rb0);
        }
        m = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
        // (two-sided: with no valid entry in the first chunk the reference is 0)
        const bool redo = m != -INFINITY && fabsf(m * c2 - mxe) > kSafe;
        if (!__any_sync(0xffffffffu, redo)) break;
        if (redo) mxe = m * c2;
      }
      const float mx = m == -INFINITY ? -INFINITY : mxe;  // every row invalid: all p = 0
      const float l = (lp[0] + lp[1]) + (lp[2] + lp[3]);
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(p_ready);
      mbar_arrive(&idx_free[i & 1]);
      // O / l (0 when no row was valid) as 32-head x 128-byte tiles in
      // 128-byte-swizzled shared memory, each written out by one TMA store;
      // heads past H fall outside the map and are not written. Dims
      // [0, 256) (TMEM half B) are read out as soon as their MMAs retire,
      // through this warp's own tile (the P buffer is still read by the
      // second half's MMAs), and then free half B for the next unit's
      // logits; dims [256, 512) (half A) go through four tiles of the P
      // buffer once every PV MMA has retired.
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const int head0 = w.hb * kHeads + quad * 32;
      auto put_tile = [&](const uint32_t (&wd)[32], int x, uint8_t* tile) {
        const uint32_t tb = smem_u32(tile);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          st_shared_v4(tb + sw128_offset(lane, k),
                       make_uint4(wd[4 * k], wd[4 * k + 1], wd[4 * k + 2], wd[4 * k + 3]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && head0 < a.H) {
          tma_store_4d(&omap, tile, x, w.sp, head0, w.b);
          bulk_commit();
        }
      };
      uint8_t* own_tile = tiles1 + quad * 4096;
      int nt = 0;  // tiles of the P buffer issued by this warp in this unit
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        ok = mbar_wait(half == 0 ? o1_full : o2_full, static_cast<uint32_t>(i & 1), abort_flag, a.status, a.wait_ns);
        __syncwarp();
        if (!ok) break;
        tc_fence_after();
        const uint32_t tcol = tlane + (half == 0 ? col_b : col_a);
        auto place = [&](const uint32_t (&wd)[32], int x) {
          uint8_t* tile;
          if (half == 0) {
            if (lane == 0) bulk_wait_read<0>();  // this warp's tile is read out
            __syncwarp();
            tile = own_tile;
          } else {
            const int slot = nt % C::kOutSlots;
            if (nt >= C::kOutSlots) {
              if (lane == 0) bulk_wait_read<C::kOutSlots - 1>();  // the slot's previous store has read it
              __syncwarp();
            }
            tile = tiles + slot * 4096;
            ++nt;
          }
          put_tile(wd, x, tile);
        };
        if (a.out_f32) {
#pragma unroll 1
          for (int t = 0; t < 8; ++t) {  // 32 dims per tile
            uint32_t rv[32];
            tmem_ld32_issue(tcol + 32u * t, rv);
            tmem_ld_wait(rv);
#pragma unroll
            for (int j = 0; j < 32; ++j) rv[j] = __float_as_uint(__uint_as_float(rv[j]) * inv_l);
            place(rv, half * 256 + 32 * t);
          }
        } else {
#pragma unroll 1
          for (int t = 0; t < 4; ++t) {  // 64 dims per tile
            uint32_t rv[64];
            tmem_ld64_issue(tcol + 64u * t, rv);
            tmem_ld_wait64(rv);
            uint32_t wd[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
              wd[j] = pack_bf16x2(__uint_as_float(rv[2 * j]) * inv_l, __uint_as_float(rv[2 * j + 1]) * inv_l);
            place(wd, half * 256 + 64 * t);
          }
        }
        tc_fence_before();
        mbar_arrive(half == 0 ? o1_free : o2_free);
      }
      if (!ok) break;
      if (lane == 0) bulk_wait_read<0>();  // the tiles (the next unit's P buffer) are read out
      __syncwarp();
      const int head = w.hb * kHeads + r;
      if (head < a.H) {
        const int64_t row = (static_cast<int64_t>(w.b) * a.H + head) * a.splits + w.sp;
        a.part_ml[row * 2 + 0] = mx;
        a.part_ml[row * 2 + 1] = l;
      }
    }
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// One warp, one half of one (query, head) row gw = b H + h: merge the
// splits' normalised partials (m, l, O / l) over dims [256 half, 256 half +
// 256), add e^{sink} once to the denominator, normalise, gate, write out (and
// lse, from half 0). Lane `lane` owns the 8 consecutive dims 256 half +
// 8 lane + [0, 8): one 16-byte load per split for bf16 partials, two for
// fp32. Every split of a chunk of CH splits is requested before any is
// reduced, so one memory latency covers a chunk; chunks are merged with a
// running maximum.
template <bool F32>
IC_DEV void combine_half(const MlaArgs& a, int64_t gw, int half, int lane) {
  constexpr int CH = F32 ? 4 : 8;
  constexpr int NV = F32 ? 2 : 1;  // 16-byte words per split and lane
  const int h = static_cast<int>(gw % a.H);
  const int S = a.splits;
  const int d0 = half * 256 + lane * 8;
  const float2* ml = reinterpret_cast<const float2*>(a.part_ml) + gw * S;
  uint4 graw = make_uint4(0, 0, 0, 0);  // 8 bf16 gate logits, unpacked at the end
  if (a.gate) graw = __ldg(reinterpret_cast<const uint4*>(a.gate + gw * kDv + d0));
  const float sink2 = a.sink[h] * kLog2e;
  // the sink's term e^{sink - M}, M = sink so far (no term for a sink of -inf)
  float M = sink2, den = sink2 == -INFINITY ? 0.f : 1.f;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int s0 = 0; s0 < S; s0 += CH) {
    float2 mlv[CH];
    uint4 raw[CH][NV];
#pragma unroll
    for (int u = 0; u < CH; ++u) {
      if (s0 + u < S) {
        mlv[u] = __ldcg(&ml[s0 + u]);
        const int64_t off = (gw * S + s0 + u) * kDv + d0;
        if constexpr (F32) {
          raw[u][0] = __ldcg(reinterpret_cast<const uint4*>(static_cast<const float*>(a.part_o) + off));
          raw[u][NV - 1] = __ldcg(reinterpret_cast<const uint4*>(static_cast<const float*>(a.part_o) + off + 4));
        } else {
          raw[u][0] = __ldcg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.part_o) + off));
        }
      } else {
        mlv[u] = make_float2(-INFINITY, 0.f);
      }
    }
    float Mc = M;
#pragma unroll
    for (int u = 0; u < CH; ++u) Mc = fmaxf(Mc, mlv[u].x);
    const float sc = M == Mc ? 1.f : exp2f(M - Mc);  // (M = Mc = -inf: nothing to rescale)
    den *= sc;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= sc;
    M = Mc;
#pragma unroll
    for (int u = 0; u < CH; ++u) {
      if (mlv[u].x == -INFINITY) continue;  // no valid row in that split
      const float wgt = exp2f(mlv[u].x - Mc) * mlv[u].y;
      den += wgt;
      if constexpr (F32) {
        const uint32_t w[8] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w,
                               raw[u][NV - 1].x, raw[u][NV - 1].y, raw[u][NV - 1].z, raw[u][NV - 1].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(wgt, __uint_as_float(w[e]), acc[e]);
      } else {
        const uint32_t w[4] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(wgt, bf16_lane(w[e >> 1], e & 1), acc[e]);
      }
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;  // (no valid row and no sink: out = 0)
  const uint32_t gwd[4] = {graw.x, graw.y, graw.z, graw.w};
  float o[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    o[e] = acc[e] * inv;
    if (a.gate) o[e] *= 1.f / (1.f + __expf(-bf16_lane(gwd[e >> 1], e & 1)));
  }
  if (a.out_f32) {
    float* dst = static_cast<float*>(a.out) + gw * kDv + d0;
    *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(o[4], o[5], o[6], o[7]);
  } else {
    uint4 pk;
    pk.x = pack_bf16x2(o[0], o[1]);
    pk.y = pack_bf16x2(o[2], o[3]);
    pk.z = pack_bf16x2(o[4], o[5]);
    pk.w = pack_bf16x2(o[6], o[7]);
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + gw * kDv + d0) = pk;
  }
  if (a.lse && half == 0 && lane == 0) a.lse[gw] = den > 0.f ? (M + log2f(den)) / kLog2e : -INFINITY;
}

// The split combine: one warp per half of a (query, head) row, after the
// main kernel has completed.
__global__ void __launch_bounds__(128) mla_combine_kernel(const MlaArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t item = static_cast<int64_t>(blockIdx.x) * 4 + warp;  // half-rows
  pdl_trigger();
  pdl_wait();
  if (item >= 2 * static_cast<int64_t>(a.B) * a.H) return;
  if (a.out_f32) combine_half<true>(a, item >> 1, static_cast<int>(item & 1), lane);
  else combine_half<false>(a, item >> 1, static_cast<int>(item & 1), lane);
}

constexpr int kCombThreads = 512;
constexpr int kCombRowsPerBar = 16;  // one barrier for the CTA's rows

// Row gw from its staged partials prow ([S][512]) and (m, l) pairs mr:
// dims 8 q + 256 c, c < 2.
template <bool F32>
IC_DEV void combine_staged_row(const MlaArgs& a, const uint8_t* prow, const float2* mr, int64_t gw, float sink2,
                               int q, const uint4 (&graw)[2]) {
  constexpr int ES = F32 ? 4 : 2;
  const int S = a.splits;
  float M = sink2;
  for (int s2 = 0; s2 < S; ++s2) M = fmaxf(M, mr[s2].x);
  float den = sink2 == -INFINITY ? 0.f : ex2_approx(sink2 - M);  // (no term for a sink of -inf)
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
  // one split's contribution (a split with no valid row has weight 0)
  auto add_split = [&](int s2) {
    const float2 v = mr[s2];
    const float wgt = v.x == -INFINITY ? 0.f : ex2_approx(v.x - M) * v.y;
    den += wgt;
    const uint8_t* ps = prow + static_cast<size_t>(s2) * kDv * ES;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      if constexpr (F32) {
        const float4 x0 = ld_shared_v4f(ps + (8 * q + 256 * c) * 4);
        const float4 x1 = ld_shared_v4f(ps + (8 * q + 256 * c) * 4 + 16);
        const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[8 * c + e] = fmaf(wgt, xv[e], acc[8 * c + e]);
      } else {
        const uint4 w4 = *reinterpret_cast<const uint4*>(ps + (8 * q + 256 * c) * 2);
        const uint32_t wd[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[8 * c + e] = fmaf(wgt, bf16_lane(wd[e >> 1], e & 1), acc[8 * c + e]);
      }
    }
  };
  int s2 = 0;
  for (; s2 + 1 < S; s2 += 2) {
    add_split(s2);
    add_split(s2 + 1);
  }
  if (s2 < S) add_split(s2);
  const float inv = den > 0.f ? 1.f / den : 0.f;  // (no valid row and no sink: out = 0)
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const uint32_t gwd[4] = {graw[c].x, graw[c].y, graw[c].z, graw[c].w};
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      o[e] = acc[8 * c + e] * inv;
      // sigmoid with the hardware 2^x and reciprocal (relative error ~2^-21)
      if (a.gate) o[e] *= __fdividef(1.f, 1.f + ex2_approx(-kLog2e * bf16_lane(gwd[e >> 1], e & 1)));
    }
    if (a.out_f32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + gw * kDv + 8 * q + 256 * c);
      dst[0] = make_float4(o[0], o[1], o[2], o[3]);
      dst[1] = make_float4(o[4], o[5], o[6], o[7]);
    } else {
      uint4 pk;
      pk.x = pack_bf16x2(o[0], o[1]);
      pk.y = pack_bf16x2(o[2], o[3]);
      pk.z = pack_bf16x2(o[4], o[5]);
      pk.w = pack_bf16x2(o[6], o[7]);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + gw * kDv + 8 * q + 256 * c) = pk;
    }
  }
  if (a.lse && q == 0) a.lse[gw] = den > 0.f ? (M + log2f(den)) / kLog2e : -INFINITY;
}

// The split combine with the partials staged by TMA: CTA c takes head rows
// [c rpc, c rpc + rpc) of all queries (row = b H + h); one bulk copy per 32 KB
// brings their partials (the S splits of a row are contiguous) into shared
// memory with no register cost, so every row of the grid is in flight at
// once (one barrier: per-row-pair barriers measured slower). Thread t
// serves row t / 32 and dims 8 (t % 32) + 256 c, c < 2 (32 consecutive
// threads read 512 consecutive bytes of a split row); two splits are reduced
// per step.
template <bool F32>
__global__ void __launch_bounds__(kCombThreads) mla_combine_bulk_kernel(const MlaArgs a, int rpc) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int ES = F32 ? 4 : 2;
  const int S = a.splits;
  const int64_t rows = static_cast<int64_t>(a.B) * a.H;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * rpc;
  const int nrows = static_cast<int>(rows - row0 < rpc ? rows - row0 : rpc);
  const uint32_t row_bytes = static_cast<uint32_t>(S) * kDv * ES;
  uint8_t* pbuf = smem;
  float2* mlb = reinterpret_cast<float2*>(smem + static_cast<size_t>(rpc) * row_bytes);
  // one barrier per kCombRowsPerBar rows
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(rpc) * row_bytes +
                                               ((static_cast<size_t>(rpc) * S * 8 + 15) & ~size_t(15)));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 8);
  const int t = threadIdx.x;
  const int ngroups = (nrows + kCombRowsPerBar - 1) / kCombRowsPerBar;
  if (t == 0) {
    for (int i = 0; i < 8; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();
  if (nrows <= 0) return;
  if (t == 0) {
    const uint8_t* src = static_cast<const uint8_t*>(a.part_o) + row0 * row_bytes;
    for (int gi = 0; gi < ngroups; ++gi) {
      const int r0 = gi * kCombRowsPerBar;
      const int nr = nrows - r0 < kCombRowsPerBar ? nrows - r0 : kCombRowsPerBar;
      const uint32_t bytes = static_cast<uint32_t>(nr) * row_bytes;
      mbar_arrive_expect_tx(&bars[gi], bytes);
      const size_t off = static_cast<size_t>(r0) * row_bytes;
      for (uint32_t o = 0; o < bytes; o += 32768u)
        bulk_load(pbuf + off + o, src + off + o, bytes - o < 32768u ? bytes - o : 32768u, &bars[gi]);
    }
  }
  const float2* ml = reinterpret_cast<const float2*>(a.part_ml);
  for (int i = t; i < nrows * S; i += kCombThreads) mlb[i] = __ldcg(&ml[row0 * S + i]);
  const int r = t >> 5, q = t & 31;
  const bool active = r < nrows;
  const int64_t gw = row0 + r;
  uint4 graw[2];
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    graw[c] = make_uint4(0, 0, 0, 0);
    if (active && a.gate) graw[c] = __ldg(reinterpret_cast<const uint4*>(a.gate + gw * kDv + 8 * q + 256 * c));
  }
  const float sink2 = active ? __ldg(&a.sink[gw % a.H]) * kLog2e : 0.f;
  __syncthreads();  // (m, l) in shared memory
  // this row's partials
  const bool ok = active && mbar_wait(&bars[r / kCombRowsPerBar], 0u, abort_flag, a.status, a.wait_ns);
  if (ok) combine_staged_row<F32>(a, pbuf + static_cast<size_t>(r) * row_bytes, mlb + r * S, gw, sink2, q, graw);
  // every copy has landed (or its wait gave up) before the CTA exits
  if (t == 0)
    for (int gi = 0; gi < ngroups; ++gi) mbar_drain(&bars[gi], 0u);
}

// Rows per CTA of the staged combine: as many as fit two CTAs per SM (at most
// 16); 0 if one row does not fit.
int combine_rows_per_cta(int splits, bool f32, size_t* smem_bytes) {
  static int sm_bytes = 0, reserved = 0;
  if (sm_bytes == 0) {
    int dev = 0, v = 0, rsv = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess) v = 0;
    if (cudaDeviceGetAttribute(&rsv, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess) rsv = 1024;
    reserved = rsv;
    sm_bytes = v > 0 ? v : 1;
  }
  const size_t row_bytes = static_cast<size_t>(splits) * kDv * (f32 ? 4 : 2);
  const size_t per_row = row_bytes + static_cast<size_t>(splits) * 8;
  const size_t fixed = 16 + 80;  // (m, l) padding, barriers, abort flag
  const int64_t usable = static_cast<int64_t>(sm_bytes) / 2 - reserved - static_cast<int64_t>(fixed);
  int rpc = usable > 0 ? static_cast<int>(static_cast<size_t>(usable) / per_row) : 0;
  if (rpc > 16) rpc = 16;
  if (rpc < 1) return 0;
  *smem_bytes = static_cast<size_t>(rpc) * row_bytes + ((static_cast<size_t>(rpc) * splits * 8 + 15) & ~size_t(15)) + 80;
  return rpc;
}

template <int TS>
cudaError_t launch_ts(const CUtensorMap& qmap, const CUtensorMap& omap, const MlaArgs& a, cudaStream_t stream,
                      bool pdl) {
  using C = MlaCfg<TS>;
  auto kern = sparse_mla_kernel<TS>;
  static bool done[64] = {false};  // one flag set per template instance
  cudaError_t e = set_smem_once(kern, C::kSmemBytes, done);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, dim3(a.ctas), dim3(kThreads), C::kSmemBytes, stream, pdl, qmap, omap, a);
}

}  // namespace

int mla_smem_bytes(int ts) {
  switch (ts) {
    case 64: return MlaCfg<64>::kSmemBytes;
    case 128: return MlaCfg<128>::kSmemBytes;
    default: return MlaCfg<256>::kSmemBytes;
  }
}

cudaError_t launch_sparse_mla(const CUtensorMap& qmap, const CUtensorMap& omap, const MlaArgs& a, cudaStream_t stream,
                              bool pdl, int* launches) {
  cudaError_t e;
  switch (a.ts) {
    case 64: e = launch_ts<64>(qmap, omap, a, stream, pdl); break;
    case 128: e = launch_ts<128>(qmap, omap, a, stream, pdl); break;
    case 256: e = launch_ts<256>(qmap, omap, a, stream, pdl); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  size_t cbytes = 0;
  const int rpc = combine_rows_per_cta(a.splits, a.out_f32 != 0, &cbytes);
  if (rpc > 0) {
    auto kern = a.out_f32 ? mla_combine_bulk_kernel<true> : mla_combine_bulk_kernel<false>;
    static bool done_b[2][64] = {{false}};
    e = set_smem_once(kern, 232448, done_b[a.out_f32 ? 1 : 0]);
    if (e != cudaSuccess) return e;
    const int64_t rows = static_cast<int64_t>(a.B) * a.H;
    const dim3 grid(static_cast<unsigned>((rows + rpc - 1) / rpc));
    e = launch_kernel(kern, grid, dim3(kCombThreads), cbytes, stream, true, a, rpc);
  } else {
    const int64_t warps = 2 * static_cast<int64_t>(a.B) * a.H;  // one per half row
    const dim3 grid(static_cast<unsigned>((warps + 3) / 4));
    e = launch_kernel(mla_combine_kernel, grid, dim3(128), 0, stream, true, a);
  }
  if (e != cudaSuccess) return e;
  *launches += 2;
  return cudaGetLastError();
}

}  // namespace ic
