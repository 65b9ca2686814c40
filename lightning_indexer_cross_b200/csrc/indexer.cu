// Lightning indexer on sm_100a tensor cores.
//
//   score[b, s] = sum_h w[b,h] * max(0, q[b,h,:] . k_b[s,:])
//
// (Hy4 IndexCache explainer, Jargon "Indexer": the cheap pass that scores
// every cached position; DeepSeek lightning-indexer form.)
//
// Mapping. One tcgen05.mma per 16-wide slice of d_I computes a tile
//   D[128 keys x n] = K_tile[128 x d_I] . Qg[n x d_I]^T,    n = G * HP
// where Qg stacks the (padded) heads of G queries that read the same key
// tile. With one cache shared by all queries, two such groups (two TMEM
// accumulators) use every key tile a CTA loads. Keys are the M side, so each TMEM lane holds one key's n head logits
// and the epilogue thread owning that lane does ReLU, the w_h weighting and
// the head sum in registers -- no cross-thread reduction. With one cache per
// query G = 1 (n = HP, the decode case); with one cache shared by many
// queries G = 256 / HP (prefill chunks, the layer stack), so each key byte
// feeds up to 256 head columns.
//
// Warp roles (one CTA per SM, persistent over a contiguous range of
// (query group, key tile) work items):
//   warp 0      TMA producer: 128-key tiles of the key cache into a ring of
//               shared-memory stages (128-byte swizzle, K-major).
//   warp 1      TMEM owner and MMA issuer (one elected lane).
//   warps 2..    epilogue: TMEM -> registers -> score row; also stage the
//               query groups' head weights, and one of their threads issues
//               the TMA loads of the groups' Q (swizzled, zero-padded heads).
//               warps 2..9, two per TMEM lane quadrant, each reducing one
//               half of the columns.
//   warps 10..13 (e4m3 keys only). With d_I = 128 the key tiles go to the
//               MMA as they are (tcgen05 kind::f8f6f4, e4m3 x e4m3, fp32
//               accumulation), and these warps, once per query group, split
//               each query column (one head of one query) into two e4m3
//               parts, q s = hi + lo, with s a power of two that puts the
//               column's largest |q| in [128, 256): hi = e4m3(q s) keeps its
//               leading 4 bits, lo = e4m3(q s - hi) the next 4, so the sum
//               equals the bf16 value exactly for every element with
//               |q s| >= 2^-2 (smaller ones keep a 2^-10 grid); each key tile
//               then takes two MMA passes, hi and lo, into one accumulator, and
//               the head weight w is read as w / s. With d_I = 64 they widen
//               the e4m3 tiles to f16 in shared memory (one conversion
//               instruction per two codes; exact) and the staged bf16
//               queries to f16 in place for kind::f16 (two f16 operands; a
//               bf16 query value is exact in f16 from 2^-14 up to 65504, an
//               error under 2^-25 below; the path needs |q| < 65504). The
//               per-token scale is applied to the head sum, since
//               ReLU(c x) = c ReLU(x) for c >= 0.
#include <cuda_fp8.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace ic {

namespace {

constexpr int kTileKeys = 128;
constexpr int kMaxCols = 256;  // MMA N limit for M = 128
constexpr int kEpiWarp0 = 2;

// Named barrier over n threads that also ORs a predicate across them: every
// participating thread gets the same answer.
IC_DEV bool named_bar_or(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1 : 0), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// tcgen05.mma with e4m3 A and B from shared memory (kind::f8f6f4: K = 32 per
// instruction; the instruction descriptor's A and B formats 0 are e4m3).
IC_DEV void mma_e4m3_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// PAIR: two query groups (two Q slots, one TMEM accumulator each) share every
// key tile a CTA loads -- one cache shared by all queries; half the key-tile
// traffic, two key stages instead of four.
template <int D_I, bool FP8, bool PAIR>
struct IdxCfg {
  static constexpr int kBlocks = D_I / 64;                        // 64-element (128 B) swizzle blocks
  static constexpr int kTileBytes = kTileKeys * D_I * 2;          // bf16 tile
  static constexpr int kRawBytes = FP8 ? kTileKeys * D_I : 0;     // e4m3 tile
  // e4m3 keys with d_I = 128: 128-byte rows, 128-byte swizzle, read by the
  // MMA directly (kind::f8f6f4); no bf16 / f16 key stages
  static constexpr bool kF8Mma = FP8 && D_I == 128;
  static constexpr int kStages =
      kF8Mma ? 0 : (FP8 ? 2 : (PAIR ? (D_I == 128 ? 2 : 4) : (D_I == 128 ? 4 : 6)));  // bf16 stages
  static constexpr int kRawStages = kF8Mma ? 6 : (FP8 ? 4 : 0);
  static constexpr int kQSlots = PAIR ? 2 : 1;
  // a slot: the group's stacked query columns, bf16 (or f16) in kBlocks
  // 64-dim blocks; kF8Mma: the e4m3 high parts, then the low parts, 128 B
  // per column each (the same 64 KB)
  static constexpr int kQSlotBytes = kMaxCols * D_I * 2;
  static constexpr int kQPartBytes = kMaxCols * 128;
  static constexpr int kQBytes = kQSlots * kQSlotBytes;
  // 8 epilogue warps, two per TMEM lane quadrant, each reducing one half of
  // the columns (two warps per SM sub-partition hide each other's TMEM-load
  // and FMA latencies; measured: four per quadrant at the 96 registers of 18
  // warps spill and run slower); e4m3 keys add 4 converter warps (measured at
  // the 1M-token per-query shape: 260 us, against 292 us with 4 epilogue
  // warps reducing whole rows, whose two 64-column loads in flight spilled).
  static constexpr int kEpiWarps = 8;
  static constexpr int kHalves = 2;
  static constexpr int kEpiThreads = kEpiWarps * 32;
  static constexpr int kConvWarps = FP8 ? 4 : 0;  // e4m3 -> f16 converter warps
  static constexpr int kConvThreads = kConvWarps * 32;
  static constexpr int kThreads = (kEpiWarp0 + kEpiWarps + kConvWarps) * 32;
  // smem layout offsets (from a 1024-aligned base)
  static constexpr int kOffStages = 0;
  static constexpr int kOffRaw = kOffStages + kStages * kTileBytes;
  static constexpr int kOffQ = kOffRaw + kRawStages * kRawBytes;
  static constexpr int kOffW = kOffQ + kQBytes;
  static constexpr int kOffNv = kOffW + kQSlots * kMaxCols * 4;
  static constexpr int kOffQs = kOffNv + kQSlots * 16 * 8;        // kF8Mma: 1 / s of each query column
  static constexpr int kOffBar = kOffQs + (kF8Mma ? kMaxCols * 4 : 0);
  static constexpr int kNumBars = 2 * kStages + 2 * kRawStages + 4 + 3;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  static_assert(!(FP8 && PAIR), "e4m3 keys take one group per tile");
  static_assert(kOffQ % 1024 == 0 && kRawBytes % 1024 == 0, "swizzled operands 1024-byte aligned");
  static_assert(kSmemBytes <= 232448, "fits one CTA per SM");
};

// DUAL: the group's heads fill at most half of the accumulator columns
// (n <= 128, one group per tile), so a work item takes two consecutive key
// tiles: the first accumulates into columns [0, n), the second into
// [128, 128 + n), and each half of the epilogue warps reduces one tile.
template <int D_I, int HP, bool FP8, bool PAIR, bool DUAL>
__global__ void __launch_bounds__(IdxCfg<D_I, FP8, PAIR>::kThreads, 1)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                      const IndexerArgs a) {
  using C = IdxCfg<D_I, FP8, PAIR>;
  static_assert(!(DUAL && PAIR), "two tiles per item take one query group");
  constexpr int P = C::kQSlots;  // query groups per work item
  constexpr int TPI = DUAL ? 2 : 1;  // key tiles per work item
  constexpr int GMAX = kMaxCols / HP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem + C::kOffStages;
  uint8_t* raw = smem + C::kOffRaw;
  uint8_t* qs = smem + C::kOffQ;
  float* ws = reinterpret_cast<float*>(smem + C::kOffW);
  int64_t* nvs = reinterpret_cast<int64_t*>(smem + C::kOffNv);
  float* qinv = reinterpret_cast<float*>(smem + C::kOffQs);  // kF8Mma
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;                          // [kStages] bf16 tile ready
  uint64_t* empty = full + C::kStages;            // [kStages] bf16 tile consumed
  uint64_t* raw_full = empty + C::kStages;        // [kRawStages]
  uint64_t* raw_empty = raw_full + C::kRawStages; // [kRawStages]
  uint64_t* acc_full = raw_empty + C::kRawStages; // [2]
  uint64_t* acc_empty = acc_full + 2;             // [2]
  uint64_t* q_ready = acc_empty + 2;              // [1]
  uint64_t* mma_done = q_ready + 1;               // [1] every MMA issued has completed
  uint64_t* q_conv = mma_done + 1;                // [1] (e4m3 keys) the queries are in f16
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_trigger();

  // This CTA's contiguous share of the work list: item (pair, tile) covers
  // query groups P pair .. P pair + P - 1 (fewer at the end) on one key tile
  // (DUAL: item (group, j) covers one group on key tiles 2j and 2j + 1).
  const int64_t total = a.total_items;
  const int64_t lo = total * blockIdx.x / gridDim.x;
  const int64_t hi = total * (blockIdx.x + 1) / gridDim.x;
  const int ncols = a.G * HP;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full[i], FP8 ? C::kConvThreads : 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < C::kRawStages; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], C::kF8Mma ? 1 : C::kConvThreads);  // kF8Mma: freed by the MMA commit
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::kEpiThreads);
    }
    mbar_init(q_ready, 1);
    mbar_init(mma_done, 1);
    mbar_init(q_conv, FP8 ? C::kConvThreads : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&qmap);
  }
  pdl_wait();
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int64_t jt = 0;  // key tiles loaded (the stage sequence)
      bool ok = true;
      for (int64_t wi = lo; wi < hi && ok; ++wi) {
        const int grp = static_cast<int>(wi / a.tiles) * P;  // first group of the item
        const int t0 = static_cast<int>(wi % a.tiles) * TPI;
        const int z = a.per_query ? grp : 0;
        // (a second tile past the end reads as zeros; its scores are not stored)
        for (int h = 0; h < TPI; ++h, ++jt) {
          if constexpr (!FP8) {
            const int st = static_cast<int>(jt % C::kStages);
            const uint32_t ph = static_cast<uint32_t>((jt / C::kStages) & 1);
            if (!mbar_wait(&empty[st], ph ^ 1, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
            mbar_arrive_expect_tx(&full[st], C::kTileBytes);
#pragma unroll
            for (int bk = 0; bk < C::kBlocks; ++bk)
              tma_load_3d(stages + st * C::kTileBytes + bk * (kTileKeys * 128), &kmap, &full[st], bk * 64,
                          (t0 + h) * kTileKeys, z);
          } else {
            const int st = static_cast<int>(jt % C::kRawStages);
            const uint32_t ph = static_cast<uint32_t>((jt / C::kRawStages) & 1);
            if (!mbar_wait(&raw_empty[st], ph ^ 1, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
            mbar_arrive_expect_tx(&raw_full[st], C::kRawBytes);
            tma_load_3d(raw + st * C::kRawBytes, &kmap, &raw_full[st], 0, (t0 + h) * kTileKeys, z);
          }
        }
      }
      if (*abort_flag) {
        // wind down: let every load this thread issued land before exiting
        const int S = FP8 ? C::kRawStages : C::kStages;
        uint64_t* fb = FP8 ? raw_full : full;
        const int64_t issued = jt;  // loads actually issued before the abort
        for (int64_t j = (issued > S ? issued - S : 0); j < issued; ++j)
          mbar_drain(&fb[j % S], static_cast<uint32_t>((j / S) & 1));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // bf16 keys: bf16 x bf16; e4m3 keys: e4m3 x e4m3 (kF8Mma) or both
      // operands widened to f16 -- format 0 of kind::f8f6f4 and of kind::f16
      // alike, so one descriptor serves both
      const uint32_t idesc = FP8 ? idesc_f16_f32(128, ncols) : idesc_bf16_f32(128, ncols, false, false);
      const uint32_t q_addr = smem_u32(qs);
      int cur_grp = -1;
      uint32_t q_phase = 0;
      int64_t it = 0, si = 0;  // items; (item, group) sub-items -> accumulator si & 1
      int64_t jt = 0;          // key tiles consumed (the stage sequence)
      bool ok = true;
      // key tile j: wait until it is in shared memory; its operand address
      auto tile_in = [&](int64_t j, uint32_t& a_addr) -> bool {
        if constexpr (C::kF8Mma) {
          const int rs = static_cast<int>(j % C::kRawStages);
          if (!mbar_wait(&raw_full[rs], static_cast<uint32_t>((j / C::kRawStages) & 1), abort_flag, a.status,
                         a.wait_ns))
            return false;
          a_addr = smem_u32(raw + rs * C::kRawBytes);
        } else {
          const int st = static_cast<int>(j % C::kStages);
          if (!mbar_wait(&full[st], static_cast<uint32_t>((j / C::kStages) & 1), abort_flag, a.status, a.wait_ns))
            return false;
          a_addr = smem_u32(stages + st * C::kTileBytes);
        }
        tc_fence_after();
        return true;
      };
      // D[128 keys x ncols] (+)= tile . Q^T over d_I
      auto tile_mma = [&](uint32_t d_tmem, uint32_t a_addr, uint32_t qb) {
        if constexpr (C::kF8Mma) {
#pragma unroll
          for (int part = 0; part < 2; ++part)  // high, then low parts of the queries
#pragma unroll
            for (int kk = 0; kk < D_I / 32; ++kk)
              mma_e4m3_ss(d_tmem, sw128_desc(a_addr + kk * 32, 16, 1024),
                          sw128_desc(qb + part * C::kQPartBytes + kk * 32, 16, 1024), idesc, (part | kk) != 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < D_I / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * (kTileKeys * 128) + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * (kMaxCols * 128) + (kk & 3) * 32;
            mma_bf16_ss(d_tmem, sw128_desc(a_addr + koff, 16, 1024), sw128_desc(qb + qoff, 16, 1024), idesc,
                        kk > 0 ? 1u : 0u);
          }
        }
      };
      // the stage of key tile j is free once the MMAs issued so far complete
      auto tile_out = [&](int64_t j) {
        if constexpr (C::kF8Mma) mma_commit(&raw_empty[j % C::kRawStages]);
        else mma_commit(&empty[j % C::kStages]);
      };
      for (int64_t wi = lo; wi < hi && ok; ++wi, ++it) {
        const int grp = static_cast<int>(wi / a.tiles) * P;
        const int ng = P == 1 ? 1 : (a.groups - grp < P ? a.groups - grp : P);
        if (grp != cur_grp) {
          if (!mbar_wait(FP8 ? q_conv : q_ready, q_phase, abort_flag, a.status, a.wait_ns)) break;
          q_phase ^= 1;
          cur_grp = grp;
        }
        if constexpr (DUAL) {
          // one accumulator, two key tiles: columns [0, n) and [128, 128 + n)
          const int acc = static_cast<int>(si & 1);
          const uint32_t aph = static_cast<uint32_t>((si >> 1) & 1);
          if (!mbar_wait(&acc_empty[acc], aph ^ 1, abort_flag, a.status, a.wait_ns)) break;
          tc_fence_after();
          for (int h = 0; h < 2 && ok; ++h, ++jt) {
            uint32_t a_addr;
            if (!tile_in(jt, a_addr)) { ok = false; break; }
            tile_mma(tmem_base + acc * 256 + h * 128, a_addr, q_addr);
            tile_out(jt);
          }
          if (!ok) break;
          mma_commit(&acc_full[acc]);
          ++si;
          continue;
        }
        uint32_t a_addr;
        const int64_t j = jt++;
        if (!tile_in(j, a_addr)) break;
        for (int sub = 0; sub < ng; ++sub, ++si) {
          const int acc = static_cast<int>(si & 1);
          const uint32_t aph = static_cast<uint32_t>((si >> 1) & 1);
          if (!mbar_wait(&acc_empty[acc], aph ^ 1, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
          tc_fence_after();
          tile_mma(tmem_base + acc * 256, a_addr, q_addr + sub * C::kQSlotBytes);
          mma_commit(&acc_full[acc]);
        }
        if (!ok) break;
        tile_out(j);
      }
      // make sure nothing issued is still running before TMEM is released
      mma_commit(mma_done);
      mbar_drain(mma_done, 0u);
    }
  } else if (warp < kEpiWarp0 + C::kEpiWarps) {
    // ------------------------------------------------------------ epilogue
    constexpr int kNumEpiThreads = C::kEpiThreads;
    const int et = threadIdx.x - kEpiWarp0 * 32;    // 0 .. kNumEpiThreads-1
    const int quad = warp & 3;                       // TMEM lane quadrant this warp may access
    const int half = (warp - kEpiWarp0) >> 2;        // which half of the columns
    const int row = quad * 32 + lane;                // key row inside the tile
    int cur_grp = -1;
    int64_t si = 0;  // (item, group) sub-items, as counted by the MMA issuer
    uint32_t q_loads = 0;  // query-slot loads issued (by thread et == 0)
    uint32_t conv_phase = 0;  // kF8Mma: the converters' query splits completed
    bool got = true;
    // A warp that gives up on a wait (got = false) does no more work but
    // keeps meeting every named barrier of the epilogue, so the eight warps
    // always take the same barriers; at the next query group they all leave
    // together.
    for (int64_t wi = lo; wi < hi; ++wi) {
      const int grp = static_cast<int>(wi / a.tiles) * P;
      const int ng = P == 1 ? 1 : (a.groups - grp < P ? a.groups - grp : P);
      const int t = static_cast<int>(wi % a.tiles);
      if (grp != cur_grp) {
        // All MMAs of the previous item's groups finished (their accumulators
        // were drained below), so Q and the weights can be replaced.
        if (named_bar_or(1, kNumEpiThreads, !got || *abort_flag != 0)) break;
        // Q of each slot: one TMA load per 64-dim block of the box (d_I 64,
        // HP heads, G queries), written in the 128-byte-swizzled K-major
        // layout the MMA reads; heads past H_I and queries past B are zero
        // filled. The MMA issuer waits for the bytes on q_ready.
        ++q_loads;
        if (et == 0) {
          if constexpr (C::kF8Mma) {
            mbar_arrive(q_ready);  // the slot is free: the converters read the queries themselves
          } else {
            mbar_arrive_expect_tx(q_ready, static_cast<uint32_t>(ng * C::kBlocks * HP * a.G * 128));
            for (int slot = 0; slot < ng; ++slot)
#pragma unroll
              for (int bk = 0; bk < C::kBlocks; ++bk)
                tma_load_3d(qs + slot * C::kQSlotBytes + bk * (kMaxCols * 128), &qmap, q_ready, bk * 64, 0,
                            (grp + slot) * a.G);
          }
        }
        for (int slot = 0; slot < ng; ++slot) {
          const int b0 = (grp + slot) * a.G;
          float* wslot = ws + slot * kMaxCols;
          for (int i = et; i < kMaxCols; i += kNumEpiThreads) {
            const int ii = DUAL ? (i & 127) : i;  // (DUAL: both halves hold the group's heads)
            const int g = ii / HP, h = ii % HP, b = b0 + g;
            wslot[i] = (g < a.G && h < a.H_I && b < a.B) ? a.w[static_cast<int64_t>(b) * a.H_I + h] : 0.f;
          }
          if (et < GMAX) {
            const int b = b0 + et;
            nvs[slot * 16 + et] = (et < a.G && b < a.B) ? (a.n_valid ? a.n_valid[b] : a.N) : 0;
          }
        }
        named_bar_sync(1, kNumEpiThreads);
        if constexpr (C::kF8Mma) {
          // the weights of the columns split as q s = hi + lo become w / s
          const bool fail = !mbar_wait(q_conv, conv_phase, abort_flag, a.status, a.wait_ns);
          conv_phase ^= 1;
          if (named_bar_or(1, kNumEpiThreads, fail)) {  // every epilogue thread leaves together
            got = false;
            break;
          }
          for (int i = et; i < kMaxCols; i += kNumEpiThreads) {
            const int col = DUAL ? (i & 127) : i;  // (columns past ncols: weight 0, qinv unwritten)
            if (col < ncols) ws[i] *= qinv[col];
          }
          named_bar_sync(1, kNumEpiThreads);
        }
        cur_grp = grp;
      }
      if (!got) {
        si += ng;  // (this warp gave up: no waits or work until the next group's barrier)
        continue;
      }
      for (int sub = 0; sub < ng; ++sub, ++si) {
      const int acc = static_cast<int>(si & 1);
      const uint32_t aph = static_cast<uint32_t>((si >> 1) & 1);
      // (DUAL: half h reduces key tile 2 t + h)
      const int64_t s = static_cast<int64_t>(DUAL ? 2 * t + half : t) * kTileKeys + row;
      // e4m3 keys: this key's scale, requested before the accumulator wait
      // so that its latency is hidden behind it
      float scale = 1.f;
      if constexpr (FP8) {
        const int64_t zb = a.per_query ? grp + sub : 0;
        if (s < a.N) scale = __ldg(a.k_scale + zb * a.scale_batch_stride + s);
      }
      got = mbar_wait(&acc_full[acc], aph, abort_flag, a.status, a.wait_ns);
      got = __all_sync(0xffffffffu, got);  // tcgen05.ld below is warp-collective: one answer per warp
      if (!got) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * 256;
      const int b0 = (grp + sub) * a.G;
      const float* wsl = ws + sub * kMaxCols;
      const int64_t* nvsl = nvs + sub * 16;
      // One half of the columns = a contiguous run of whole queries.
      auto tile_half = [&](auto half_c) {
        constexpr int H = decltype(half_c)::value;
        // last column of this half's accumulator that the MMAs wrote
        const int lim = DUAL ? H * 128 + ncols : ncols;
        constexpr int kChunks = kMaxCols / 32 / C::kHalves;  // 32-column chunks of this half
        constexpr int kC0 = H * kChunks;
        constexpr int kQ = GMAX / C::kHalves;                 // queries of this half
        constexpr int kQ0 = H * kQ;
        // Four partial sums per query keep the FMA dependency chains short:
        // for 64 or more heads two packed pairs (columns 4i, 4i+1 and 4i+2,
        // 4i+3; one packed FMA per two columns), else NP scalars (more
        // queries per warp; packed pairs would spill).
        constexpr bool kPacked = HP >= 64;
        constexpr int NP = HP >= 64 ? 4 : (HP == 32 ? 2 : 1);
        float2 sum2[kPacked ? kQ : 1][2];
        float sum[kPacked ? 1 : kQ][NP];
#pragma unroll
        for (int g = 0; g < (kPacked ? kQ : 1); ++g) sum2[g][0] = sum2[g][1] = make_float2(0.f, 0.f);
#pragma unroll
        for (int g = 0; g < (kPacked ? 1 : kQ); ++g)
#pragma unroll
          for (int p = 0; p < NP; ++p) sum[g][p] = 0.f;
        // The half's columns come in as two 64-column TMEM loads issued back
        // to back with a single wait: one load latency per tile, not one per
        // 32 columns.
        static_assert(kChunks == 4 || kChunks == 8, "half = 128 or 256 columns");
        constexpr int kLoads = kChunks / 2;  // 64-column loads of this half
        constexpr int kPerWait = C::kHalves == 1 ? 2 : 1;  // 64-column loads per wait (whole rows)
        // w * ReLU(logit) for 32 columns starting at cbase (their weights:
        // kWBatch 16-byte loads issued back to back, then used)
        constexpr int kWBatch = 8;
        auto reduce32 = [&](const auto& rvv, int off, int cbase) {
#pragma unroll
          for (int k0 = 0; k0 < 8; k0 += kWBatch) {
          float4 wv[8];
#pragma unroll
          for (int k = k0; k < k0 + kWBatch; ++k) wv[k] = ld_shared_v4f(wsl + cbase + 4 * k);
#pragma unroll
          for (int k = k0; k < k0 + kWBatch; ++k) {
            const int j = 4 * k;  // 4 columns of one query (HP is a multiple of 16)
            if constexpr (kPacked) {
              float2 (&acc)[2] = sum2[(cbase + j) / HP - kQ0];
              const float2 x01 = make_float2(fmaxf(__uint_as_float(rvv[off + j]), 0.f),
                                             fmaxf(__uint_as_float(rvv[off + j + 1]), 0.f));
              const float2 x23 = make_float2(fmaxf(__uint_as_float(rvv[off + j + 2]), 0.f),
                                             fmaxf(__uint_as_float(rvv[off + j + 3]), 0.f));
              acc[0] = ffma2(make_float2(wv[k].x, wv[k].y), x01, acc[0]);
              acc[1] = ffma2(make_float2(wv[k].z, wv[k].w), x23, acc[1]);
            } else {
              const float wj[4] = {wv[k].x, wv[k].y, wv[k].z, wv[k].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float& acc_ref = sum[(cbase + j + e) / HP - kQ0][(j + e) % NP];
                acc_ref = fmaf(wj[e], fmaxf(__uint_as_float(rvv[off + j + e]), 0.f), acc_ref);
              }
            }
          }
          }
        };
        if constexpr (kPerWait == 1) {
          const int c0 = kC0 * 32;
          if (c0 + kChunks * 32 <= lim) {
            // every column of the half is present: 64-column TMEM loads, the
            // next one in flight while the current one is reduced
            uint32_t ra[64], rb[64];
            tmem_ld64_issue(taddr + c0, ra);
            tmem_ld_wait64(ra);
#pragma unroll
            for (int c = 0; c < kLoads; c += 2) {
              tmem_ld64_issue(taddr + c0 + (c + 1) * 64, rb);
              reduce32(ra, 0, c0 + c * 64);
              reduce32(ra, 32, c0 + c * 64 + 32);
              tmem_ld_wait64(rb);
              if (c + 2 < kLoads) tmem_ld64_issue(taddr + c0 + (c + 2) * 64, ra);
              reduce32(rb, 0, c0 + (c + 1) * 64);
              reduce32(rb, 32, c0 + (c + 1) * 64 + 32);
              if (c + 2 < kLoads) tmem_ld_wait64(ra);
            }
          } else {
            // a partial half: one 64-column load at a time
#pragma unroll
            for (int pass = 0; pass < kLoads; ++pass) {
              const int cA = c0 + 64 * pass;
              if (cA < lim) {
                uint32_t ra[64];
                tmem_ld64_issue(taddr + cA, ra);
                tmem_ld_wait64(ra);
                reduce32(ra, 0, cA);
                reduce32(ra, 32, cA + 32);
              }
            }
          }
        } else {
          // whole rows: two 64-column loads in flight per wait
#pragma unroll
          for (int pass = 0; pass < kLoads; pass += 2) {
            const int cA = (kC0 + 2 * pass) * 32, cB = cA + 64;
            const bool haveA = cA < lim, haveB = cB < lim && pass + 1 < kLoads;
            uint32_t ra[64], rb[64];
            if (haveA) tmem_ld64_issue(taddr + cA, ra);
            if (haveB) tmem_ld64_issue(taddr + cB, rb);
            if (haveA) tmem_ld_wait64(ra);
            if (haveB) tmem_ld_wait64(rb);
            if (haveA) {
              reduce32(ra, 0, cA);
              reduce32(ra, 32, cA + 32);
            }
            if (haveB) {
              reduce32(rb, 0, cB);
              reduce32(rb, 32, cB + 32);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[acc]);
        if (s < a.N) {
#pragma unroll
          for (int g = 0; g < kQ; ++g) {
            const int gg = DUAL ? g : kQ0 + g;  // (DUAL: both halves hold the same queries)
            if (gg < a.G && b0 + gg < a.B) {
              float tot = 0.f;
              if constexpr (kPacked) {
                tot = (sum2[g][0].x + sum2[g][0].y) + (sum2[g][1].x + sum2[g][1].y);
              } else {
#pragma unroll
                for (int p = 0; p < NP; ++p) tot += sum[g][p];
              }
              const float val = (s < nvsl[gg]) ? tot * scale : -INFINITY;
              a.scores[static_cast<int64_t>(b0 + gg) * a.N + s] = val;
            }
          }
        }
      };
      if constexpr (C::kHalves == 2) {
        if (half == 0) tile_half(std::integral_constant<int, 0>{});
        else tile_half(std::integral_constant<int, 1>{});
      } else {
        tile_half(std::integral_constant<int, 0>{});
      }
      }
    }
    // the last query-slot load this thread issued has landed before the CTA
    // can exit (it is otherwise waited on only by the MMA issuer, which may
    // have given up)
    if (et == 0 && q_loads > 0) mbar_drain(q_ready, (q_loads - 1) & 1u);
  } else if constexpr (FP8) {
    // ------------------------------------------------------------ e4m3 -> f16
    const int ct = threadIdx.x - (kEpiWarp0 + C::kEpiWarps) * 32;  // 0 .. kConvThreads - 1
    if constexpr (C::kF8Mma) {
      // Once per query group, each query column (head h of query b) split as
      // q s = hi + lo into the slot's two e4m3 operands (128-byte rows,
      // 128-byte swizzle), 1 / s to qinv; the slot is rewritten only after
      // the previous group's MMAs have completed (the epilogue frees it).
      int cur_grp = -1;
      uint32_t q_phase = 0;
      const uint32_t qhi = smem_u32(qs), qlo = qhi + C::kQPartBytes;
      for (int64_t wi = lo; wi < hi; ++wi) {
        const int grp = static_cast<int>(wi / a.tiles) * P;
        if (grp == cur_grp) continue;
        if (!mbar_wait(q_ready, q_phase, abort_flag, a.status, a.wait_ns)) break;
        q_phase ^= 1;
        cur_grp = grp;
        const int b0 = grp * a.G;
        for (int r = ct; r < ncols; r += C::kConvThreads) {
          const int g = r / HP, h = r % HP, b = b0 + g;
          const bool valid = g < a.G && h < a.H_I && b < a.B;
          const uint4* src = reinterpret_cast<const uint4*>(a.q + (static_cast<int64_t>(b) * a.H_I + h) * D_I);
          // two passes over the column's 256 bytes (few registers: these
          // warps share the register budget of the epilogue)
          float mx = 0.f;
#pragma unroll 1
          for (int c = 0; c < D_I / 8; ++c) {
            const uint4 x = valid ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
            const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(bf16_lane(w4[e >> 1], e & 1)));
          }
          // s = 2^(7 - E) for 2^E <= mx < 2^(E + 1): mx s in [128, 256)
          int E = static_cast<int>((__float_as_uint(mx) >> 23) & 0xFFu) - 127;
          E = E < -119 ? -119 : E;
          const float sc = __uint_as_float(static_cast<uint32_t>(127 + 7 - E) << 23);
          qinv[r] = mx > 0.f ? __uint_as_float(static_cast<uint32_t>(127 - 7 + E) << 23) : 1.f;
#pragma unroll 1
          for (int c = 0; c < D_I / 16; ++c) {  // 16 elements: one 16-byte chunk of codes
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) hw[j] = lw[j] = 0u;
#pragma unroll
            for (int half = 0; half < 2; ++half) {  // elements 16 c + 8 half .. + 7
              const uint4 x = valid ? __ldg(src + 2 * c + half) : make_uint4(0, 0, 0, 0);
              const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
              for (int e = 0; e < 8; ++e) {  // element 8 half + e of the chunk: byte (8 half + e) % 4 of word
                const float v = bf16_lane(w4[e >> 1], e & 1) * sc;
                const __nv_fp8_storage_t hc = __nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
                const float hv = __half2float(__half(__nv_cvt_fp8_to_halfraw(hc, __NV_E4M3)));
                const __nv_fp8_storage_t lc = __nv_cvt_float_to_fp8(v - hv, __NV_SATFINITE, __NV_E4M3);
                const int k = 8 * half + e;  // 0 .. 15, lowest byte first
                hw[k >> 2] |= static_cast<uint32_t>(hc) << (8 * (k & 3));
                lw[k >> 2] |= static_cast<uint32_t>(lc) << (8 * (k & 3));
              }
            }
            st_shared_v4(qhi + sw128_offset(r, c), make_uint4(hw[0], hw[1], hw[2], hw[3]));
            st_shared_v4(qlo + sw128_offset(r, c), make_uint4(lw[0], lw[1], lw[2], lw[3]));
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(q_conv);
      }
    } else {
      int64_t jt = 0;  // key tiles converted (the stage sequence)
      int cur_grp = -1;
      uint32_t q_phase = 0;
      bool ok = true;
      for (int64_t wi = lo; wi < hi && ok; ++wi) {
        const int grp = static_cast<int>(wi / a.tiles) * P;
        if (grp != cur_grp) {
          // the group's queries, staged as bf16 by TMA, become f16 in place
          // (element by element, so the swizzled positions stay); the slot is
          // rewritten only after the previous group's MMAs have completed
          if (!mbar_wait(q_ready, q_phase, abort_flag, a.status, a.wait_ns)) break;
          q_phase ^= 1;
          cur_grp = grp;
          constexpr int kRowChunks = 8;  // 16-byte chunks per 128-byte row
          const int nchunks = C::kBlocks * ncols * kRowChunks;
          for (int i = ct; i < nchunks; i += C::kConvThreads) {
            const int bk = i / (ncols * kRowChunks), rem = i % (ncols * kRowChunks);
            uint4* pq = reinterpret_cast<uint4*>(qs + bk * (kMaxCols * 128) + rem * 16);
            const uint4 v = *pq;
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const __half2 h = __floats2half2_rn(bf16_lane(w4[j], 0), bf16_lane(w4[j], 1));
              o[j] = *reinterpret_cast<const uint32_t*>(&h);
            }
            *pq = make_uint4(o[0], o[1], o[2], o[3]);
          }
          fence_proxy_async_smem();
          mbar_arrive(q_conv);
        }
        for (int h = 0; h < TPI; ++h, ++jt) {
        const int rs = static_cast<int>(jt % C::kRawStages);
        const uint32_t rph = static_cast<uint32_t>((jt / C::kRawStages) & 1);
        const int bs = static_cast<int>(jt % C::kStages);
        const uint32_t bph = static_cast<uint32_t>((jt / C::kStages) & 1);
        if (!mbar_wait(&raw_full[rs], rph, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
        if (!mbar_wait(&empty[bs], bph ^ 1, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
        const uint8_t* src = raw + rs * C::kRawBytes;
        uint8_t* dst = stages + bs * C::kTileBytes;
        constexpr int kChunks16 = D_I / 16;  // 16-element e4m3 chunks per row
#pragma unroll 2
        for (int i = ct; i < kTileKeys * kChunks16; i += C::kConvThreads) {
          const int r = i / kChunks16, c = i % kChunks16;
          const uint4 in = *reinterpret_cast<const uint4*>(src + r * D_I + c * 16);
          const uint32_t w4[4] = {in.x, in.y, in.z, in.w};
          uint32_t o[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) e4m3x4_to_f16x4(w4[j], o[2 * j], o[2 * j + 1]);
          // 16 f16 = two 16-byte chunks: element offsets c*16 and c*16+8. The
          // eight threads of a row write chunks 2(c%4) and 2(c%4)+1 of block
          // c/4; the odd block's threads write their second chunk first, so
          // each store instruction covers eight distinct chunk positions of a
          // row (no bank conflicts).
          const int e0 = c * 16;
          const uint32_t base = smem_u32(dst + (e0 >> 6) * (kTileKeys * 128));
          const int ch = (e0 & 63) >> 3;
          const bool second_first = D_I == 128 && ((c >> 2) & 1);
          const uint4 v0 = make_uint4(o[0], o[1], o[2], o[3]), v1 = make_uint4(o[4], o[5], o[6], o[7]);
          st_shared_v4(base + sw128_offset(r, second_first ? ch + 1 : ch), second_first ? v1 : v0);
          st_shared_v4(base + sw128_offset(r, second_first ? ch : ch + 1), second_first ? v0 : v1);
        }
        fence_proxy_async_smem();
        mbar_arrive(&raw_empty[rs]);
        mbar_arrive(&full[bs]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int D_I, int HP, bool FP8, bool PAIR, bool DUAL>
cudaError_t launch_indexer_inst(const CUtensorMap& map, const CUtensorMap& qmap, const IndexerArgs& a, int grid,
                                cudaStream_t stream, bool pdl) {
  using C = IdxCfg<D_I, FP8, PAIR>;
  auto kern = indexer_tc_kernel<D_I, HP, FP8, PAIR, DUAL>;
  static bool done[64] = {false};  // one flag set per template instance
  cudaError_t e = set_smem_once(kern, C::kSmemBytes, done);
  if (e != cudaSuccess) return e;
  e = launch_kernel(kern, dim3(grid), dim3(C::kThreads), C::kSmemBytes, stream, pdl, map, qmap, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D_I, bool FP8, bool PAIR, bool DUAL>
cudaError_t dispatch_hp(int HP, const CUtensorMap& map, const CUtensorMap& qmap, const IndexerArgs& a, int grid,
                        cudaStream_t s, bool pdl) {
  switch (HP) {
    case 16: return launch_indexer_inst<D_I, 16, FP8, PAIR, DUAL>(map, qmap, a, grid, s, pdl);
    case 32: return launch_indexer_inst<D_I, 32, FP8, PAIR, DUAL>(map, qmap, a, grid, s, pdl);
    case 64: return launch_indexer_inst<D_I, 64, FP8, PAIR, DUAL>(map, qmap, a, grid, s, pdl);
    case 128: return launch_indexer_inst<D_I, 128, FP8, PAIR, DUAL>(map, qmap, a, grid, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int indexer_smem_bytes(int d_I, bool fp8) {
  if (d_I == 64) return fp8 ? IdxCfg<64, true, false>::kSmemBytes : IdxCfg<64, false, true>::kSmemBytes;
  return fp8 ? IdxCfg<128, true, false>::kSmemBytes : IdxCfg<128, false, true>::kSmemBytes;
}

cudaError_t launch_indexer(const CUtensorMap& map, const CUtensorMap& qmap, const IndexerArgs& a, int HP, int d_I,
                           bool fp8, int grid, cudaStream_t stream, bool pdl) {
  const bool dual = a.dual != 0;
  if (fp8) {
    if (d_I == 64) return dual ? dispatch_hp<64, true, false, true>(HP, map, qmap, a, grid, stream, pdl)
                               : dispatch_hp<64, true, false, false>(HP, map, qmap, a, grid, stream, pdl);
    if (d_I == 128) return dual ? dispatch_hp<128, true, false, true>(HP, map, qmap, a, grid, stream, pdl)
                                : dispatch_hp<128, true, false, false>(HP, map, qmap, a, grid, stream, pdl);
    return cudaErrorInvalidValue;
  }
  if (a.pair == 2) {
    if (d_I == 64) return dispatch_hp<64, false, true, false>(HP, map, qmap, a, grid, stream, pdl);
    if (d_I == 128) return dispatch_hp<128, false, true, false>(HP, map, qmap, a, grid, stream, pdl);
    return cudaErrorInvalidValue;
  }
  if (d_I == 64) return dual ? dispatch_hp<64, false, false, true>(HP, map, qmap, a, grid, stream, pdl)
                             : dispatch_hp<64, false, false, false>(HP, map, qmap, a, grid, stream, pdl);
  if (d_I == 128) return dual ? dispatch_hp<128, false, false, true>(HP, map, qmap, a, grid, stream, pdl)
                              : dispatch_hp<128, false, false, false>(HP, map, qmap, a, grid, stream, pdl);
  return cudaErrorInvalidValue;
}

}  // namespace ic
