// Top-k selection over indexer score rows (Hy4 IndexCache explainer, Jargon
// "Top-k selection": keep the k highest-scoring cached tokens).
//
// Radix select on the order-preserving 32-bit key of each fp32 score
// (negative floats: all bits flipped; others: sign bit set). Two launches,
// neither of which ever waits on another CTA:
//   histogram  each CTA builds the 12-bit histogram of key[31:20] over its
//              slice of the row in shared memory and adds its nonzero bins
//              into the row's histogram in global memory; the last CTA of the
//              row (atomic ticket) reads it once, clears it for the next
//              call and picks the bin d1 holding the k-th key.
//   filter     keys in bins above d1 are final and are written straight to
//              the output (compacted per CTA with one warp scan per 128
//              keys, one atomic reservation per CTA); keys in bin d1 are
//              candidates, appended with their keys to a per-row buffer. The
//              last CTA of the row resolves the exact k-th key T among the
//              candidates (two more 10-bit digits), writes the candidates
//              above T, and then the r keys equal to T with the lowest
//              indices -- ties resolve toward the lower index, so the
//              selected set is deterministic -- and finally zeroes the row's
//              control words for the next call.
// If bin d1 holds more candidates than the buffer, the last CTA runs the same
// two digits over the row itself (correct, slower; only for rows whose scores
// crowd into one 1/16-octave bin).
// Rows with n_valid <= k take every valid index and pad with -1.
#include "common.cuh"
#include "kernels.h"

namespace ic {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins1 = 4096;      // first digit: key[31:20]
constexpr int kBins2 = 1024;      // second and third digits: key[19:10], key[9:0]
constexpr int kUnroll = 4;        // float4 loads in flight per lane
constexpr int kLocalCap = 2048;   // per-CTA shared buffer of indices (each list)
constexpr int kTieCap = 2048;     // ties resolved in shared memory up to this many
constexpr int kRegCand = 16;      // candidates per thread held in registers by the last CTA

// per-row control block (kCtrlWords 32-bit words, one 128-byte line per row)
enum : int {
  kAboveCount = 0,  // keys written above bin d1
  kCandCount = 1,   // candidates appended (may exceed the capacity)
  kTicket = 2,      // CTAs of the filter pass finished
  kHistTicket = 3,  // CTAs of the histogram pass finished
  kBin = 4,         // d1: the first-digit bin of the k-th key
  kBinRank = 5,     // rank of the k-th key inside bin d1
  kBinCount = 6,    // keys in bin d1 over the whole row
};

IC_DEV uint32_t score_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

IC_DEV int64_t row_valid(const TopkArgs& a, int b) {
  int64_t nv = a.n_valid ? a.n_valid[b] : a.N;
  return nv < 0 ? 0 : (nv > a.N ? a.N : nv);
}

IC_DEV uint32_t* row_ctrl(const TopkArgs& a, int b) { return a.counters + static_cast<int64_t>(b) * kCtrlWords; }

// Given per-digit counts (ascending digit) in shared memory and a 1-based
// rank kr, find the digit d holding the kr-th largest key:
//   above(d) < kr <= above(d) + counts[d],  above(d) = sum_{d' > d} counts[d'].
// Writes d and kr - above(d) to shared memory. All threads must call.
IC_DEV void select_digit(const uint32_t* counts, int nbins, uint32_t kr, int* d_out, uint32_t* kr_out,
                         uint32_t* warp_tot) {
  const int per = nbins / kThreads;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  if (t == 0) {  // defaults, overwritten below by the thread that finds the digit
    *d_out = 0;
    *kr_out = 1;
  }
  uint32_t local = 0;
  for (int j = 0; j < per; ++j) local += counts[t * per + j];
  uint32_t v = local;  // inclusive suffix sum within the warp
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t n = __shfl_down_sync(0xffffffffu, v, off);
    if (lane + off < 32) v += n;
  }
  if (lane == 0) warp_tot[warp] = v;
  __syncthreads();
  uint32_t above = v - local;
  for (int w = warp + 1; w < kWarps; ++w) above += warp_tot[w];
  if (above < kr && kr <= above + local) {
    uint32_t acc = above;
    for (int j = per - 1; j >= 0; --j) {
      const uint32_t c = counts[t * per + j];
      if (acc + c >= kr) {
        *d_out = t * per + j;
        *kr_out = kr - acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
}

// Visit positions [lo, hi) of row b: f(i, key, valid) for every position, in
// warp-uniform steps (all 32 lanes call f together), with kUnroll
// independent 16-byte loads in flight per lane.
template <typename F>
IC_DEV void for_slice(const TopkArgs& a, int b, int64_t lo, int64_t hi, F&& f) {
  const float* row = a.scores + static_cast<int64_t>(b) * a.N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool vec = ((a.N & 3) == 0) && ((lo & 3) == 0);
  if (vec) {
    constexpr int kWarpSpan = kUnroll * 128;
    for (int64_t base = lo + static_cast<int64_t>(warp) * kWarpSpan; base < hi; base += kThreads * 4 * kUnroll) {
      float4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * 128 + lane * 4;
        if (i + 3 < hi) {
          v[u] = __ldcg(reinterpret_cast<const float4*>(row + i));
        } else {
          v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (i < hi) v[u].x = __ldcg(row + i);
          if (i + 1 < hi) v[u].y = __ldcg(row + i + 1);
          if (i + 2 < hi) v[u].z = __ldcg(row + i + 2);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * 128 + lane * 4;
        f(i, score_key(v[u].x), i < hi);
        f(i + 1, score_key(v[u].y), i + 1 < hi);
        f(i + 2, score_key(v[u].z), i + 2 < hi);
        f(i + 3, score_key(v[u].w), i + 3 < hi);
      }
    }
  } else {
    for (int64_t base = lo + static_cast<int64_t>(warp) * 32 * kUnroll; base < hi; base += kThreads * kUnroll) {
      float v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * 32 + lane;
        v[u] = i < hi ? __ldcg(row + i) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * 32 + lane;
        f(i, score_key(v[u]), i < hi);
      }
    }
  }
}

// Shared-memory histogram increment (native shared atomics; measured faster
// on B200 than grouping equal bins with __match_any_sync first).
IC_DEV void hist_add(uint32_t* h, uint32_t bin, bool take) {
  if (take) atomicAdd(&h[bin], 1u);
}

// Append (i, key) to shared lists when `take` (warp-aggregated; all 32 lanes
// call). Entries past `cap` are not stored but still counted.
IC_DEV void list_push_key(int32_t* list, uint32_t* keys, uint32_t* count, uint32_t cap, int64_t i, uint32_t key,
                          bool take) {
  const uint32_t bal = __ballot_sync(0xffffffffu, take);
  if (!bal) return;
  const int lane = threadIdx.x & 31;
  uint32_t base = 0;
  if (lane == 0) base = atomicAdd(count, static_cast<uint32_t>(__popc(bal)));
  base = __shfl_sync(0xffffffffu, base, 0);
  if (take) {
    const uint32_t pos = base + __popc(bal & ((1u << lane) - 1u));
    if (pos < cap) {
      list[pos] = static_cast<int32_t>(i);
      keys[pos] = key;
    }
  }
}

// Append i to a shared list when `take` (warp-aggregated; all 32 lanes call).
// Entries past `cap` are not stored but still counted.
IC_DEV void list_push(int32_t* list, uint32_t* count, uint32_t cap, int64_t i, bool take) {
  const uint32_t bal = __ballot_sync(0xffffffffu, take);
  if (!bal) return;
  const int lane = threadIdx.x & 31;
  uint32_t base = 0;
  if (lane == 0) base = atomicAdd(count, static_cast<uint32_t>(__popc(bal)));
  base = __shfl_sync(0xffffffffu, base, 0);
  if (take) {
    const uint32_t pos = base + __popc(bal & ((1u << lane) - 1u));
    if (pos < cap) list[pos] = static_cast<int32_t>(i);
  }
}

// ------------------------------------------------------------------ pass 1
__global__ void __launch_bounds__(kThreads) topk_hist_kernel(const TopkArgs a) {
  __shared__ __align__(16) uint32_t sh_hist[kBins1];
  __shared__ uint32_t warp_tot[kWarps];
  __shared__ int sh_d;
  __shared__ uint32_t sh_kr;
  __shared__ int sh_last;
  const int b = blockIdx.y, c = blockIdx.x;
  pdl_trigger();
  pdl_wait();
  const int64_t nv = row_valid(a, b);
  if (nv <= a.k) return;  // the filter pass takes every valid index
  const int64_t lo = static_cast<int64_t>(c) * a.slice;
  const int64_t hi = lo + a.slice < nv ? lo + a.slice : nv;
  for (int j = threadIdx.x; j < kBins1; j += kThreads) sh_hist[j] = 0;
  __syncthreads();
  if (lo < hi)
    for_slice(a, b, lo, hi, [&](int64_t, uint32_t key, bool valid) { hist_add(sh_hist, key >> 20, valid); });
  __syncthreads();
  // this CTA's nonzero bins into the row's histogram (a few hundred atomics)
  uint32_t* rh = a.hist + static_cast<int64_t>(b) * kBins1;
  for (int j = threadIdx.x; j < kBins1; j += kThreads) {
    const uint32_t v = sh_hist[j];
    if (v) atomicAdd(&rh[j], v);
  }
  // the last CTA of the row picks the bin of the k-th key once for everyone
  uint32_t* ctrl = row_ctrl(a, b);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) sh_last = atomicAdd(&ctrl[kHistTicket], 1u) == static_cast<uint32_t>(a.cpr) - 1;
  __syncthreads();
  if (!sh_last) return;
  __threadfence();
  // read the whole row's histogram, and leave it zero for the next call
  for (int j = threadIdx.x; j < kBins1 / 4; j += kThreads) {
    reinterpret_cast<uint4*>(sh_hist)[j] = __ldcg(reinterpret_cast<const uint4*>(rh) + j);
    reinterpret_cast<uint4*>(rh)[j] = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  select_digit(sh_hist, kBins1, static_cast<uint32_t>(a.k), &sh_d, &sh_kr, warp_tot);
  if (threadIdx.x == 0) {
    ctrl[kBin] = static_cast<uint32_t>(sh_d);
    ctrl[kBinRank] = sh_kr;
    ctrl[kBinCount] = sh_hist[sh_d];
  }
}

// ------------------------------------------------------------------ pass 2
struct FilterShared {
  uint32_t hist[kBins1];
  int32_t above[kLocalCap];
  int32_t cand[kLocalCap];
  uint32_t cand_key[kLocalCap];
  uint32_t warp_tot[kWarps];
  uint32_t n_above, n_cand, base_above, base_cand;
  int d;
  uint32_t kr;
  int last;
};

// Exact resolution of the k-th key within bin d1 by the last CTA of the row.
// `visit(f)` enumerates (index, key, valid) for a superset of the keys of bin
// d1 (the candidate buffer, or the whole row when the buffer overflowed).
template <typename Visit>
IC_DEV void resolve_bin(const TopkArgs& a, int b, int64_t nv, uint32_t d1, uint32_t kr1, uint32_t n_above,
                        FilterShared& sh, Visit&& visit) {
  int32_t* out = a.idx + static_cast<int64_t>(b) * a.k;
  uint32_t* h = sh.hist;
  // digit 2: key[19:10]
  for (int j = threadIdx.x; j < kBins2; j += kThreads) h[j] = 0;
  __syncthreads();
  visit([&](int64_t, uint32_t key, bool ok) { hist_add(h, (key >> 10) & 0x3FFu, ok && (key >> 20) == d1); });
  __syncthreads();
  select_digit(h, kBins2, kr1, &sh.d, &sh.kr, sh.warp_tot);
  const uint32_t p2 = (d1 << 10) | static_cast<uint32_t>(sh.d);
  const uint32_t kr2 = sh.kr;
  __syncthreads();
  // digit 3: key[9:0]
  for (int j = threadIdx.x; j < kBins2; j += kThreads) h[j] = 0;
  __syncthreads();
  visit([&](int64_t, uint32_t key, bool ok) { hist_add(h, key & 0x3FFu, ok && (key >> 10) == p2); });
  __syncthreads();
  select_digit(h, kBins2, kr2, &sh.d, &sh.kr, sh.warp_tot);
  const uint32_t T = (p2 << 10) | static_cast<uint32_t>(sh.d);
  const uint32_t r = sh.kr;                      // keys equal to T to take (>= 1)
  const uint32_t n_ties = h[sh.d];               // keys equal to T
  const uint32_t n_hi = kr1 - r;                 // keys of bin d1 above T
  __syncthreads();
  // keys of bin d1 above T
  if (threadIdx.x == 0) sh.n_above = 0;
  __syncthreads();
  visit([&](int64_t i, uint32_t key, bool ok) {
    const bool take = ok && (key >> 20) == d1 && key > T;
    const uint32_t bal = __ballot_sync(0xffffffffu, take);
    if (!bal) return;
    const int lane = threadIdx.x & 31;
    uint32_t base = 0;
    if (lane == 0) base = atomicAdd(&sh.n_above, static_cast<uint32_t>(__popc(bal)));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (take) {
      const uint32_t pos = base + __popc(bal & ((1u << lane) - 1u));
      if (pos < n_hi) out[n_above + pos] = static_cast<int32_t>(i);
      else record_status(a.status, IC_ERR_BAD_INDEX);  // cannot happen with consistent counts
    }
  });
  __syncthreads();
  // the r lowest-index keys equal to T
  int32_t* tie_out = out + (a.k - r);
  if (n_ties <= static_cast<uint32_t>(kTieCap)) {
    if (threadIdx.x == 0) sh.n_cand = 0;
    __syncthreads();
    visit([&](int64_t i, uint32_t key, bool ok) { list_push(sh.cand, &sh.n_cand, kTieCap, i, ok && key == T); });
    __syncthreads();
    const uint32_t n = sh.n_cand;
    for (uint32_t x = threadIdx.x; x < n; x += kThreads) {
      const int32_t me = sh.cand[x];
      uint32_t rank = 0;  // ties with a lower index
      for (uint32_t y = 0; y < n; ++y) rank += sh.cand[y] < me;
      if (rank < r) tie_out[rank] = me;
    }
  } else {
    // many exact ties: scan the row in index order
    const float* row = a.scores + static_cast<int64_t>(b) * a.N;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t taken = 0;
    for (int64_t base = 0; base < nv && taken < r; base += kThreads) {
      const int64_t i = base + threadIdx.x;
      const bool tie = (i < nv) && score_key(__ldcg(row + i)) == T;
      const uint32_t bal = __ballot_sync(0xffffffffu, tie);
      if (lane == 0) sh.warp_tot[warp] = __popc(bal);
      __syncthreads();
      uint32_t before = 0, total = 0;
      for (int w = 0; w < kWarps; ++w) {
        if (w < warp) before += sh.warp_tot[w];
        total += sh.warp_tot[w];
      }
      const uint32_t pos = taken + before + __popc(bal & ((1u << lane) - 1u));
      if (tie && pos < r) tie_out[pos] = static_cast<int32_t>(i);
      taken += total;
      __syncthreads();
    }
  }
}

// Classify keys [lo, hi) of row b against bin d1, four consecutive keys per
// lane (lo a multiple of 4): 4-bit masks of the keys above bin d1 and in bin
// d1; one vote per 128 keys skips the (common) empty case, else one warp scan
// of the packed counts (above | cand << 16) gives every lane its positions in
// both shared lists. keys4(i) returns the keys of positions i .. i+3 (any
// value past hi).
template <typename Keys4>
IC_DEV void filter_scan4(FilterShared& sh, int64_t lo, int64_t hi, uint32_t d1, Keys4&& keys4) {
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  constexpr int kWarpSpan = kUnroll * 128;
  for (int64_t base = lo + static_cast<int64_t>(warp) * kWarpSpan; base < hi; base += kThreads * 4 * kUnroll) {
    uint4 kv[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) kv[u] = keys4(base + u * 128 + lane * 4);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i0 = base + u * 128 + lane * 4;
      const int64_t rem = hi - i0;  // valid keys from i0 on
      const uint32_t kk[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
      uint32_t ma = 0, mc = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t bin = kk[e] >> 20;
        const bool valid = e < rem;
        ma |= (valid && bin > d1) ? (1u << e) : 0u;
        mc |= (valid && bin == d1) ? (1u << e) : 0u;
      }
      if (__ballot_sync(0xffffffffu, (ma | mc) != 0u) == 0u) continue;
      const uint32_t cnt = static_cast<uint32_t>(__popc(ma)) | (static_cast<uint32_t>(__popc(mc)) << 16);
      uint32_t incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += n;
      }
      const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
      uint32_t ba = 0, bc = 0;
      if (lane == 31) {
        if (tot & 0xffffu) ba = atomicAdd(&sh.n_above, tot & 0xffffu);
        if (tot >> 16) bc = atomicAdd(&sh.n_cand, tot >> 16);
      }
      ba = __shfl_sync(0xffffffffu, ba, 31);
      bc = __shfl_sync(0xffffffffu, bc, 31);
      const uint32_t ex = incl - cnt;
      uint32_t pa = ba + (ex & 0xffffu), pc = bc + (ex >> 16);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if ((ma >> e) & 1u) {
          if (pa < static_cast<uint32_t>(kLocalCap)) sh.above[pa] = static_cast<int32_t>(i0 + e);
          ++pa;
        }
        if ((mc >> e) & 1u) {
          if (pc < static_cast<uint32_t>(kLocalCap)) {
            sh.cand[pc] = static_cast<int32_t>(i0 + e);
            sh.cand_key[pc] = kk[e];
          }
          ++pc;
        }
      }
    }
  }
}

IC_DEV void filter_resolve(const TopkArgs& a, int b, int64_t nv, uint32_t d1, uint32_t kr1, uint32_t n_cand_row,
                           FilterShared& sh);
IC_DEV void resolve_candidates(const TopkArgs& a, int b, int64_t nv, uint32_t d1, uint32_t kr1,
                               uint32_t n_cand_row, FilterShared& sh);

// After the scan of [lo, hi): write this CTA's final keys and candidates out
// (one reservation per list), take the row's filter ticket, and in the last
// CTA resolve bin d1 and zero the row's control words.
IC_DEV void filter_finish(const TopkArgs& a, int b, int64_t nv, int64_t lo, int64_t hi, uint32_t d1, uint32_t kr1,
                          uint32_t n_cand_row, FilterShared& sh) {
  const int t = threadIdx.x;
  int32_t* out = a.idx + static_cast<int64_t>(b) * a.k;
  uint32_t* ctrl = row_ctrl(a, b);
  const uint32_t n_above = static_cast<uint32_t>(a.k) - kr1;
  __syncthreads();
  // flush: one reservation per list per CTA; if a shared list overflowed,
  // the slice is scanned again and written through the reserved ranges
  const uint32_t na = sh.n_above, nc = sh.n_cand;
  if (t == 0) {
    sh.base_above = na ? atomicAdd(&ctrl[kAboveCount], na) : 0u;
    sh.base_cand = nc ? atomicAdd(&ctrl[kCandCount], nc) : 0u;
  }
  __syncthreads();
  int32_t* cbuf = a.cand + static_cast<int64_t>(b) * a.cand_cap;
  uint32_t* ckbuf = a.cand_key + static_cast<int64_t>(b) * a.cand_cap;
  if (na <= static_cast<uint32_t>(kLocalCap) && nc <= static_cast<uint32_t>(kLocalCap)) {
    for (uint32_t j = t; j < na; j += kThreads) {
      const uint32_t gp = sh.base_above + j;
      if (gp < n_above) out[gp] = sh.above[j];
      else record_status(a.status, IC_ERR_BAD_INDEX);
    }
    for (uint32_t j = t; j < nc; j += kThreads) {
      const uint32_t gp = sh.base_cand + j;
      if (gp < static_cast<uint32_t>(a.cand_cap)) {
        cbuf[gp] = sh.cand[j];
        ckbuf[gp] = sh.cand_key[j];
      }
    }
  } else {
    __syncthreads();
    if (t == 0) {
      sh.n_above = 0;
      sh.n_cand = 0;
    }
    __syncthreads();
    if (lo < hi)
      for_slice(a, b, lo, hi, [&](int64_t i, uint32_t key, bool valid) {
        const uint32_t bin = key >> 20;
        const bool ta = valid && bin > d1, tc = valid && bin == d1;
        const int lane = threadIdx.x & 31;
        const uint32_t ba = __ballot_sync(0xffffffffu, ta), bc = __ballot_sync(0xffffffffu, tc);
        uint32_t oa = 0, oc = 0;
        if (lane == 0) {
          if (ba) oa = atomicAdd(&sh.n_above, static_cast<uint32_t>(__popc(ba)));
          if (bc) oc = atomicAdd(&sh.n_cand, static_cast<uint32_t>(__popc(bc)));
        }
        oa = __shfl_sync(0xffffffffu, oa, 0);
        oc = __shfl_sync(0xffffffffu, oc, 0);
        const uint32_t lt = (1u << lane) - 1u;
        if (ta) {
          const uint32_t gp = sh.base_above + oa + __popc(ba & lt);
          if (gp < n_above) out[gp] = static_cast<int32_t>(i);
          else record_status(a.status, IC_ERR_BAD_INDEX);
        }
        if (tc) {
          const uint32_t gp = sh.base_cand + oc + __popc(bc & lt);
          if (gp < static_cast<uint32_t>(a.cand_cap)) {
            cbuf[gp] = static_cast<int32_t>(i);
            ckbuf[gp] = key;
          }
        }
      });
  }
  filter_resolve(a, b, nv, d1, kr1, n_cand_row, sh);
}

// Take the row's filter ticket (this CTA's keys are written out); the last
// CTA of the row resolves bin d1 and zeroes the row's control words.
IC_DEV void filter_resolve(const TopkArgs& a, int b, int64_t nv, uint32_t d1, uint32_t kr1, uint32_t n_cand_row,
                           FilterShared& sh) {
  const int t = threadIdx.x;
  uint32_t* ctrl = row_ctrl(a, b);
  // the last CTA of the row resolves bin d1
  __threadfence();
  __syncthreads();
  if (t == 0) sh.last = atomicAdd(&ctrl[kTicket], 1u) == static_cast<uint32_t>(a.cpr) - 1;
  __syncthreads();
  if (!sh.last) return;
  __threadfence();
  resolve_candidates(a, b, nv, d1, kr1, n_cand_row, sh);
  // every CTA of the row is done with the control words: leave them zero
  __syncthreads();
  if (t < kCtrlWords) ctrl[t] = 0u;
}

// The exact k-th key among the row's candidates of bin d1 (positions and keys
// in the row's candidate buffers), and the output entries it decides.
IC_DEV void resolve_candidates(const TopkArgs& a, int b, int64_t nv, uint32_t d1, uint32_t kr1,
                               uint32_t n_cand_row, FilterShared& sh) {
  const int t = threadIdx.x;
  const uint32_t n_above = static_cast<uint32_t>(a.k) - kr1;
  int32_t* cbuf = a.cand + static_cast<int64_t>(b) * a.cand_cap;
  uint32_t* ckbuf = a.cand_key + static_cast<int64_t>(b) * a.cand_cap;
  if (n_cand_row <= static_cast<uint32_t>(kRegCand * kThreads) &&
      n_cand_row <= static_cast<uint32_t>(a.cand_cap)) {
    // up to kRegCand candidates per thread (positions and keys), fetched once
    // into registers; every digit pass then runs on them
    const uint32_t n = n_cand_row;
    int32_t ci[kRegCand];
    uint32_t ck[kRegCand];
#pragma unroll
    for (int u = 0; u < kRegCand; ++u) {
      const uint32_t x = static_cast<uint32_t>(u) * kThreads + t;
      ci[u] = x < n ? __ldcg(cbuf + x) : 0;
      ck[u] = x < n ? __ldcg(ckbuf + x) : 0u;
    }
    resolve_bin(a, b, nv, d1, kr1, n_above, sh, [&](auto&& f) {
#pragma unroll
      for (int u = 0; u < kRegCand; ++u) {
        if (static_cast<uint32_t>(u) * kThreads >= n) break;  // the same for every thread
        const uint32_t x = static_cast<uint32_t>(u) * kThreads + t;
        f(static_cast<int64_t>(ci[u]), ck[u], x < n);
      }
    });
  } else if (n_cand_row <= static_cast<uint32_t>(a.cand_cap)) {
    // a larger bin: batches of 8 candidates per thread per round trip
    const uint32_t n = n_cand_row;
    resolve_bin(a, b, nv, d1, kr1, n_above, sh, [&](auto&& f) {
      for (uint32_t base = 0; base < n; base += 8 * kThreads) {  // warp-uniform bound
        int32_t bi[8];
        uint32_t bk[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t x = base + static_cast<uint32_t>(u) * kThreads + t;
          bi[u] = x < n ? __ldcg(cbuf + x) : 0;
          bk[u] = x < n ? __ldcg(ckbuf + x) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t x = base + static_cast<uint32_t>(u) * kThreads + t;
          f(static_cast<int64_t>(bi[u]), bk[u], x < n);
        }
      }
    });
  } else {
    resolve_bin(a, b, nv, d1, kr1, n_above, sh, [&](auto&& f) { for_slice(a, b, 0, nv, f); });
  }
}

// Rows with n_valid <= k: every valid index, padded with -1 (CTA 0 of the row).
IC_DEV bool small_row(const TopkArgs& a, int b, int c, int64_t nv) {
  if (nv > a.k) return false;
  if (c == 0) {
    int32_t* out = a.idx + static_cast<int64_t>(b) * a.k;
    for (int i = threadIdx.x; i < a.k; i += kThreads) out[i] = i < nv ? i : -1;
  }
  return true;
}

__global__ void __launch_bounds__(kThreads) topk_filter_kernel(const TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  FilterShared& sh = *reinterpret_cast<FilterShared*>(smem_raw);
  const int b = blockIdx.y, c = blockIdx.x;
  const int t = threadIdx.x;
  pdl_trigger();
  pdl_wait();
  const int64_t nv = row_valid(a, b);
  if (small_row(a, b, c, nv)) return;
  uint32_t* ctrl = row_ctrl(a, b);
  // the bin of the k-th key, chosen by the histogram pass
  const uint32_t d1 = __ldcg(&ctrl[kBin]);
  const uint32_t kr1 = __ldcg(&ctrl[kBinRank]);        // rank of the k-th key inside bin d1
  const uint32_t n_cand_row = __ldcg(&ctrl[kBinCount]); // keys in bin d1 (whole row)
  if (t == 0) {
    sh.n_above = 0;
    sh.n_cand = 0;
  }
  __syncthreads();
  const int64_t lo = static_cast<int64_t>(c) * a.slice;
  const int64_t hi = lo + a.slice < nv ? lo + a.slice : nv;
  if (lo < hi) {
    if (((a.N & 3) == 0) && ((lo & 3) == 0)) {
      const float* row = a.scores + static_cast<int64_t>(b) * a.N;
      filter_scan4(sh, lo, hi, d1, [&](int64_t i) {
        float4 v;
        if (i + 3 < hi) {
          v = __ldcg(reinterpret_cast<const float4*>(row + i));
        } else {
          v = make_float4(0.f, 0.f, 0.f, 0.f);
          if (i < hi) v.x = __ldcg(row + i);
          if (i + 1 < hi) v.y = __ldcg(row + i + 1);
          if (i + 2 < hi) v.z = __ldcg(row + i + 2);
        }
        return make_uint4(score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w));
      });
    } else {
      for_slice(a, b, lo, hi, [&](int64_t i, uint32_t key, bool valid) {
        const uint32_t bin = key >> 20;
        // a few percent of the keys reach bin d1: one vote skips the rest
        if (__ballot_sync(0xffffffffu, valid && bin >= d1) == 0u) return;
        list_push(sh.above, &sh.n_above, kLocalCap, i, valid && bin > d1);
        list_push_key(sh.cand, sh.cand_key, &sh.n_cand, kLocalCap, i, key, valid && bin == d1);
      });
    }
  }
  filter_finish(a, b, nv, lo, hi, d1, kr1, n_cand_row, sh);
}

// ------------------------------------------------------------------ one launch
// Both passes in one kernel, one thread-block cluster per row (C <= 4 CTAs,
// one per SM, each a slice of at most kFusedSlice keys kept in shared
// memory; measured on B200: the CTAs of larger clusters are spread one per SM
// and the grid then runs in several waves). The CTAs of
// a row exchange histograms, counts and the chosen bin through distributed
// shared memory between cluster barriers, so nothing is kept in global memory
// between calls and no CTA waits on a flag:
//   1 keys of the slice into shared memory and their 12-bit histogram;
//   2 CTA r sums bins [r 4096/C, (r+1) 4096/C) over the cluster; every CTA
//     finds the portion and then the bin d1 holding the k-th key;
//   3 each CTA counts its keys above d1 and in d1, takes its offsets from the
//     lower-ranked CTAs' counts and writes final keys and candidates straight
//     to their positions;
//   4 CTA 0 resolves the k-th key among the candidates.
constexpr int kFusedSlice = 32768;  // keys per CTA slice kept in shared memory
constexpr int kSliceVecs = kFusedSlice / (kThreads * 4);  // float4 loads per thread
static_assert(kFusedSlice % (kThreads * 4 * kUnroll) == 0, "whole groups per lane");

struct FusedShared {
  FilterShared f;
  __align__(16) uint32_t part[kBins1];  // this CTA's portion of the row histogram
  uint32_t portion_total;
  uint32_t na, nc;        // this CTA's keys above bin d1 / in bin d1
  uint32_t pq, krp;       // portion holding the k-th key, rank inside it
  uint32_t wsum[kWarps];
  __align__(16) uint32_t keys[kFusedSlice + 4];
};

__global__ void __launch_bounds__(kThreads, 1) topk_cluster_kernel(const TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  FusedShared& fs = *reinterpret_cast<FusedShared*>(smem_raw);
  FilterShared& sh = fs.f;
  const int b = blockIdx.y;
  const int C = a.cpr;                           // cluster = the row's CTAs
  const uint32_t r = cluster_ctarank();
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  pdl_trigger();
  pdl_wait();
  const int64_t nv = row_valid(a, b);
  // the whole cluster takes this branch together, before any cluster barrier
  if (small_row(a, b, static_cast<int>(r), nv)) return;
  const int64_t lo = static_cast<int64_t>(r) * a.slice;
  const int64_t hi = lo + a.slice < nv ? lo + a.slice : nv;
  const int n = lo < hi ? static_cast<int>(hi - lo) : 0;  // <= kFusedSlice
  for (int j = t; j < kBins1; j += kThreads) sh.hist[j] = 0;
  __syncthreads();
  // 1: keys and histogram; every load of the slice is in flight at once
  {
    const float* row = a.scores + static_cast<int64_t>(b) * a.N + lo;
    float4 v[kSliceVecs];
#pragma unroll
    for (int u = 0; u < kSliceVecs; ++u) {
      const int j = (u * kThreads + t) * 4;
      if (j + 3 < n) {
        v[u] = __ldcg(reinterpret_cast<const float4*>(row + j));
      } else {
        v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j < n) v[u].x = __ldcg(row + j);
        if (j + 1 < n) v[u].y = __ldcg(row + j + 1);
        if (j + 2 < n) v[u].z = __ldcg(row + j + 2);
      }
    }
#pragma unroll
    for (int u = 0; u < kSliceVecs; ++u) {
      const int j = (u * kThreads + t) * 4;
      if (j < n) {
        const uint4 kv = make_uint4(score_key(v[u].x), score_key(v[u].y), score_key(v[u].z), score_key(v[u].w));
        *reinterpret_cast<uint4*>(&fs.keys[j]) = kv;
        hist_add(sh.hist, kv.x >> 20, true);
        hist_add(sh.hist, kv.y >> 20, j + 1 < n);
        hist_add(sh.hist, kv.z >> 20, j + 2 < n);
        hist_add(sh.hist, kv.w >> 20, j + 3 < n);
      }
    }
  }
  __syncthreads();
  cluster_sync();
  // 2: CTA r sums bins [r P, (r+1) P) of the cluster's histograms (16-byte
  // remote loads, consecutive across lanes) and their total; the portion
  // holding the k-th key is found from the C totals, and every CTA selects
  // the bin d1 inside it from that portion's sums
  const int P = kBins1 / C;
  {
    const uint4* hist4 = reinterpret_cast<const uint4*>(sh.hist);
    uint32_t mine = 0;
    for (int j = t; j < P / 4; j += kThreads) {
      uint4 hv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        hv[q] = q < C ? ld_dsmem_v4(dsmem_addr(&hist4[r * (P / 4) + j], static_cast<uint32_t>(q)))
                      : make_uint4(0, 0, 0, 0);
      uint4 sum;
      sum.x = (hv[0].x + hv[1].x) + (hv[2].x + hv[3].x);
      sum.y = (hv[0].y + hv[1].y) + (hv[2].y + hv[3].y);
      sum.z = (hv[0].z + hv[1].z) + (hv[2].z + hv[3].z);
      sum.w = (hv[0].w + hv[1].w) + (hv[2].w + hv[3].w);
      reinterpret_cast<uint4*>(fs.part)[j] = sum;
      mine += (sum.x + sum.y) + (sum.z + sum.w);
    }
    mine = __reduce_add_sync(0xffffffffu, mine);
    if (lane == 0) fs.wsum[warp] = mine;
    __syncthreads();
    if (warp == 0) {
      uint32_t v = lane < kWarps ? fs.wsum[lane] : 0u;
      v = __reduce_add_sync(0xffffffffu, v);
      if (lane == 0) fs.portion_total = v;
    }
  }
  __syncthreads();
  cluster_sync();
  if (warp == 0) {
    // lane q < C: portion q's total; portions in descending bin order, the
    // one holding the k-th largest key
    const uint32_t tq = static_cast<uint32_t>(lane) < static_cast<uint32_t>(C)
                            ? ld_dsmem_u32(dsmem_addr(&fs.portion_total, static_cast<uint32_t>(lane)))
                            : 0u;
    uint32_t above = tq;  // inclusive suffix sum over q' >= q
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t n2 = __shfl_down_sync(0xffffffffu, above, off);
      if (lane + off < 32) above += n2;
    }
    const uint32_t kk = static_cast<uint32_t>(a.k);
    const bool holds = lane < C && above - tq < kk && kk <= above;
    const uint32_t bal = __ballot_sync(0xffffffffu, holds);
    const int q = bal ? __ffs(bal) - 1 : 0;
    const uint32_t above_q = __shfl_sync(0xffffffffu, above - tq, q);
    if (lane == 0) {
      fs.pq = static_cast<uint32_t>(q);
      fs.krp = bal ? kk - above_q : 1u;
    }
  }
  __syncthreads();
  const uint32_t pq = fs.pq;
  for (int j = t; j < P / 4; j += kThreads)
    reinterpret_cast<uint4*>(sh.hist)[j] = ld_dsmem_v4(dsmem_addr(&reinterpret_cast<const uint4*>(fs.part)[j], pq));
  __syncthreads();
  select_digit(sh.hist, P, fs.krp, &sh.d, &sh.kr, sh.warp_tot);
  const uint32_t d1 = pq * static_cast<uint32_t>(P) + static_cast<uint32_t>(sh.d);
  const uint32_t kr1 = sh.kr;                   // rank of the k-th key inside bin d1
  const uint32_t n_cand_row = sh.hist[sh.d];    // keys in bin d1 (whole row)
  const uint32_t n_above = static_cast<uint32_t>(a.k) - kr1;
  // 3: each lane classifies its keys (groups of four consecutive keys)
  // against bin d1 -- above: key > the bin's top; candidate: key in the bin --
  // and keeps one byte of hit bits per group (above | candidate << 4) in
  // registers. One warp scan of the packed counts (above | cand << 16; a lane
  // sees at most kFusedSlice / kThreads keys) and a prefix over the warps and
  // the cluster's lower-ranked CTAs give every lane its first position in
  // both lists; the second sweep visits only the hit bits, in the same order.
  const uint32_t cand_lo = d1 << 20, cand_hi = cand_lo | 0xFFFFFu;
  constexpr int kGroups = kFusedSlice / (kThreads * 4);  // groups of four keys per lane
  constexpr int kWarpKeys = 128 * kUnroll;
  auto group_first = [&](int gi) {  // first key of the lane's group gi (slice-relative)
    return (gi / kUnroll) * (kThreads * 4 * kUnroll) + warp * kWarpKeys + (gi % kUnroll) * 128 + lane * 4;
  };
  uint32_t hits[kGroups / 4];
  uint32_t lcnt = 0;
#pragma unroll
  for (int gi = 0; gi < kGroups; ++gi) {
    const int j0 = group_first(gi);
    const uint4 kv = *reinterpret_cast<const uint4*>(&fs.keys[j0]);
    const int rem = n - j0;
    const uint32_t vmask = rem >= 4 ? 0xFu : (rem > 0 ? (1u << rem) - 1u : 0u);
    const uint32_t ma = ((kv.x > cand_hi ? 1u : 0u) | (kv.y > cand_hi ? 2u : 0u) | (kv.z > cand_hi ? 4u : 0u) |
                         (kv.w > cand_hi ? 8u : 0u)) & vmask;
    const uint32_t mc = (((kv.x - cand_lo) < 0x100000u ? 1u : 0u) | ((kv.y - cand_lo) < 0x100000u ? 2u : 0u) |
                         ((kv.z - cand_lo) < 0x100000u ? 4u : 0u) | ((kv.w - cand_lo) < 0x100000u ? 8u : 0u)) &
                        vmask;
    if (gi % 4 == 0) hits[gi / 4] = 0u;
    hits[gi / 4] |= (ma | (mc << 4)) << (8 * (gi % 4));
    lcnt += static_cast<uint32_t>(__popc(ma)) | (static_cast<uint32_t>(__popc(mc)) << 16);
  }
  uint32_t incl = lcnt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t m = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += m;
  }
  if (lane == 31) fs.wsum[warp] = incl;  // the warp's total
  __syncthreads();
  if (t == 0) {
    uint32_t run = 0;
    for (int w = 0; w < kWarps; ++w) {
      const uint32_t v = fs.wsum[w];
      fs.wsum[w] = run;  // exclusive prefix over this CTA's warps
      run += v;
    }
    fs.na = run & 0xffffu;
    fs.nc = run >> 16;
  }
  __syncthreads();
  cluster_sync();
  if (warp == 0) {
    // lane q < r: counts of the lower-ranked CTA q
    uint32_t ba = 0, bc = 0;
    if (static_cast<uint32_t>(lane) < r) {
      ba = ld_dsmem_u32(dsmem_addr(&fs.na, static_cast<uint32_t>(lane)));
      bc = ld_dsmem_u32(dsmem_addr(&fs.nc, static_cast<uint32_t>(lane)));
    }
    ba = __reduce_add_sync(0xffffffffu, ba);
    bc = __reduce_add_sync(0xffffffffu, bc);
    if (lane == 0) {
      sh.base_above = ba;
      sh.base_cand = bc;
    }
  }
  __syncthreads();
  {
    int32_t* out = a.idx + static_cast<int64_t>(b) * a.k;
    int32_t* cbuf = a.cand + static_cast<int64_t>(b) * a.cand_cap;
    uint32_t* ckbuf = a.cand_key + static_cast<int64_t>(b) * a.cand_cap;
    const uint32_t first = fs.wsum[warp] + incl - lcnt;  // this lane's first positions (packed)
    // This CTA's entries go to [base, base + count) of each list: staged in
    // shared memory, then copied out with consecutive stores (or stored
    // directly when a count exceeds the staging lists).
    const uint32_t na = fs.na, nc = fs.nc;
    const bool staged = na <= static_cast<uint32_t>(kLocalCap) && nc <= static_cast<uint32_t>(kLocalCap);
    uint32_t pa = first & 0xffffu, pc = first >> 16;  // positions within this CTA's ranges
#pragma unroll
    for (int gi = 0; gi < kGroups; ++gi) {
      const uint32_t h = (hits[gi / 4] >> (8 * (gi % 4))) & 0xFFu;
      if (h == 0u) continue;
      const int j0 = group_first(gi);
      uint32_t ma = h & 0xFu, mc = h >> 4;
      while (ma) {
        const int e = __ffs(ma) - 1;
        const int32_t pos = static_cast<int32_t>(lo + j0 + e);
        if (staged) {
          sh.above[pa] = pos;
        } else {
          const uint32_t gp = sh.base_above + pa;
          if (gp < n_above) out[gp] = pos;
          else record_status(a.status, IC_ERR_BAD_INDEX);  // cannot happen with consistent counts
        }
        ++pa;
        ma &= ma - 1u;
      }
      while (mc) {
        const int e = __ffs(mc) - 1;
        const int32_t pos = static_cast<int32_t>(lo + j0 + e);
        if (staged) {
          sh.cand[pc] = pos;
          sh.cand_key[pc] = fs.keys[j0 + e];
        } else {
          const uint32_t gp = sh.base_cand + pc;
          if (gp < static_cast<uint32_t>(a.cand_cap)) {
            cbuf[gp] = pos;
            ckbuf[gp] = fs.keys[j0 + e];
          }
        }
        ++pc;
        mc &= mc - 1u;
      }
    }
    if (staged) {
      __syncthreads();
      for (uint32_t j = t; j < na; j += kThreads) {
        const uint32_t gp = sh.base_above + j;
        if (gp < n_above) out[gp] = sh.above[j];
        else record_status(a.status, IC_ERR_BAD_INDEX);  // cannot happen with consistent counts
      }
      for (uint32_t j = t; j < nc; j += kThreads) {
        const uint32_t gp = sh.base_cand + j;
        if (gp < static_cast<uint32_t>(a.cand_cap)) {
          cbuf[gp] = sh.cand[j];
          ckbuf[gp] = sh.cand_key[j];
        }
      }
    }
  }
  // 4: every CTA's writes are visible to CTA 0, and no CTA reads another's
  // shared memory after this barrier
  __syncthreads();
  cluster_sync();
  if (r != 0) return;
  resolve_candidates(a, b, nv, d1, kr1, n_cand_row, sh);
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t stream, bool pdl, int* launches) {
  dim3 grid(a.cpr, a.B);
  cudaError_t e;
  if (a.fused) {
    static bool done_c[64] = {false};
    e = set_smem_once(topk_cluster_kernel, static_cast<int>(sizeof(FusedShared)), done_c);
    if (e != cudaSuccess) return e;
    e = launch_kernel_cluster(topk_cluster_kernel, grid, dim3(kThreads), sizeof(FusedShared), stream, pdl,
                              static_cast<unsigned>(a.cpr), a);
    if (e != cudaSuccess) return e;
    *launches += 1;
    return cudaGetLastError();
  }
  static bool done[64] = {false};  // one flag set per device
  e = set_smem_once(topk_filter_kernel, static_cast<int>(sizeof(FilterShared)), done);
  if (e != cudaSuccess) return e;
  // the filter pass overlaps the histogram pass's tail; the histogram pass
  // overlaps the previous kernel when the caller says one precedes it
  e = launch_kernel(topk_hist_kernel, grid, dim3(kThreads), 0, stream, pdl, a);
  if (e != cudaSuccess) return e;
  e = launch_kernel(topk_filter_kernel, grid, dim3(kThreads), sizeof(FilterShared), stream, true, a);
  if (e != cudaSuccess) return e;
  *launches += 2;
  return cudaGetLastError();
}

}  // namespace ic
