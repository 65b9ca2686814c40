// Top-k selection over indexer score rows (Hy4 IndexCache explainer, Jargon
// "Top-k selection": keep the k highest-scoring cached tokens).
//
// Radix select on the order-preserving 32-bit key of each fp32 score
// (negative floats: all bits flipped; others: sign bit set), in digits of
// 11, 11 and 10 bits, most significant first. Each row is split across
// `cpr` CTAs; every pass is its own launch, so no CTA ever waits on another:
//   pass 1  histogram of key[31:21] over the row's valid positions
//   pass 2  histogram of key[20:10] over keys whose top digit is the k-th's
//   pass 3  histogram of key[9:0]  over keys whose top 22 bits match
//   emit    keys > T (T = the exact k-th key) are compacted per CTA in
//           shared memory and written with one atomic reservation per CTA;
//           the last CTA of the row (atomic ticket) writes the r lowest-index
//           keys equal to T, so ties resolve toward the lower index and the
//           selected set is deterministic.
// After each histogram pass the last CTA of the row (atomic ticket) turns the
// row's global histogram into the chosen digit and the remaining rank, kept
// in a per-row state word that the next pass reads once.
// Rows with n_valid <= k take every valid index and pad with -1.
#include "common.cuh"
#include "kernels.h"

namespace ic {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kUnroll = 4;        // float4 loads in flight per lane
constexpr int kLocalCap = 4096;   // per-CTA shared buffer of selected indices

// per-row control block (kCtrlWords 32-bit words, one 128-byte line per row)
enum : int {
  kAboveCount = 0,  // emitted keys > T
  kTicket0 = 1,     // tickets of pass 1..3 and emit: kTicket0 + p
  kPrefix = 8,      // digits chosen so far (key bits above the current digit)
  kRank = 9,        // remaining rank within the keys matching the prefix
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

// Visit this CTA's slice of row b: f(i, key, valid) for every position, in
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

// Warp-aggregated shared-memory histogram increment; all 32 lanes call.
IC_DEV void hist_add(uint32_t* h, uint32_t bin, bool take) {
  if (__ballot_sync(0xffffffffu, take) == 0u) return;  // common in passes 2 and 3
  const uint32_t b = take ? bin : 0xFFFFFFFFu;
  const uint32_t peers = __match_any_sync(0xffffffffu, b);
  const int leader = __ffs(peers) - 1;
  if (take && (threadIdx.x & 31) == leader) atomicAdd(&h[bin], __popc(peers));
}

template <int PASS>
__global__ void __launch_bounds__(kThreads) topk_hist_kernel(const TopkArgs a) {
  __shared__ uint32_t sh_hist[kBins];
  __shared__ uint32_t warp_tot[kWarps];
  __shared__ int sh_d;
  __shared__ uint32_t sh_kr;
  __shared__ int sh_last;
  const int b = blockIdx.y, c = blockIdx.x;
  const int64_t nv = row_valid(a, b);
  if (nv <= a.k) return;  // the emit pass takes every valid index
  uint32_t* ctrl = row_ctrl(a, b);
  const int64_t lo = static_cast<int64_t>(c) * a.slice;
  const int64_t hi = lo + a.slice < nv ? lo + a.slice : nv;
  const uint32_t prefix = PASS > 1 ? __ldcg(&ctrl[kPrefix]) : 0u;
  const uint32_t kr = PASS > 1 ? __ldcg(&ctrl[kRank]) : static_cast<uint32_t>(a.k);
  for (int j = threadIdx.x; j < kBins; j += kThreads) sh_hist[j] = 0;
  __syncthreads();
  if (lo < hi) {
    for_slice(a, b, lo, hi, [&](int64_t, uint32_t key, bool valid) {
      if (PASS == 1) hist_add(sh_hist, key >> 21, valid);
      if (PASS == 2) hist_add(sh_hist, (key >> 10) & 0x7FFu, valid && (key >> 21) == prefix);
      if (PASS == 3) hist_add(sh_hist, key & 0x3FFu, valid && (key >> 10) == prefix);
    });
  }
  __syncthreads();
  uint32_t* g = a.hist + (static_cast<int64_t>(PASS - 1) * a.B + b) * kBins;
  for (int j = threadIdx.x; j < kBins; j += kThreads)
    if (sh_hist[j]) atomicAdd(g + j, sh_hist[j]);
  // last CTA of the row: choose this pass's digit once for everyone
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) sh_last = atomicAdd(&ctrl[kTicket0 + PASS - 1], 1u) == static_cast<uint32_t>(a.cpr) - 1;
  __syncthreads();
  if (!sh_last) return;
  __threadfence();
  const int nb = PASS == 3 ? 1024 : kBins;
  for (int j = threadIdx.x; j < nb; j += kThreads) sh_hist[j] = __ldcg(g + j);
  __syncthreads();
  select_digit(sh_hist, nb, kr, &sh_d, &sh_kr, warp_tot);
  if (threadIdx.x == 0) {
    const int shift = PASS == 3 ? 10 : 11;
    ctrl[kPrefix] = (prefix << shift) | static_cast<uint32_t>(sh_d);
    ctrl[kRank] = sh_kr;
  }
}

__global__ void __launch_bounds__(kThreads) topk_emit_kernel(const TopkArgs a) {
  __shared__ int32_t sh_sel[kLocalCap];
  __shared__ uint32_t sh_n;
  __shared__ uint32_t sh_base;
  __shared__ uint32_t warp_cnt[kWarps];
  __shared__ int sh_last;
  const int b = blockIdx.y, c = blockIdx.x;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  int32_t* out = a.idx + static_cast<int64_t>(b) * a.k;
  const int64_t nv = row_valid(a, b);
  if (nv <= a.k) {
    if (c == 0)
      for (int i = t; i < a.k; i += kThreads) out[i] = i < nv ? i : -1;
    return;
  }
  uint32_t* ctrl = row_ctrl(a, b);
  const uint32_t T = __ldcg(&ctrl[kPrefix]);  // the exact k-th key
  const uint32_t r = __ldcg(&ctrl[kRank]);    // keys equal to T to take, >= 1
  const uint32_t n_above = static_cast<uint32_t>(a.k) - r;
  if (t == 0) sh_n = 0;
  __syncthreads();

  const int64_t lo = static_cast<int64_t>(c) * a.slice;
  const int64_t hi = lo + a.slice < nv ? lo + a.slice : nv;
  uint32_t my_ties = 0;
  if (lo < hi) {
    for_slice(a, b, lo, hi, [&](int64_t i, uint32_t key, bool valid) {
      const bool above = valid && key > T;
      const uint32_t bal = __ballot_sync(0xffffffffu, above);
      if (bal) {
        uint32_t base = 0;
        if (lane == 0) base = atomicAdd(&sh_n, static_cast<uint32_t>(__popc(bal)));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (above) {
          const uint32_t pos = base + __popc(bal & ((1u << lane) - 1u));
          if (pos < kLocalCap) {
            sh_sel[pos] = static_cast<int32_t>(i);
          } else {  // shared buffer full: reserve globally, one at a time
            const uint32_t gp = atomicAdd(&ctrl[kAboveCount], 1u);
            if (gp < n_above) out[gp] = static_cast<int32_t>(i);
            else record_status(a.status, IC_ERR_BAD_INDEX);
          }
        }
      }
      if (valid && key == T) ++my_ties;
    });
  }
  __syncthreads();
  const uint32_t n_local = sh_n < kLocalCap ? sh_n : kLocalCap;
  if (t == 0) sh_base = n_local ? atomicAdd(&ctrl[kAboveCount], n_local) : 0u;
  __syncthreads();
  for (uint32_t j = t; j < n_local; j += kThreads) {
    const uint32_t gp = sh_base + j;
    if (gp < n_above) out[gp] = sh_sel[j];
    else record_status(a.status, IC_ERR_BAD_INDEX);  // cannot happen with consistent histograms
  }
  // CTA total of ties
#pragma unroll
  for (int off = 16; off; off >>= 1) my_ties += __shfl_down_sync(0xffffffffu, my_ties, off);
  if (lane == 0) warp_cnt[warp] = my_ties;
  __syncthreads();
  if (t == 0) {
    uint32_t tot = 0;
    for (int w = 0; w < kWarps; ++w) tot += warp_cnt[w];
    a.tie_counts[static_cast<int64_t>(b) * a.cpr + c] = tot;
    __threadfence();
    sh_last = atomicAdd(&ctrl[kTicket0 + 3], 1u) == static_cast<uint32_t>(a.cpr) - 1;
  }
  __syncthreads();
  if (!sh_last) return;
  __threadfence();

  // Last CTA of the row: the r lowest-index ties, slice by slice in order.
  uint32_t taken = 0;
  const float* row = a.scores + static_cast<int64_t>(b) * a.N;
  for (int j = 0; j < a.cpr && taken < r; ++j) {
    const uint32_t cnt = __ldcg(&a.tie_counts[static_cast<int64_t>(b) * a.cpr + j]);
    if (cnt == 0) continue;
    const int64_t slo = static_cast<int64_t>(j) * a.slice;
    const int64_t shi = slo + a.slice < nv ? slo + a.slice : nv;
    for (int64_t base = slo; base < shi && taken < r; base += kThreads) {
      const int64_t i = base + t;
      const bool tie = (i < shi) && score_key(__ldcg(row + i)) == T;
      const uint32_t bal = __ballot_sync(0xffffffffu, tie);
      if (lane == 0) warp_cnt[warp] = __popc(bal);
      __syncthreads();
      uint32_t before = 0;
      for (int w = 0; w < warp; ++w) before += warp_cnt[w];
      uint32_t total = 0;
      for (int w = 0; w < kWarps; ++w) total += warp_cnt[w];
      const uint32_t pos = taken + before + __popc(bal & ((1u << lane) - 1u));
      if (tie && pos < r) out[n_above + pos] = static_cast<int32_t>(i);
      taken += total;
      __syncthreads();
    }
  }
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t stream, int* launches) {
  dim3 grid(a.cpr, a.B);
  topk_hist_kernel<1><<<grid, kThreads, 0, stream>>>(a);
  topk_hist_kernel<2><<<grid, kThreads, 0, stream>>>(a);
  topk_hist_kernel<3><<<grid, kThreads, 0, stream>>>(a);
  topk_emit_kernel<<<grid, kThreads, 0, stream>>>(a);
  *launches += 4;
  return cudaGetLastError();
}

}  // namespace ic
