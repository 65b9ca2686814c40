// Top-k selection over indexer score rows (Hy4 IndexCache explainer, Jargon
// "Top-k selection": keep the k highest-scoring cached tokens), in one pass
// over the scores.
//
//   sample   one CTA per row reads a sample spread over the row (all of it
//            when the row has at most 2 x kSample scores) and takes a
//            threshold T at which about kAlpha * k of the row's keys are
//            expected: the lower edge of the 22-bit key bin holding the
//            (kAlpha * k * m / n)-th largest of the m sampled keys (exactly
//            the k-th largest when the whole row was read).
//   filter   the row's CTAs scan their slices once and append every position
//            whose key is >= T to the row's candidate buffer (staged per CTA
//            in shared memory, one reservation per CTA). The last CTA of the
//            row (atomic ticket) selects the k best candidates by radix
//            select on (key, position) composites -- ties toward the lower
//            position -- and leaves the row's control words zero.
// Exactness does not depend on the sample. If at least k keys are >= T, the
// k-th largest key is >= T and every key of the top-k is a candidate. If
// fewer than k are, or more than the buffer holds, the last CTA selects over
// the whole row itself (slower, same result).
// Keys are the order-preserving 32-bit images of the fp32 scores. Rows with
// n_valid <= k take every valid index and pad with -1.
#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace ic {

namespace {

constexpr int kT = 512;
constexpr int kSample = 8192;       // sampled keys per row (the whole row up to 2 x this)
constexpr float kAlpha = 2.f;       // candidates expected per row, in units of k
constexpr int kLocalCap = 4096;     // candidates one filter CTA stages in shared memory
constexpr int kSmemCand = 6144;     // candidates the last CTA selects in shared memory (2k expected, 1.5 x margin)
constexpr int kUnroll = 4;          // float4 loads in flight per thread in the scan

// per-row control words (kCtrlWords 32-bit words, one 128-byte line per row)
enum : int { kCount = 0, kTicket = 1, kThresh = 2 };

IC_DEV int64_t row_valid(const TopkArgs& a, int b) {
  const int64_t nv = a.n_valid ? a.n_valid[b] : a.N;
  return nv < 0 ? 0 : (nv > a.N ? a.N : nv);
}

// Rows with n_valid <= k: every valid index, padded with -1 (CTA 0 of the row).
IC_DEV void small_row(const TopkArgs& a, int b, int64_t nv) {
  int32_t* out = a.idx + static_cast<int64_t>(b) * a.k;
  for (int i = threadIdx.x; i < a.k; i += kT) out[i] = i < nv ? i : -1;
}

struct SampleShared {
  uint32_t hist[4096];
  uint32_t warp_tot[kT / 32];
  int d;
  uint32_t kr;
  uint32_t keys[2 * kSample];
};

__global__ void __launch_bounds__(kT) topk_sample_kernel(const TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SampleShared& sh = *reinterpret_cast<SampleShared*>(smem_raw);
  const int b = blockIdx.x, t = threadIdx.x;
  pdl_trigger();
  pdl_wait();
  const int64_t nv = row_valid(a, b);
  if (nv <= a.k) return;
  const float* row = a.scores + static_cast<int64_t>(b) * a.N;
  // the sample: the whole row, or nb blocks of 32 consecutive scores spread
  // evenly over it
  int m;
  uint32_t s;  // rank of the threshold key inside the sample
  if (nv <= 2 * kSample) {
    m = static_cast<int>(nv);
    for (int i = t; i < m; i += kT) sh.keys[i] = order_key(__ldcg(row + i));
    s = static_cast<uint32_t>(a.k);
  } else {
    // block j: one of the whole 32-score blocks of stretch j of the row,
    // picked by a multiplicative hash of j (so the sample does not line up
    // with regularly spaced positions of the row)
    constexpr int nb = kSample / 32;
    m = kSample;
    const int64_t blocks = nv / 32;  // whole 32-score blocks inside the row
    for (int i = t; i < m; i += kT) {
      const int j = i >> 5;
      const int64_t b0 = static_cast<int64_t>(j) * blocks / nb, b1 = static_cast<int64_t>(j + 1) * blocks / nb;
      const uint32_t h = (static_cast<uint32_t>(j) + 1u) * 2654435761u;
      const int64_t start = (b0 + static_cast<int64_t>(h >> 8) % (b1 - b0)) * 32;
      sh.keys[i] = order_key(__ldcg(row + start + (i & 31)));
    }
    const double want = static_cast<double>(kAlpha) * a.k * m / static_cast<double>(nv);
    s = static_cast<uint32_t>(want < 1.0 ? 1.0 : (want > m ? m : want));
  }
  // the s-th largest sampled key's 22-bit bin: digit 1 = key[31:20], then
  // digit 2 = key[19:10] among the keys of that bin
  for (int i = t; i < 4096; i += kT) sh.hist[i] = 0;
  __syncthreads();
  for (int i = t; i < m; i += kT) atomicAdd(&sh.hist[sh.keys[i] >> 20], 1u);
  __syncthreads();
  find_digit<kT>(sh.hist, 4096, s, &sh.d, &sh.kr, sh.warp_tot);
  const uint32_t d1 = static_cast<uint32_t>(sh.d), kr1 = sh.kr;
  __syncthreads();
  for (int i = t; i < 1024; i += kT) sh.hist[i] = 0;
  __syncthreads();
  for (int i = t; i < m; i += kT) {
    const uint32_t x = sh.keys[i];
    if ((x >> 20) == d1) atomicAdd(&sh.hist[(x >> 10) & 0x3FFu], 1u);
  }
  __syncthreads();
  find_digit<kT>(sh.hist, 1024, kr1, &sh.d, &sh.kr, sh.warp_tot);
  if (t == 0)
    a.counters[static_cast<int64_t>(b) * kCtrlWords + kThresh] = (d1 << 20) | (static_cast<uint32_t>(sh.d) << 10);
}

// The staging lists are written out before the row's last CTA selects, so
// its candidate array reuses their space (50 KB a CTA).
struct FilterShared {
  union {
    struct {
      int32_t pos[kLocalCap];
      uint32_t key[kLocalCap];
    };
    uint64_t cand[kSmemCand];
  };
  uint32_t n_local, base;
  int last;
  SelectShared sel;
};
static_assert(kSmemCand * 8 >= kLocalCap * 8, "the candidate array covers the staging lists");

__global__ void __launch_bounds__(kT) topk_filter_kernel(const TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  FilterShared& sh = *reinterpret_cast<FilterShared*>(smem_raw);
  const int b = blockIdx.y, c = blockIdx.x;
  const int t = threadIdx.x, lane = t & 31;
  pdl_trigger();
  pdl_wait();
  const int64_t nv = row_valid(a, b);
  if (nv <= a.k) {
    if (c == 0) small_row(a, b, nv);
    return;
  }
  uint32_t* ctrl = a.counters + static_cast<int64_t>(b) * kCtrlWords;
  const uint32_t T = __ldcg(&ctrl[kThresh]);
  // the fp32 value whose order key is T (every finite value when T lies at
  // or below the key of -inf)
  const float tf = T <= 0x007FFFFFu ? -INFINITY : __uint_as_float((T & 0x80000000u) ? (T & 0x7FFFFFFFu) : ~T);
  int32_t* cbuf = a.cand + static_cast<int64_t>(b) * a.cand_cap;
  uint32_t* ckbuf = a.cand_key + static_cast<int64_t>(b) * a.cand_cap;
  if (t == 0) sh.n_local = 0;
  __syncthreads();
  // positions whose key is >= T: staged in shared memory (warp-aggregated);
  // past the staging capacity, appended straight to the row's buffer
  auto push = [&](int64_t i, uint32_t key, bool take) {
    const uint32_t bal = __ballot_sync(0xffffffffu, take);
    if (!bal) return;
    uint32_t base = 0;
    if (lane == 0) base = atomicAdd(&sh.n_local, static_cast<uint32_t>(__popc(bal)));
    base = __shfl_sync(0xffffffffu, base, 0);
    const uint32_t p = base + __popc(bal & ((1u << lane) - 1u));
    if (take) {
      if (p < static_cast<uint32_t>(kLocalCap)) {
        sh.pos[p] = static_cast<int32_t>(i);
        sh.key[p] = key;
      }
    }
    if (base + __popc(bal) > static_cast<uint32_t>(kLocalCap)) {
      // overflow of the staging lists: reserve in the row's buffer directly
      const bool over = take && p >= static_cast<uint32_t>(kLocalCap);
      const uint32_t ob = __ballot_sync(0xffffffffu, over);
      uint32_t gb = 0;
      if (lane == 0 && ob) gb = atomicAdd(&ctrl[kCount], static_cast<uint32_t>(__popc(ob)));
      gb = __shfl_sync(0xffffffffu, gb, 0);
      if (over) {
        const uint32_t gp = gb + __popc(ob & ((1u << lane) - 1u));
        if (gp < static_cast<uint32_t>(a.cand_cap)) {
          cbuf[gp] = static_cast<int32_t>(i);
          ckbuf[gp] = key;
        }
      }
    }
  };
  // The same for the candidates among a lane's four consecutive keys
  // (mask m): the warp's inclusive scan of the counts gives every lane its
  // first slot after one reservation by the last lane.
  auto push4 = [&](int64_t i, uint32_t m, const float4& x) {
    const uint32_t cnt = static_cast<uint32_t>(__popc(m));
    uint32_t incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    uint32_t base = 0;
    if (lane == 31) base = atomicAdd(&sh.n_local, incl);
    base = __shfl_sync(0xffffffffu, base, 31);
    uint32_t p = base + incl - cnt;
    const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if ((m >> e) & 1u) {
        const uint32_t key = order_key(xs[e]);
        if (p < static_cast<uint32_t>(kLocalCap)) {
          sh.pos[p] = static_cast<int32_t>(i + e);
          sh.key[p] = key;
        } else {
          // past the staging capacity: straight to the row's buffer
          const uint32_t gp = atomicAdd(&ctrl[kCount], 1u);
          if (gp < static_cast<uint32_t>(a.cand_cap)) {
            cbuf[gp] = static_cast<int32_t>(i + e);
            ckbuf[gp] = key;
          }
        }
        ++p;
      }
    }
  };
  const int64_t lo = static_cast<int64_t>(c) * a.slice;
  const int64_t hi = lo + a.slice < nv ? lo + a.slice : nv;
  const float* row = a.scores + static_cast<int64_t>(b) * a.N;
  if (lo < hi) {
    if (((a.N & 3) == 0) && ((lo & 3) == 0)) {
      const int warp = t >> 5;
      constexpr int kWarpSpan = kUnroll * 128;
      for (int64_t base = lo + static_cast<int64_t>(warp) * kWarpSpan; base < hi; base += kT * 4 * kUnroll) {
        float4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int64_t i = base + u * 128 + lane * 4;
          if (i + 3 < hi) {
            v[u] = __ldcg(reinterpret_cast<const float4*>(row + i));
          } else {
            v[u] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            if (i < hi) v[u].x = __ldcg(row + i);
            if (i + 1 < hi) v[u].y = __ldcg(row + i + 1);
            if (i + 2 < hi) v[u].z = __ldcg(row + i + 2);
          }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int64_t i = base + u * 128 + lane * 4;
          // x >= tf picks every key >= T (plus -0.0 when tf is +0.0: an extra
          // candidate, harmless to the exact selection); keys are formed
          // only for the candidates
          const bool h0 = i < hi && v[u].x >= tf, h1 = i + 1 < hi && v[u].y >= tf, h2 = i + 2 < hi && v[u].z >= tf,
                     h3 = i + 3 < hi && v[u].w >= tf;
          // a group of 128 keys with no candidate is skipped on one vote;
          // otherwise one warp scan of the lanes' counts and one shared
          // reservation place the group's candidates
          const uint32_t m = (h0 ? 1u : 0u) | (h1 ? 2u : 0u) | (h2 ? 4u : 0u) | (h3 ? 8u : 0u);
          if (__ballot_sync(0xffffffffu, m != 0u) == 0u) continue;
          push4(i, m, v[u]);
        }
      }
    } else {
      for (int64_t base = lo; base < hi; base += kT) {
        const int64_t i = base + t;
        const float x = i < hi ? __ldcg(row + i) : -INFINITY;
        const uint32_t key = order_key(x);
        push(i, key, i < hi && key >= T);
      }
    }
  }
  __syncthreads();
  // one reservation for this CTA's staged candidates, then consecutive stores
  const uint32_t nl = sh.n_local < static_cast<uint32_t>(kLocalCap) ? sh.n_local : kLocalCap;
  if (t == 0) sh.base = nl ? atomicAdd(&ctrl[kCount], nl) : 0u;
  __syncthreads();
  for (uint32_t j = t; j < nl; j += kT) {
    const uint32_t gp = sh.base + j;
    if (gp < static_cast<uint32_t>(a.cand_cap)) {
      cbuf[gp] = sh.pos[j];
      ckbuf[gp] = sh.key[j];
    }
  }
  // the last CTA of the row selects
  __threadfence();
  __syncthreads();
  if (t == 0) sh.last = atomicAdd(&ctrl[kTicket], 1u) == static_cast<uint32_t>(a.cpr) - 1;
  __syncthreads();
  if (!sh.last) return;
  __threadfence();
  const uint32_t n = __ldcg(&ctrl[kCount]);
  int32_t* out = a.idx + static_cast<int64_t>(b) * a.k;
  auto emit = [&](uint64_t key, uint32_t p) { out[p] = composite_pos(key); };
  const uint32_t k = static_cast<uint32_t>(a.k);
  if (n >= k && n <= static_cast<uint32_t>(kSmemCand) && n <= static_cast<uint32_t>(a.cand_cap)) {
    for (uint32_t j = t; j < n; j += kT) sh.cand[j] = composite_key(__ldcg(ckbuf + j), __ldcg(cbuf + j));
    __syncthreads();
    select_k_largest<kT>(sh.sel, n, k, [&](int64_t i) { return sh.cand[i]; }, emit);
  } else if (n >= k && n <= static_cast<uint32_t>(a.cand_cap)) {
    select_k_largest<kT>(sh.sel, n, k,
                         [&](int64_t i) { return composite_key(__ldcg(ckbuf + i), __ldcg(cbuf + i)); }, emit);
  } else {
    // the threshold missed (fewer than k keys above it, or more than the
    // buffer holds): select over the whole row
    select_k_largest<kT>(sh.sel, nv, k,
                         [&](int64_t i) { return composite_key(order_key(__ldcg(row + i)), static_cast<int32_t>(i)); },
                         emit);
  }
  // every CTA of the row is done with the control words: leave them zero
  if (t < kCtrlWords) ctrl[t] = 0u;
}

}  // namespace

int topk_threshold_smem_bytes() { return static_cast<int>(sizeof(FilterShared)); }

cudaError_t launch_topk_threshold(const TopkArgs& a, cudaStream_t stream, bool pdl, int* launches) {
  static bool done_s[64] = {false}, done_f[64] = {false};
  cudaError_t e = set_smem_once(topk_sample_kernel, static_cast<int>(sizeof(SampleShared)), done_s);
  if (e != cudaSuccess) return e;
  e = set_smem_once(topk_filter_kernel, static_cast<int>(sizeof(FilterShared)), done_f);
  if (e != cudaSuccess) return e;
  e = launch_kernel(topk_sample_kernel, dim3(a.B), dim3(kT), sizeof(SampleShared), stream, pdl, a);
  if (e != cudaSuccess) return e;
  e = launch_kernel(topk_filter_kernel, dim3(a.cpr, a.B), dim3(kT), sizeof(FilterShared), stream, true, a);
  if (e != cudaSuccess) return e;
  *launches += 2;
  return cudaGetLastError();
}

}  // namespace ic
