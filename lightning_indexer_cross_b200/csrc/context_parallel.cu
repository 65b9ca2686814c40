// Context-parallel decode over G ranks, each holding a contiguous shard of the
// N cached tokens (Hy4 IndexCache explainer, TL;DR and Jargon "Sparse
// attention": the 1M-token context is what the indexer has to score; the
// shard split keeps each rank's share of that pass local).
//
// Per F layer, rank r scores its shard and keeps its local top-k; the union
// of the ranks' local top-k sets holds the global top-k (every token of the
// global top-k is among the k best of its own shard), so after one exchange
// of (score, global index) candidates every rank selects the same global
// top-k. Attention then runs per rank over the selected rows it owns, without
// the sink; the ranks' partial outputs (o_r, lse_r) merge exactly as
//   out = sum_r e^{lse_r} o_r / (e^{sink} + sum_r e^{lse_r}),
// with the sink added once, then the gate.
//
// Kernels here (the exchanges themselves are NCCL collectives issued by the
// caller):
//   cp_candidates_kernel  (score, global index) of each local top-k entry
//   cp_merge_topk_kernel  the k best of the gathered candidates of a row,
//                         ties toward the lower global index; also the
//                         row's indices local to this rank's shard
//   cp_combine_kernel     merge of the ranks' partial attention outputs
#include "common.cuh"
#include "kernels.h"

namespace ic {

namespace {

constexpr int kMergeThreads = 512;

__global__ void __launch_bounds__(256) cp_candidates_kernel(const CpCandArgs a) {
  pdl_trigger();
  pdl_wait();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(a.B) * a.k) return;
  const int64_t b = i / a.k;
  const int32_t x = a.idx[i];
  float s = -INFINITY;
  int32_t g = -1;
  if (x >= 0 && x < a.N_local) {
    s = a.scores[b * a.N_local + x];
    g = static_cast<int32_t>(x + a.offset);
  } else if (x != -1) {
    record_status(a.status, IC_ERR_BAD_INDEX);
  }
  a.cand_score[i] = s;
  a.cand_idx[i] = g;
}

// Composite 64-bit key of a candidate: the order-preserving key of its score
// above, the complement of its global index below, so that "larger key" means
// a higher score, then a lower index; padding (index -1) ranks last among
// equal scores.
IC_DEV uint64_t cand_key(float s, int32_t g) {
  const uint32_t u = __float_as_uint(s);
  const uint32_t hi = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  const uint32_t lo = ~static_cast<uint32_t>(g);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// One CTA per row: the k largest composite keys of the row's n candidates
// (n <= kCpMaxCand, held in shared memory), found by an MSB-first radix
// select with 8-bit digits; it stops as soon as the digit holding the k-th
// key is taken whole.
__global__ void __launch_bounds__(kMergeThreads) cp_merge_topk_kernel(const CpMergeArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem_raw);
  __shared__ uint32_t hist[256];
  __shared__ int sel_digit;
  __shared__ uint32_t sel_rank, sel_count;
  __shared__ uint32_t n_out, n_eq;
  const int b = blockIdx.x, t = threadIdx.x;
  pdl_trigger();
  pdl_wait();
  const int n = a.G * a.kin;
  for (int i = t; i < n; i += kMergeThreads) {
    const int64_t off = (i / a.kin) * a.seg_stride + static_cast<int64_t>(b) * a.kin + i % a.kin;
    keys[i] = cand_key(a.cand_score[off], a.cand_idx[off]);
  }
  if (t == 0) {
    n_out = 0;
    n_eq = 0;
  }
  __syncthreads();
  int32_t* og = a.idx_global + static_cast<int64_t>(b) * a.k;
  int32_t* ol = a.idx_local + static_cast<int64_t>(b) * a.k;
  auto emit = [&](uint64_t key, uint32_t pos) {
    if (pos >= static_cast<uint32_t>(a.k)) return;  // cannot happen with consistent counts
    const int32_t g = static_cast<int32_t>(~static_cast<uint32_t>(key & 0xffffffffull));
    og[pos] = g;
    if (ol) ol[pos] = (g >= 0 && g >= a.lo && g < a.hi) ? static_cast<int32_t>(g - a.lo) : -1;
  };
  if (n <= a.k) {
    // every candidate is selected; the rest of the row is padding
    for (int i = t; i < a.k; i += kMergeThreads) {
      if (i < n) emit(keys[i], static_cast<uint32_t>(i));
      else {
        og[i] = -1;
        if (ol) ol[i] = -1;
      }
    }
    return;
  }
  // prefix: the selected keys are those whose top (64 - shift) bits exceed
  // `prefix`, plus `kr` of those equal to it
  uint64_t prefix = 0;
  int shift = 64;
  uint32_t kr = static_cast<uint32_t>(a.k);
  bool whole = false;
  while (shift > 0) {
    const int s2 = shift - 8;
    for (int i = t; i < 256; i += kMergeThreads) hist[i] = 0;
    __syncthreads();
    for (int i = t; i < n; i += kMergeThreads) {
      const uint64_t x = keys[i];
      if (shift == 64 || (x >> shift) == prefix) atomicAdd(&hist[(x >> s2) & 0xffu], 1u);
    }
    __syncthreads();
    if (t < 32) {
      // digits in descending order: lane l sums digits 255 - 8l .. 248 - 8l
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = hist[255 - 8 * t - e];
        sum += c[e];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (t >= off) incl += v;
      }
      uint32_t above = incl - sum;  // keys in higher digits than this lane's
      if (above < kr && kr <= incl) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (above < kr && kr <= above + c[e]) {
            sel_digit = 255 - 8 * t - e;
            sel_rank = kr - above;
            sel_count = c[e];
          }
          above += c[e];
        }
      }
    }
    __syncthreads();
    prefix = (shift == 64 ? 0ull : (prefix << 8)) | static_cast<uint64_t>(sel_digit);
    shift = s2;
    kr = sel_rank;
    if (sel_count == kr) {
      whole = true;
      break;
    }
    __syncthreads();
  }
  // keys above the prefix, then `kr` keys equal to it (all of them when the
  // digit was taken whole; equal full keys are identical candidates)
  const uint32_t n_above = static_cast<uint32_t>(a.k) - kr;
  for (int i = t; i < n; i += kMergeThreads) {
    const uint64_t x = keys[i];
    const uint64_t top = shift == 64 ? 0ull : (x >> shift);
    if (top > prefix) {
      emit(x, atomicAdd(&n_out, 1u));
    } else if (top == prefix) {
      const uint32_t e = atomicAdd(&n_eq, 1u);
      if (whole || e < kr) emit(x, n_above + e);
    }
  }
}

// One warp per (query, head) row: out = gate * sum_r e^{lse_r - M} o_r /
// (e^{sink - M} + sum_r e^{lse_r - M}), M the largest of sink and the lse_r.
__global__ void __launch_bounds__(256) cp_combine_kernel(const CpCombineArgs a) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  const int64_t rows = static_cast<int64_t>(a.B) * a.H;
  if (row >= rows) return;
  const int h = static_cast<int>(row % a.H);
  const float sink = a.sink[h];
  float M = sink;
  for (int r = 0; r < a.G; ++r) M = fmaxf(M, a.part_lse[r * a.lse_stride + row]);
  float den = (M == -INFINITY) ? 0.f : expf(sink - M);
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
  for (int r = 0; r < a.G; ++r) {
    const float l = a.part_lse[r * a.lse_stride + row];
    if (l == -INFINITY) continue;  // no selected row on that rank
    const float wgt = expf(l - M);
    den += wgt;
    const float* o = a.part_out + r * a.out_stride + row * 512;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float4 v = *reinterpret_cast<const float4*>(o + c * 128 + lane * 4);
      acc[4 * c + 0] = fmaf(wgt, v.x, acc[4 * c + 0]);
      acc[4 * c + 1] = fmaf(wgt, v.y, acc[4 * c + 1]);
      acc[4 * c + 2] = fmaf(wgt, v.z, acc[4 * c + 2]);
      acc[4 * c + 3] = fmaf(wgt, v.w, acc[4 * c + 3]);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int64_t d0 = row * 512 + c * 128 + lane * 4;
    float o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      o[e] = acc[4 * c + e] * inv;
      if (a.gate) o[e] *= 1.f / (1.f + __expf(-__bfloat162float(a.gate[d0 + e])));
    }
    if (a.out_f32) {
      *reinterpret_cast<float4*>(static_cast<float*>(a.out) + d0) = make_float4(o[0], o[1], o[2], o[3]);
    } else {
      uint2 pk;
      pk.x = pack_bf16x2(o[0], o[1]);
      pk.y = pack_bf16x2(o[2], o[3]);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + d0) = pk;
    }
  }
  if (a.lse && lane == 0) a.lse[row] = (den > 0.f) ? M + logf(den) : -INFINITY;
}

}  // namespace

cudaError_t launch_cp_candidates(const CpCandArgs& a, cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(a.B) * a.k;
  const dim3 grid(static_cast<unsigned>((n + 255) / 256));
  cudaError_t e = launch_kernel(cp_candidates_kernel, grid, dim3(256), 0, stream, false, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_cp_merge_topk(const CpMergeArgs& a, cudaStream_t stream) {
  static bool done[64] = {false};
  const int bytes = kCpMaxCand * 8;
  cudaError_t e = set_smem_once(cp_merge_topk_kernel, bytes, done);
  if (e != cudaSuccess) return e;
  e = launch_kernel(cp_merge_topk_kernel, dim3(a.B), dim3(kMergeThreads), static_cast<size_t>(a.G) * a.kin * 8,
                    stream, false, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_cp_combine(const CpCombineArgs& a, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(a.B) * a.H;
  const dim3 grid(static_cast<unsigned>((rows + 7) / 8));
  cudaError_t e = launch_kernel(cp_combine_kernel, grid, dim3(256), 0, stream, false, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace ic
