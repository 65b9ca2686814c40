// Cache-append step on sm_100a: the new tokens' indexer keys and latent rows
// are written into the caches, and the queries' rotary dims are rotated.
//
//   key row  = LayerNorm-with-bias(k_raw)  (Hy4-preview porting issue,
//              "Indexer" bullet), stored as bf16, or as e4m3 codes with one
//              fp32 scale per token (max|y| / 448, round to nearest even,
//              saturating);
//   kv row   = kv_raw with its 64 rotary dims [512, 576) rotated pairwise,
//              adjacent pairs (2i, 2i+1) ("RoPE is interleaved" bullet,
//              is_neox_style=False), angle = position * base^(-2i/64);
//   q        = the same rotation of each head's rotary dims, in place.
//
// The step moves about 2.8 KB per token: it is bound by launch latency at
// decode sizes and by HBM for long prefill chunks, never by arithmetic, so
// one plain kernel does all of it. CTA t < T appends token t (warp 0 the key,
// warps 1-2 copy the 512 latent dims as 16-byte words, warp 3 rotates the 32
// rotary pairs); CTA T + b rotates query b's heads. Angles are formed and
// their sine and cosine taken in double: at positions near 10^6 a float
// angle would be off by ~0.06 rad.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace ic {

namespace {

constexpr int kRowD = 576;
constexpr int kLatent = 512;
constexpr int kPairs = (kRowD - kLatent) / 2;  // 32 rotary pairs
constexpr int kThreads = 128;

// cos / sin of position * base^(-2i/64) for rotary pair i
IC_DEV void rope_angle(int64_t position, int i, double log2_base, double* c, double* s) {
  const double theta = exp2(-(2.0 * i / (2.0 * kPairs)) * log2_base);
  sincos(static_cast<double>(position) * theta, s, c);
}

// rotate one (x[2i], x[2i+1]) bf16 pair held as a 32-bit word
IC_DEV uint32_t rotate_pair(uint32_t w, double c, double s) {
  const double a = bf16_lane(w, 0), b = bf16_lane(w, 1);
  const __nv_bfloat16 lo = __double2bfloat16(a * c - b * s);
  const __nv_bfloat16 hi = __double2bfloat16(a * s + b * c);
  return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) | (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}

template <int D_I>
__global__ void __launch_bounds__(kThreads) cache_append_kernel(const AppendArgs a) {
  constexpr int kPer = D_I / 32;  // key elements per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  if (t < a.T) {
    const int64_t r = a.pos[t];
    if (r < 0 || r >= a.N) {  // not a row of the cache: nothing is written
      if (threadIdx.x == 0) record_status(a.status, IC_ERR_BAD_INDEX);
      return;
    }
    const int64_t c = t;  // destination cache when the batch strides are nonzero
    if (warp == 0) {
      // LayerNorm with bias over the d_I dims of this token's key
      float x[kPer];
      const __nv_bfloat16* src = a.k_raw + static_cast<int64_t>(t) * D_I + lane * kPer;
#pragma unroll
      for (int e = 0; e < kPer; ++e) x[e] = __bfloat162float(src[e]);
      float sum = 0.f;
#pragma unroll
      for (int e = 0; e < kPer; ++e) sum += x[e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      const float mean = sum / D_I;
      float sq = 0.f;
#pragma unroll
      for (int e = 0; e < kPer; ++e) sq = fmaf(x[e] - mean, x[e] - mean, sq);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      const float inv = 1.f / sqrtf(sq / D_I + a.eps);
      float y[kPer];
#pragma unroll
      for (int e = 0; e < kPer; ++e) y[e] = fmaf((x[e] - mean) * inv, a.gamma[lane * kPer + e], a.beta[lane * kPer + e]);
      if (!a.fp8) {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.key_cache) + c * a.k_bs + r * D_I + lane * kPer;
#pragma unroll
        for (int e = 0; e < kPer; ++e) dst[e] = __float2bfloat16_rn(y[e]);
      } else {
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < kPer; ++e) amax = fmaxf(amax, fabsf(y[e]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float scale = amax > 0.f ? amax / 448.f : 1.f;
        uint8_t* dst = static_cast<uint8_t*>(a.key_cache) + c * a.k_bs + r * D_I + lane * kPer;
#pragma unroll
        for (int e = 0; e < kPer; ++e)
          dst[e] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(y[e] / scale, __NV_SATFINITE, __NV_E4M3));
        if (lane == 0) a.key_scale[c * a.s_bs + r] = scale;
      }
    } else if (warp < 3) {
      // latent dims: 64 words of 16 bytes
      const int wd = threadIdx.x - 32;  // 0..63
      const uint4* src = reinterpret_cast<const uint4*>(a.kv_raw + static_cast<int64_t>(t) * kRowD);
      uint4* dst = reinterpret_cast<uint4*>(a.kv_cache + c * a.kv_bs + r * kRowD);
      dst[wd] = src[wd];
    } else {
      // rotary dims: pair `lane`
      double cs, sn;
      rope_angle(r, lane, a.log2_base, &cs, &sn);
      const uint32_t* src = reinterpret_cast<const uint32_t*>(a.kv_raw + static_cast<int64_t>(t) * kRowD + kLatent);
      uint32_t* dst = reinterpret_cast<uint32_t*>(a.kv_cache + c * a.kv_bs + r * kRowD + kLatent);
      dst[lane] = rotate_pair(src[lane], cs, sn);
    }
    return;
  }
  // ---------------------------------------------------------------- queries
  const int b = t - a.T;
  __shared__ double cs_s[kPairs], sn_s[kPairs];
  if (threadIdx.x < kPairs) rope_angle(a.q_pos[b], threadIdx.x, a.log2_base, &cs_s[threadIdx.x], &sn_s[threadIdx.x]);
  __syncthreads();
  // A head's rotary dims are 128 contiguous bytes: 8 words of 16 bytes, word
  // j holding pairs 4j .. 4j+3 (words 64 .. 71 of the head's 72). Thread x
  // takes words x, x + kThreads, ... of the query, kWordsPer at a time with
  // every load issued before the first store.
  constexpr int kWordsPer = 8;
  constexpr int kHeadWords = kRowD * 2 / 16;     // 72
  constexpr int kRotWord0 = kLatent * 2 / 16;    // 64
  uint4* qb = reinterpret_cast<uint4*>(a.q + static_cast<int64_t>(b) * a.H * kRowD);
  const int words = a.H * 8;
  for (int base = 0; base < words; base += kThreads * kWordsPer) {
    uint4 v[kWordsPer];
#pragma unroll
    for (int j = 0; j < kWordsPer; ++j) {
      const int x = base + j * kThreads + threadIdx.x;
      if (x < words) v[j] = qb[(x >> 3) * kHeadWords + kRotWord0 + (x & 7)];
    }
#pragma unroll
    for (int j = 0; j < kWordsPer; ++j) {
      const int x = base + j * kThreads + threadIdx.x;
      if (x < words) {
        const int i0 = 4 * (x & 7);
        uint4 o;
        o.x = rotate_pair(v[j].x, cs_s[i0], sn_s[i0]);
        o.y = rotate_pair(v[j].y, cs_s[i0 + 1], sn_s[i0 + 1]);
        o.z = rotate_pair(v[j].z, cs_s[i0 + 2], sn_s[i0 + 2]);
        o.w = rotate_pair(v[j].w, cs_s[i0 + 3], sn_s[i0 + 3]);
        qb[(x >> 3) * kHeadWords + kRotWord0 + (x & 7)] = o;
      }
    }
  }
}

}  // namespace

cudaError_t launch_cache_append(const AppendArgs& a, cudaStream_t stream) {
  const int grid = a.T + (a.q ? a.B : 0);
  if (a.d_I == 64)
    cache_append_kernel<64><<<grid, kThreads, 0, stream>>>(a);
  else
    cache_append_kernel<128><<<grid, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace ic
