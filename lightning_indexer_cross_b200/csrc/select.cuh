// Exact selection of the k largest of n 64-bit keys by one CTA: an
// MSB-first radix select with 8-bit digits that stops as soon as the digit
// holding the k-th key is taken whole. Keys are read through an accessor, so
// they may sit in shared memory (one pass per digit over shared memory) or
// in global memory (one pass per digit over the row). Used with composite
// keys (order-preserving score key << 32 | ~position): "larger" means a
// higher score, then a lower position, which makes the k largest unique
// exactly the top-k with ties toward the lower position.
#pragma once

#include "common.cuh"

namespace ic {

struct SelectShared {
  uint32_t hist[256];
  int digit;
  uint32_t rank, count;
  uint32_t n_out, n_eq;
};

// Order-preserving 32-bit key of an fp32 score (negative: all bits flipped;
// otherwise: sign bit set).
IC_DEV uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Composite key: score key above, complemented position below.
IC_DEV uint64_t composite_key(uint32_t score_key, int32_t pos) {
  return (static_cast<uint64_t>(score_key) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(pos));
}
IC_DEV int32_t composite_pos(uint64_t key) { return static_cast<int32_t>(~static_cast<uint32_t>(key)); }

// Given per-digit counts (ascending digit) and a 1-based rank kr, the digit
// d holding the kr-th largest key: above(d) < kr <= above(d) + counts[d],
// above(d) = the counts of the digits above d. Writes d and kr - above(d).
// All NT threads must call (nbins a multiple of NT); synchronises the CTA.
template <int NT>
IC_DEV void find_digit(const uint32_t* counts, int nbins, uint32_t kr, int* d_out, uint32_t* kr_out,
                       uint32_t* warp_tot) {
  constexpr int kWarps = NT / 32;
  const int per = nbins / NT;
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

// Calls emit(key, pos) for each of the k largest keys (n > k), pos running
// over [0, k) without repeats. All NT threads of the CTA must call it; it
// synchronises the CTA. key(i) for i in [0, n).
template <int NT, typename KeyFn, typename EmitFn>
IC_DEV void select_k_largest(SelectShared& sh, int64_t n, uint32_t k, KeyFn&& key, EmitFn&& emit) {
  const int t = threadIdx.x;
  if (t == 0) {
    sh.n_out = 0;
    sh.n_eq = 0;
  }
  uint64_t prefix = 0;
  int shift = 64;
  uint32_t kr = k;
  while (shift > 0) {
    const int s2 = shift - 8;
    for (int i = t; i < 256; i += NT) sh.hist[i] = 0;
    __syncthreads();
    for (int64_t i = t; i < n; i += NT) {
      const uint64_t x = key(i);
      if (shift == 64 || (x >> shift) == prefix) atomicAdd(&sh.hist[(x >> s2) & 0xffu], 1u);
    }
    __syncthreads();
    if (t < 32) {
      // digits in descending order: lane l holds digits 255 - 8l .. 248 - 8l
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = sh.hist[255 - 8 * t - e];
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
            sh.digit = 255 - 8 * t - e;
            sh.rank = kr - above;
            sh.count = c[e];
          }
          above += c[e];
        }
      }
    }
    __syncthreads();
    prefix = (shift == 64 ? 0ull : (prefix << 8)) | static_cast<uint64_t>(sh.digit);
    shift = s2;
    kr = sh.rank;
    const bool take_whole = sh.count == kr;
    __syncthreads();  // every thread has read digit, rank and count
    if (take_whole) break;
  }
  // keys above the prefix, then kr keys equal to it (all of them when the
  // digit was taken whole; equal full keys are identical)
  const uint32_t n_above = k - kr;
  for (int64_t i = t; i < n; i += NT) {
    const uint64_t x = key(i);
    const uint64_t top = x >> shift;
    if (top > prefix) {
      const uint32_t p = atomicAdd(&sh.n_out, 1u);
      if (p < n_above) emit(x, p);
    } else if (top == prefix) {
      const uint32_t e = atomicAdd(&sh.n_eq, 1u);
      if (e < kr) emit(x, n_above + e);  // (all of them when the digit was taken whole)
    }
  }
  __syncthreads();
}

}  // namespace ic
