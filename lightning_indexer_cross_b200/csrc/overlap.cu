// Overlap of two index sets per row: count[r] = the number of valid entries
// of b[r, :] that also occur in a[r, :] (valid: 0 <= x < N; -1 padding and
// anything outside [0, N) is ignored). Used as the reuse diagnostic of the
// layer stack: how many of the tokens an S layer would select itself are in
// the index it reuses from the last F layer (Hy4 IndexCache explainer: reuse
// is free only where nearby layers want the same tokens; Bai et al. record:
// cross-layer reuse is not exact equality to each layer's own selection).
//
// One CTA per row: a bitmap of the N positions in shared memory, set from
// a's entries, then tested with b's entries; a CTA-wide sum of the hits.
#include "common.cuh"
#include "kernels.h"

namespace ic {

namespace {

constexpr int kOvThreads = 512;

__global__ void __launch_bounds__(kOvThreads) index_overlap_kernel(const int32_t* a, const int32_t* b, int k,
                                                                    int64_t N, int32_t* count) {
  extern __shared__ uint32_t bits[];
  __shared__ uint32_t warp_sum[kOvThreads / 32];
  const int r = blockIdx.x, t = threadIdx.x;
  const int words = static_cast<int>((N + 31) / 32);
  pdl_trigger();
  pdl_wait();
  for (int i = t; i < words; i += kOvThreads) bits[i] = 0u;
  __syncthreads();
  const int32_t* ar = a + static_cast<int64_t>(r) * k;
  const int32_t* br = b + static_cast<int64_t>(r) * k;
  for (int i = t; i < k; i += kOvThreads) {
    const int32_t x = __ldg(ar + i);
    if (x >= 0 && static_cast<int64_t>(x) < N) atomicOr(&bits[x >> 5], 1u << (x & 31));
  }
  __syncthreads();
  uint32_t hits = 0;
  for (int i = t; i < k; i += kOvThreads) {
    const int32_t x = __ldg(br + i);
    if (x >= 0 && static_cast<int64_t>(x) < N) hits += (bits[x >> 5] >> (x & 31)) & 1u;
  }
  hits = __reduce_add_sync(0xffffffffu, hits);
  if ((t & 31) == 0) warp_sum[t >> 5] = hits;
  __syncthreads();
  if (t < 32) {
    uint32_t v = t < kOvThreads / 32 ? warp_sum[t] : 0u;
    v = __reduce_add_sync(0xffffffffu, v);
    if (t == 0) count[r] = static_cast<int32_t>(v);
  }
}

}  // namespace

size_t index_overlap_smem_bytes(int64_t N) { return static_cast<size_t>((N + 31) / 32) * 4; }

cudaError_t launch_index_overlap(const int32_t* a, const int32_t* b, int B, int k, int64_t N, int32_t* count,
                                 cudaStream_t stream, bool pdl, int* launches) {
  const size_t smem = index_overlap_smem_bytes(N);
  static bool done[64] = {false};
  cudaError_t e = set_smem_once(index_overlap_kernel, 232448 - 1024, done);
  if (e != cudaSuccess) return e;
  e = launch_kernel(index_overlap_kernel, dim3(B), dim3(kOvThreads), smem, stream, pdl, a, b, k, N, count);
  if (e != cudaSuccess) return e;
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace ic
