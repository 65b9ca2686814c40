// Kernel argument structs and launchers of the IndexCache hot path (internal
// to the library; the public boundary is include/indexcache.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include <cuda_bf16.h>

#include "../../include/indexcache.h"

namespace ic {

// Bound, in nanoseconds, of every wait inside the kernels enqueued from now
// on (set with ic_set_wait_limit_ns).
uint64_t wait_limit_ns();

// Raise a kernel's dynamic shared-memory limit once per device (never again
// afterwards, so later calls are safe inside CUDA-graph capture). `done` is
// the caller's per-kernel flag array: kernels of one signature share a
// function type, so the flag cannot live in this template.
template <typename Kernel>
inline cudaError_t set_smem_once(Kernel kern, int bytes, bool (&done)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
  return e;
}

// Launch a kernel; with pdl set, with programmatic stream serialisation, so
// it may start while the previous kernel in the stream (one of this library's,
// which all wait with griddepcontrol.wait before touching global memory)
// finishes. Only set pdl when the previous stream operation is such a kernel.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                 bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// The same with thread-block clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                         cudaStream_t stream, bool pdl, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

struct IndexerArgs {
  // q [B, H_I, d_I] is read through its tensor map (and directly, to split it
  // into e4m3 parts, on the e4m3-key path with d_I = 128)
  const __nv_bfloat16* q;
  const float* w;              // [B, H_I]
  const float* k_scale;        // e4m3 keys: per-token scale
  int64_t scale_batch_stride;  // elements between queries' scales
  const int64_t* n_valid;      // [B] or null
  float* scores;               // [B, N]
  int* status;
  int B, H_I;
  int64_t N;
  int G;              // queries per group (share one key tile)
  int tiles;          // 128-key tiles per group
  int groups;         // ceil(B / G)
  int pair;           // groups per work item: 2 (one cache shared by all queries, >= 2 groups) or 1
  int64_t total_items;  // ceil(groups / pair) * tiles
  int per_query;      // 1: key cache z-coordinate = group (G == 1)
  int dual;           // 1: an item is one group on two key tiles (G * HP <= 128, pair == 1);
                      //    tiles then counts tile pairs
  uint64_t wait_ns;   // bound of every wait (0: give up unless already complete)
};

int indexer_smem_bytes(int d_I, bool fp8);
// map: the key cache (d_I, N, batch), 128-key boxes; qmap: the queries (d_I, H_I, B)
// with (64, HP, G) boxes, both 128-byte swizzled (e4m3 keys: 128-byte swizzle
// for d_I = 128, unswizzled rows for d_I = 64).
cudaError_t launch_indexer(const CUtensorMap& map, const CUtensorMap& qmap, const IndexerArgs& a, int HP, int d_I,
                           bool fp8, int grid, cudaStream_t stream, bool pdl);

// 32-bit words of per-row top-k control state (one 128-byte line per row,
// so rows do not contend for the same line in L2).
constexpr int kCtrlWords = 32;

struct TopkArgs {
  const float* scores;      // [B, N]
  const int64_t* n_valid;   // [B] or null
  int32_t* idx;             // [B, k]
  uint32_t* hist;           // [B][4096] row histograms of the top 12 key bits (zero between calls)
  int32_t* cand;            // [B][cand_cap] candidate positions (the k-th key's bin)
  uint32_t* cand_key;       // [B][cand_cap] their order-preserving keys
  uint32_t* counters;       // [B][kCtrlWords] per-row control state
  int* status;
  int B;
  int64_t N;
  int k;
  int cpr;                  // CTAs per row
  int64_t slice;            // elements per CTA slice
  int cand_cap;             // candidate buffer entries per row
  int fused;                // one clustered launch per row (cpr CTAs = one cluster) instead of two
};
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t stream, bool pdl, int* launches);
// The one-pass form: a sampled threshold, then one filter pass whose last
// CTA per row selects among the candidates (uses counters, cand, cand_key,
// cand_cap, cpr, slice; counters zero between calls).
cudaError_t launch_topk_threshold(const TopkArgs& a, cudaStream_t stream, bool pdl, int* launches);

// Scratch layout of the top-k passes for B rows of N scores (byte offsets
// from the start of the scratch region, which follows the status word).
enum TopkMode : int { kTopkCluster = 0, kTopkTwoPass = 1, kTopkThreshold = 2 };
struct TopkLayout {
  int cpr;         // CTAs per row
  int64_t slice;   // scores per CTA
  int mode;        // which kernels run (TopkMode)
  int fused;       // one clustered launch (cpr <= 4, slices <= 32768 scores)
  int cand_cap;
  size_t hist_off, cand_off, ckey_off, cnt_off, total;
  size_t zero_bytes;  // [0, zero_bytes): control words and row histograms, zero between calls
};
TopkLayout topk_layout(int B, int64_t N, int k);
// Validate and enqueue the top-k passes. The control words and row
// histograms ([0, zero_bytes)) must be zero on entry; every call that
// completes leaves them zero again.
ic_status_t topk_impl(const float* scores, int B, int64_t N, const int64_t* n_valid, int k, int32_t* idx,
                      uint8_t* ws, size_t ws_bytes, int* status, cudaStream_t stream, bool pdl);

struct MlaArgs {
  const __nv_bfloat16* q;    // [B, H, 576]
  const __nv_bfloat16* kv;   // latent caches
  int64_t kv_batch_stride;   // elements
  int64_t N;
  const int32_t* idx;        // [B, k]
  int k;
  const float* sink;         // [H]
  const __nv_bfloat16* gate; // [B, H, 512] or null
  float sm_scale;
  int B, H;
  int splits;                // ceil(k / TS)
  int ts;                    // selected rows per work unit
  int units;                 // splits * B * ceil(H / 128) work units
  int ctas;                  // persistent CTAs (each takes units blockIdx.x + i * ctas)
  void* part_o;              // [B, H, splits, 512] normalised O/l: bf16 if out is bf16, else fp32
  float* part_ml;            // [B, H, splits, 2]  (max in log2 units, sum)
  void* out;                 // [B, H, 512]
  int out_f32;
  float* lse;                // [B, H] or null
  int* status;
  uint64_t wait_ns;          // bound of every wait (0: give up unless already complete)
};
int mla_smem_bytes(int ts);
// qmap: 2-D tensor map over q viewed as [B*H rows, 576] bf16, box 64 x 128,
// 128-byte swizzle (one 64-dim slice of a 128-head block per load).
// omap: 4-D tensor map over part_o as [B][H][splits][512] (innermost first:
// 512, splits, H, B), box 128 bytes x 1 x 32 x 1, 128-byte swizzle (32 heads'
// rows of one 64-dim (bf16) or 32-dim (fp32) block per store).
cudaError_t launch_sparse_mla(const CUtensorMap& qmap, const CUtensorMap& omap, const MlaArgs& a,
                              cudaStream_t stream, bool pdl, int* launches);

// ---------------------------------------------------------------- index overlap
size_t index_overlap_smem_bytes(int64_t N);
cudaError_t launch_index_overlap(const int32_t* a, const int32_t* b, int B, int k, int64_t N, int32_t* count,
                                 cudaStream_t stream, bool pdl, int* launches);

// ---------------------------------------------------------------- cache append
struct AppendArgs {
  const __nv_bfloat16* k_raw;    // [T, d_I] indexer keys before the norm
  const float* gamma;            // [d_I] LayerNorm weight
  const float* beta;             // [d_I] LayerNorm bias
  float eps;
  int fp8;                       // key cache holds e4m3 codes + per-token scales
  void* key_cache;               // bf16 elements or e4m3 bytes
  float* key_scale;              // e4m3 only
  int64_t k_bs, s_bs, kv_bs;     // per-token cache strides (elements; 0 = one shared cache)
  const __nv_bfloat16* kv_raw;   // [T, 576] latent rows, rotary dims unrotated
  __nv_bfloat16* kv_cache;
  const int64_t* pos;            // [T] destination row = position
  int T, d_I;
  int64_t N;                     // rows per cache
  double log2_base;              // log2 of the RoPE base
  __nv_bfloat16* q;              // [B, H, 576] rotated in place, or null
  const int64_t* q_pos;          // [B]
  int B, H;
  int* status;
};
cudaError_t launch_cache_append(const AppendArgs& a, cudaStream_t stream);

// ---------------------------------------------------------------- output gate
struct GateArgs {
  const __nv_bfloat16* gate;  // [B, H, 128] or null (identity)
  void* out;                  // [B, H, 128] bf16 or fp32
  int out_f32;
  int B, H;
  int* status;
  uint64_t wait_ns;           // bound of every wait (0: give up unless already complete)
};
int gate_smem_bytes();
// wmap: 3-D tensor map over wv_b (512, 128, H), box 64 x 128 x 1; omap: 3-D
// over the latent outputs (512, H, B), box 64 x 1 x 128; both bf16 with the
// 128-byte swizzle.
cudaError_t launch_gate(const CUtensorMap& wmap, const CUtensorMap& omap, const GateArgs& a, cudaStream_t stream);

// ---------------------------------------------------------------- context parallel
// Candidates per row the merge holds in shared memory (G ranks x k).
constexpr int kCpMaxCand = 16384;

struct CpCandArgs {
  const float* scores;   // [B, N_local] this rank's shard scores
  const int32_t* idx;    // [B, k] local top-k (shard positions, -1 padding)
  int B, k;
  int64_t N_local;
  int64_t offset;        // global position of the shard's first token
  float* cand_score;     // [B, k]
  int32_t* cand_idx;     // [B, k] global positions (-1 padding)
  int* status;
};
cudaError_t launch_cp_candidates(const CpCandArgs& a, cudaStream_t stream);

struct CpMergeArgs {
  const float* cand_score;  // [G][B, kin] segments seg_stride elements apart
  const int32_t* cand_idx;  // the same layout: global positions (-1 padding)
  int64_t seg_stride;
  int G, B, kin, k;
  int64_t lo, hi;           // this rank's shard [lo, hi) of the global positions
  int32_t* idx_global;      // [B, k]
  int32_t* idx_local;       // [B, k] positions inside the shard, -1 elsewhere (or null)
};
cudaError_t launch_cp_merge_topk(const CpMergeArgs& a, cudaStream_t stream);

struct CpCombineArgs {
  const float* part_out;      // [G][B, H, 512] each rank's normalised partial output
  const float* part_lse;      // [G][B, H] each rank's natural-log sum (-inf: no row)
  int64_t out_stride;         // elements between ranks' outputs
  int64_t lse_stride;         // elements between ranks' lse arrays
  int G, B, H;
  const float* sink;          // [H]
  const __nv_bfloat16* gate;  // [B, H, 512] or null
  void* out;                  // [B, H, 512]
  int out_f32;
  float* lse;                 // [B, H] or null
};
cudaError_t launch_cp_combine(const CpCombineArgs& a, cudaStream_t stream);

}  // namespace ic
