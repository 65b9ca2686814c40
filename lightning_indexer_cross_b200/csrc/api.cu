// C ABI of the IndexCache hot path: argument validation (on the host, before
// any launch), workspace layouts, TMA descriptor encoding, and the F/S layer
// stack driver (Hy4-preview porting issue, "Indexer" bullet: shared layers
// reuse the last preceding full layer's top-k).
#include <cmath>
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/indexcache.h"
#include "kernels.h"

namespace {

thread_local int g_launches = 0;

// Bound of the waits inside the kernels (ic_set_wait_limit_ns).
std::atomic<uint64_t> g_wait_ns{2000000000ull};

constexpr size_t kStatusBytes = 256;  // status word + padding (keeps regions aligned)

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
template <typename T>
inline T ceil_div(T a, T b) { return (a + b - 1) / b; }

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// ------------------------------------------------------------------ indexer
int indexer_hp(int H_I) {
  int hp = ((H_I + 15) / 16) * 16;
  if (hp <= 16) return 16;
  if (hp <= 32) return 32;
  if (hp <= 64) return 64;
  return 128;
}

ic_status_t indexer_impl(const void* q, const float* w, const void* k, const float* k_scale, ic_dtype_t k_dtype,
                         int B, int H_I, int d_I, int64_t N, int64_t k_batch_stride, int64_t scale_batch_stride,
                         const int64_t* n_valid, float* scores, int* status, cudaStream_t stream, bool pdl) {
  if (!q || !w || !k || !scores) return IC_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H_I < 1 || N >= (int64_t(1) << 31)) return IC_ERR_INVALID_ARG;
  if (k_dtype != IC_BF16 && k_dtype != IC_FP8_E4M3) return IC_ERR_UNSUPPORTED;
  if (d_I != 64 && d_I != 128) return IC_ERR_UNSUPPORTED;
  if (H_I > 128) return IC_ERR_UNSUPPORTED;
  const bool fp8 = k_dtype == IC_FP8_E4M3;
  if (fp8 && !k_scale) return IC_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(w) || !aligned16(scores) || (k_scale && !aligned16(k_scale)))
    return IC_ERR_INVALID_ARG;
  if (k_batch_stride < 0 || scale_batch_stride < 0) return IC_ERR_INVALID_ARG;
  const int esz = fp8 ? 1 : 2;
  const bool per_query = k_batch_stride != 0 && B > 1;
  if (per_query && ((k_batch_stride * esz) % 16 != 0 || k_batch_stride < N * d_I)) return IC_ERR_INVALID_ARG;
  if (fp8 && per_query && scale_batch_stride < N) return IC_ERR_INVALID_ARG;

  EncodeTiledFn enc = encode_fn();
  if (!enc) return IC_ERR_CUDA;
  CUtensorMap map;
  const cuuint64_t bk = per_query ? static_cast<cuuint64_t>(B) : 1;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d_I), static_cast<cuuint64_t>(N), bk};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d_I) * esz,
                                 static_cast<cuuint64_t>(per_query ? k_batch_stride : N * d_I) * esz};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(fp8 ? d_I : 64), 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(&map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(k), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   // e4m3 keys with d_I = 128 go to the MMA as they land (128-byte
                   // rows, 128-byte swizzle); with d_I = 64 they are widened first
                   (fp8 && d_I == 64) ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return IC_ERR_INVALID_ARG;
  const int HP = indexer_hp(H_I);
  const int G = per_query ? 1 : std::min(256 / HP, B);
  // queries: (d_I, H_I, B); a (64, HP, G) box is one 64-dim block of a query
  // group's stacked heads, heads past H_I and queries past B read as zeros
  CUtensorMap qmap;
  const cuuint64_t qdims[3] = {static_cast<cuuint64_t>(d_I), static_cast<cuuint64_t>(H_I), static_cast<cuuint64_t>(B)};
  const cuuint64_t qstrides[2] = {static_cast<cuuint64_t>(d_I) * 2, static_cast<cuuint64_t>(H_I) * d_I * 2};
  const cuuint32_t qbox[3] = {64, static_cast<cuuint32_t>(HP), static_cast<cuuint32_t>(G)};
  r = enc(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), qdims, qstrides, qbox, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return IC_ERR_INVALID_ARG;

  ic::IndexerArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.w = w;
  a.k_scale = k_scale;
  a.scale_batch_stride = per_query ? scale_batch_stride : 0;
  a.n_valid = n_valid;
  a.scores = scores;
  a.status = status;
  a.B = B;
  a.H_I = H_I;
  a.N = N;
  a.G = G;
  a.tiles = static_cast<int>(ceil_div<int64_t>(N, 128));
  const int64_t groups = ceil_div<int64_t>(B, a.G);
  a.groups = static_cast<int>(groups);
  a.pair = (!fp8 && !per_query && groups >= 2) ? 2 : 1;
  // one group's heads fill at most half of the accumulator: two key tiles per
  // item, so that both halves of the epilogue reduce
  a.dual = (a.pair == 1 && a.G * HP <= 128) ? 1 : 0;
  if (a.dual) a.tiles = static_cast<int>(ceil_div<int64_t>(a.tiles, 2));
  a.total_items = ceil_div<int64_t>(groups, a.pair) * a.tiles;
  a.per_query = per_query ? 1 : 0;
  a.wait_ns = ic::wait_limit_ns();
  const int grid = static_cast<int>(std::min<int64_t>(num_sms(), a.total_items));
  cudaError_t e = ic::launch_indexer(map, qmap, a, HP, d_I, fp8, grid, stream, pdl);
  if (e != cudaSuccess) return IC_ERR_CUDA;
  g_launches += 1;
  return IC_OK;
}

}  // namespace

namespace ic {

uint64_t wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

// ------------------------------------------------------------------ top-k
TopkLayout topk_layout(int B, int64_t N, int k) {
  TopkLayout L{};
  // the row's CTAs: about two 512-thread CTAs per SM in total, at least 4096
  // scores per CTA
  const int64_t target = std::max<int64_t>(1, 2 * num_sms() / std::max(B, 1));
  int64_t cpr = std::min<int64_t>(ceil_div<int64_t>(N, 4096), target);
  cpr = std::max<int64_t>(cpr, 1);
  int64_t slice = ceil_div<int64_t>(N, cpr);
  slice = ceil_div<int64_t>(slice, 4) * 4;
  cpr = ceil_div<int64_t>(N, slice);
  L.cpr = static_cast<int>(cpr);
  L.slice = slice;
  L.mode = kTopkTwoPass;
  // one clustered launch per row (a cluster of c <= 4 CTAs, one per SM, each
  // holding up to 32768 scores) when the rows keep at least half of the SMs
  // busy; c grows while the grid still fits one wave
  if ((N & 3) == 0 && N <= 4 * 32768) {
    int c = 1;
    while (c < 4 && ceil_div<int64_t>(N, c) > 32768) c *= 2;
    while (c < 4 && int64_t(B) * c * 2 <= num_sms() && ceil_div<int64_t>(N, c * 2) >= 4096) c *= 2;
    if (int64_t(B) * c * 2 >= num_sms()) {
      L.mode = kTopkCluster;
      L.cpr = c;
      L.slice = ceil_div<int64_t>(ceil_div<int64_t>(N, c), 4) * 4;
    }
  }
  // many rows, few CTAs per row (a prefill chunk): each CTA would pass over
  // a large slice twice; one pass above a sampled threshold instead
  if (L.mode == kTopkTwoPass && L.cpr <= 4) L.mode = kTopkThreshold;
  L.fused = L.mode == kTopkCluster ? 1 : 0;
  L.cnt_off = 0;  // control words (and row histograms): zero between calls
  L.hist_off = align256(L.cnt_off + size_t(B) * ic::kCtrlWords * 4);
  if (L.mode == kTopkThreshold) {
    // candidates above the threshold: twice the expected 2k per row
    L.cand_cap = static_cast<int>(std::min<int64_t>(N, std::max<int64_t>(8192, 4 * int64_t(std::max(k, 1)))));
    L.cand_off = L.hist_off;  // no row histograms
  } else {
    // the k-th key's 1/16-octave bin rarely holds more than a few percent of
    // a row; bigger bins fall back to passes over the row itself
    L.cand_cap = static_cast<int>(std::min<int64_t>(N, std::max<int64_t>(4096, N / 16)));
    L.cand_off = align256(L.hist_off + size_t(B) * 4096 * 4);
  }
  L.zero_bytes = L.cand_off;
  L.ckey_off = align256(L.cand_off + size_t(B) * L.cand_cap * 4);
  L.total = align256(L.ckey_off + size_t(B) * L.cand_cap * 4);
  return L;
}

ic_status_t topk_impl(const float* scores, int B, int64_t N, const int64_t* n_valid, int k, int32_t* idx,
                      uint8_t* ws, size_t ws_bytes, int* status, cudaStream_t stream, bool pdl) {
  if (!scores || !idx || !ws) return IC_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || N >= (int64_t(1) << 31) || k < 1 || k > 16384) return IC_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(idx)) return IC_ERR_INVALID_ARG;
  TopkLayout L = topk_layout(B, N, k);
  if (ws_bytes < L.total) return IC_ERR_INVALID_ARG;
  ic::TopkArgs a{};
  a.scores = scores;
  a.n_valid = n_valid;
  a.idx = idx;
  a.hist = reinterpret_cast<uint32_t*>(ws + L.hist_off);
  a.cand = reinterpret_cast<int32_t*>(ws + L.cand_off);
  a.cand_key = reinterpret_cast<uint32_t*>(ws + L.ckey_off);
  a.counters = reinterpret_cast<uint32_t*>(ws + L.cnt_off);
  a.cand_cap = L.cand_cap;
  a.status = status;
  a.B = B;
  a.N = N;
  a.k = k;
  a.cpr = L.cpr;
  a.slice = L.slice;
  a.fused = L.fused;
  int launches = 0;
  cudaError_t e = L.mode == kTopkThreshold ? ic::launch_topk_threshold(a, stream, pdl, &launches)
                                            : ic::launch_topk(a, stream, pdl, &launches);
  if (e != cudaSuccess) return IC_ERR_CUDA;
  g_launches += launches;
  return IC_OK;
}

}  // namespace ic

namespace {

using ic::TopkLayout;
using ic::topk_layout;
using ic::topk_impl;

// ------------------------------------------------------------------ indexer -> top-k
// Rows per pass of the fused indexer -> top-k: all B rows when rows_per_pass
// is 0, else rows_per_pass rounded up to a multiple of 8 (whole pairs of
// 4-query groups; keeps every row offset of q, w and idx 16-byte aligned).
int fused_rows(int B, int rows_per_pass) {
  if (rows_per_pass <= 0 || rows_per_pass >= B) return B;
  const int r = (rows_per_pass + 7) / 8 * 8;
  return r < B ? r : B;
}

struct FusedLayout {
  int R;
  size_t scores_off, topk_off, total;  // offsets from the start of the region
  TopkLayout tk;
};

FusedLayout fused_layout(int B, int64_t N, int topk, int rows_per_pass) {
  FusedLayout L{};
  L.R = fused_rows(B, rows_per_pass);
  L.tk = topk_layout(L.R, N, topk);
  L.scores_off = 0;
  L.topk_off = align256(size_t(L.R) * N * 4);
  L.total = align256(L.topk_off + L.tk.total);
  return L;
}

// Scores of R rows at a time into the region's scratch, then their top-k;
// the next pass reuses the scratch. The first kernel launches with
// programmatic serialisation only if `pdl` (it follows one of the
// library's kernels in the stream).
ic_status_t indexer_topk_impl(const void* q, const float* w, const void* k, const float* k_scale, ic_dtype_t k_dtype,
                              int B, int H_I, int d_I, int64_t N, int64_t k_batch_stride, int64_t scale_batch_stride,
                              const int64_t* n_valid, int topk, int rows_per_pass, int32_t* idx, uint8_t* region,
                              size_t region_bytes, int* status, cudaStream_t stream, bool pdl, int* launches) {
  if (!q || !w || !k || !idx || !region) return IC_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H_I < 1 || topk < 1) return IC_ERR_INVALID_ARG;
  const FusedLayout L = fused_layout(B, N, topk, rows_per_pass);
  if (region_bytes < L.total || !aligned16(region)) return IC_ERR_INVALID_ARG;
  const bool fp8 = k_dtype == IC_FP8_E4M3;
  const int64_t esz = fp8 ? 1 : 2;
  const bool per_query = k_batch_stride != 0 && B > 1;
  const bool per_query_scale = scale_batch_stride != 0 && B > 1;
  float* scores = reinterpret_cast<float*>(region + L.scores_off);
  for (int r0 = 0; r0 < B; r0 += L.R) {
    const int R = B - r0 < L.R ? B - r0 : L.R;
    const uint8_t* qb = static_cast<const uint8_t*>(q) + size_t(r0) * H_I * d_I * 2;
    const uint8_t* kb = static_cast<const uint8_t*>(k) + (per_query ? size_t(r0) * k_batch_stride * esz : 0);
    const float* ksb = k_scale ? k_scale + (per_query_scale ? size_t(r0) * scale_batch_stride : 0) : nullptr;
    const int64_t* nvb = n_valid ? n_valid + r0 : nullptr;
    g_launches = 0;
    ic_status_t st = indexer_impl(qb, w + size_t(r0) * H_I, kb, ksb, k_dtype, R, H_I, d_I, N,
                                  per_query ? k_batch_stride : 0, per_query_scale ? scale_batch_stride : 0, nvb,
                                  scores, status, stream, pdl || r0 > 0);
    if (st != IC_OK) return st;
    *launches += g_launches;
    g_launches = 0;
    st = topk_impl(scores, R, N, nvb, topk, idx + size_t(r0) * topk, region + L.topk_off, L.tk.total, status,
                   stream, true);
    if (st != IC_OK) return st;
    *launches += g_launches;
  }
  return IC_OK;
}

// ------------------------------------------------------------------ sparse MLA
// Selected rows per work unit: the largest of 256, 128 that still gives at
// least 4/5 of a work unit per SM, else 64.
int mla_ts(int B, int H, int k) {
  const int hb = (H + 127) / 128;
  const int sms = num_sms();
  for (int ts : {256, 128}) {
    const int64_t units = ceil_div<int64_t>(k, ts) * B * hb;
    if (units * 5 >= static_cast<int64_t>(sms) * 4) return ts;
  }
  return 64;
}

struct MlaLayout {
  int ts, splits;
  size_t o_off, ml_off, total;
};

MlaLayout mla_layout(int B, int H, int k) {
  MlaLayout L{};
  L.ts = mla_ts(B, H, k);
  L.splits = ceil_div(k, L.ts);
  L.o_off = 0;
  L.ml_off = align256(L.o_off + size_t(B) * H * L.splits * 512 * 4);
  L.total = align256(L.ml_off + size_t(B) * H * L.splits * 2 * 4);
  return L;
}

ic_status_t mla_impl(const void* q, const void* kv, int64_t kv_batch_stride, int64_t N, const int32_t* idx, int k,
                     const float* sink, const void* gate, float sm_scale, int B, int H, ic_dtype_t out_dtype,
                     void* out, float* lse, uint8_t* ws, size_t ws_bytes, int* status, cudaStream_t stream,
                     bool pdl) {
  if (!q || !kv || !idx || !sink || !out || !ws) return IC_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || k < 1 || N < 1 || N >= (int64_t(1) << 31)) return IC_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || sm_scale == INFINITY) return IC_ERR_INVALID_ARG;
  if (out_dtype != IC_BF16 && out_dtype != IC_F32) return IC_ERR_UNSUPPORTED;
  if (kv_batch_stride < 0 || (kv_batch_stride != 0 && kv_batch_stride < N * 576)) return IC_ERR_INVALID_ARG;
  if ((kv_batch_stride * 2) % 16 != 0) return IC_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(idx) || !aligned16(out) || (gate && !aligned16(gate)))
    return IC_ERR_INVALID_ARG;
  MlaLayout L = mla_layout(B, H, k);
  if (ws_bytes < L.total || !aligned16(ws)) return IC_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * H >= (int64_t(1) << 31)) return IC_ERR_INVALID_ARG;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return IC_ERR_CUDA;
  CUtensorMap qmap;
  {
    const cuuint64_t dims[2] = {576, static_cast<cuuint64_t>(B) * H};
    const cuuint64_t strides[1] = {576 * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return IC_ERR_INVALID_ARG;
  }
  CUtensorMap omap;
  {
    const bool f32 = out_dtype == IC_F32;
    const cuuint64_t es = f32 ? 4 : 2;
    const cuuint64_t dims[4] = {512, static_cast<cuuint64_t>(L.splits), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {512 * es, 512 * es * L.splits, 512 * es * L.splits * H};
    const cuuint32_t box[4] = {f32 ? 32u : 64u, 1, 32, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (enc(&omap, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, ws + L.o_off, dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return IC_ERR_INVALID_ARG;
  }
  ic::MlaArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.kv = static_cast<const __nv_bfloat16*>(kv);
  a.kv_batch_stride = B > 1 ? kv_batch_stride : 0;
  a.N = N;
  a.idx = idx;
  a.k = k;
  a.sink = sink;
  a.gate = static_cast<const __nv_bfloat16*>(gate);
  a.sm_scale = sm_scale;
  a.B = B;
  a.H = H;
  a.splits = L.splits;
  a.ts = L.ts;
  {
    const int64_t units = int64_t(L.splits) * B * ((H + 127) / 128);
    if (units >= (int64_t(1) << 31)) return IC_ERR_INVALID_ARG;
    a.units = static_cast<int>(units);
    a.ctas = static_cast<int>(std::min<int64_t>(units, num_sms()));
  }
  a.part_o = ws + L.o_off;
  a.part_ml = reinterpret_cast<float*>(ws + L.ml_off);
  a.out = out;
  a.out_f32 = out_dtype == IC_F32 ? 1 : 0;
  a.lse = lse;
  a.status = status;
  a.wait_ns = ic::wait_limit_ns();
  int launches = 0;
  cudaError_t e = ic::launch_sparse_mla(qmap, omap, a, stream, pdl, &launches);
  if (e != cudaSuccess) return IC_ERR_CUDA;
  g_launches += launches;
  return IC_OK;
}

// ------------------------------------------------------------------ stack
struct StackLayout {
  size_t fused_off, mla_off, total;
  FusedLayout fz;
  MlaLayout ml;
};

StackLayout stack_layout(const ic_stack_shape_t& s) {
  StackLayout L{};
  L.fz = fused_layout(s.B, s.N, s.topk, s.rows_per_pass);
  L.ml = mla_layout(s.B, s.H, s.topk);
  L.fused_off = kStatusBytes;
  L.mla_off = align256(L.fused_off + L.fz.total);
  L.total = align256(L.mla_off + L.ml.total);
  return L;
}

}  // namespace

extern "C" {

const char* ic_status_string(ic_status_t s) {
  switch (s) {
    case IC_OK: return "IC_OK";
    case IC_ERR_INVALID_ARG: return "IC_ERR_INVALID_ARG: bad pointer, size, alignment or schedule";
    case IC_ERR_UNSUPPORTED: return "IC_ERR_UNSUPPORTED: valid shape with no kernel in this build";
    case IC_ERR_CUDA: return "IC_ERR_CUDA: a CUDA call or launch failed";
    case IC_ERR_TIMEOUT: return "IC_ERR_TIMEOUT: a bounded wait inside a kernel gave up";
    case IC_ERR_BAD_INDEX: return "IC_ERR_BAD_INDEX: an index outside [-1, N) was read";
  }
  return "unknown ic_status_t";
}

int ic_last_launch_count(void) { return g_launches; }

void ic_set_wait_limit_ns(uint64_t ns) { g_wait_ns.store(ns, std::memory_order_relaxed); }

uint64_t ic_wait_limit_ns(void) { return g_wait_ns.load(std::memory_order_relaxed); }

size_t ic_indexer_workspace_size(void) { return kStatusBytes; }

ic_status_t ic_indexer_score(const void* q, const float* w, const void* k, const float* k_scale, ic_dtype_t k_dtype,
                             int B, int H_I, int d_I, int64_t N, int64_t k_batch_stride, int64_t scale_batch_stride,
                             const int64_t* n_valid, float* scores, void* workspace, size_t ws_bytes,
                             ic_stream_t stream) {
  g_launches = 0;
  if (!workspace || ws_bytes < kStatusBytes || !aligned16(workspace)) return IC_ERR_INVALID_ARG;
  return indexer_impl(q, w, k, k_scale, k_dtype, B, H_I, d_I, N, k_batch_stride, scale_batch_stride, n_valid,
                      scores, static_cast<int*>(workspace), reinterpret_cast<cudaStream_t>(stream), false);
}

size_t ic_topk_workspace_size(int B, int64_t N, int k) {
  if (B < 1 || N < 1) return kStatusBytes;
  return kStatusBytes + topk_layout(B, N, k).total;
}

ic_status_t ic_topk(const float* scores, int B, int64_t N, const int64_t* n_valid, int k, int32_t* idx,
                    void* workspace, size_t ws_bytes, ic_stream_t stream) {
  g_launches = 0;
  if (!workspace || ws_bytes < kStatusBytes || !aligned16(workspace)) return IC_ERR_INVALID_ARG;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return topk_impl(scores, B, N, n_valid, k, idx, ws + kStatusBytes, ws_bytes - kStatusBytes,
                   reinterpret_cast<int*>(ws), reinterpret_cast<cudaStream_t>(stream), false);
}

size_t ic_indexer_topk_workspace_size(int B, int64_t N, int k, int rows_per_pass) {
  if (B < 1 || N < 1) return kStatusBytes;
  return kStatusBytes + fused_layout(B, N, k, rows_per_pass).total;
}

ic_status_t ic_indexer_topk(const void* q, const float* w, const void* k, const float* k_scale, ic_dtype_t k_dtype,
                            int B, int H_I, int d_I, int64_t N, int64_t k_batch_stride, int64_t scale_batch_stride,
                            const int64_t* n_valid, int topk, int rows_per_pass, int32_t* idx, void* workspace,
                            size_t ws_bytes, ic_stream_t stream) {
  g_launches = 0;
  if (!workspace || ws_bytes < kStatusBytes || !aligned16(workspace)) return IC_ERR_INVALID_ARG;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int n = 0;
  const ic_status_t r = indexer_topk_impl(q, w, k, k_scale, k_dtype, B, H_I, d_I, N, k_batch_stride,
                                          scale_batch_stride, n_valid, topk, rows_per_pass, idx, ws + kStatusBytes,
                                          ws_bytes - kStatusBytes, reinterpret_cast<int*>(ws),
                                          reinterpret_cast<cudaStream_t>(stream), false, &n);
  g_launches = n;
  return r;
}

size_t ic_sparse_mla_workspace_size(int B, int H, int k) {
  if (B < 1 || H < 1 || k < 1) return kStatusBytes;
  return kStatusBytes + mla_layout(B, H, k).total;
}

ic_status_t ic_sparse_mla_decode(const void* q, const void* kv, int64_t kv_batch_stride, int64_t N,
                                 const int32_t* idx, int k, const float* sink, const void* gate, float sm_scale,
                                 int B, int H, ic_dtype_t out_dtype, void* out, float* lse, void* workspace,
                                 size_t ws_bytes, ic_stream_t stream) {
  g_launches = 0;
  if (!workspace || ws_bytes < kStatusBytes || !aligned16(workspace)) return IC_ERR_INVALID_ARG;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return mla_impl(q, kv, kv_batch_stride, N, idx, k, sink, gate, sm_scale, B, H, out_dtype, out, lse,
                  ws + kStatusBytes, ws_bytes - kStatusBytes, reinterpret_cast<int*>(ws),
                  reinterpret_cast<cudaStream_t>(stream), false);
}

size_t ic_layer_stack_workspace_size(const ic_stack_shape_t* shape) {
  if (!shape || shape->B < 1 || shape->N < 1 || shape->H < 1 || shape->topk < 1) return kStatusBytes;
  return stack_layout(*shape).total;
}

ic_status_t ic_layer_stack(const ic_layer_t* layers, int L, const char* schedule, const ic_stack_shape_t* shape,
                           int32_t* index_buf, int32_t* idx_trace, void* workspace, size_t ws_bytes,
                           ic_stream_t stream) {
  g_launches = 0;
  if (!layers || !schedule || !shape || !index_buf || !workspace || L < 1) return IC_ERR_INVALID_ARG;
  if (!aligned16(workspace) || !aligned16(index_buf) || (idx_trace && !aligned16(idx_trace)))
    return IC_ERR_INVALID_ARG;
  const ic_stack_shape_t& s = *shape;
  if (s.B < 1 || s.N < 1 || s.topk < 1 || s.H < 1) return IC_ERR_INVALID_ARG;
  // schedule: exactly L characters from {F, S}, starting with F
  for (int l = 0; l < L; ++l)
    if (schedule[l] != 'F' && schedule[l] != 'S') return IC_ERR_INVALID_ARG;
  if (schedule[L] != '\0' || schedule[0] != 'F') return IC_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l) {
    const ic_layer_t& y = layers[l];
    if (!y.q || !y.kv || !y.sink || !y.out) return IC_ERR_INVALID_ARG;
    if (schedule[l] == 'F' && (!y.q_idx || !y.w || !y.k_idx)) return IC_ERR_INVALID_ARG;
    if (schedule[l] == 'F' && s.k_dtype == IC_FP8_E4M3 && !y.k_scale) return IC_ERR_INVALID_ARG;
  }
  StackLayout SL = stack_layout(s);
  if (ws_bytes < SL.total) return IC_ERR_INVALID_ARG;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int total = 0;
  // Consecutive kernels of the stack overlap their launch and prologue with
  // the previous kernel's tail (programmatic dependent launch). The first
  // kernel of the call, and any kernel after a copy or memset, launches
  // normally.
  bool after_kernel = false;
  for (int l = 0; l < L; ++l) {
    const ic_layer_t& y = layers[l];
    if (y.wait_event) {
      if (cudaStreamWaitEvent(st, static_cast<cudaEvent_t>(y.wait_event), 0) != cudaSuccess) return IC_ERR_CUDA;
      after_kernel = false;
    }
    if (schedule[l] == 'F') {
      int n = 0;
      ic_status_t r = indexer_topk_impl(y.q_idx, y.w, y.k_idx, y.k_scale, s.k_dtype, s.B, s.H_I, s.d_I, s.N,
                                        s.k_batch_stride, s.scale_batch_stride, s.n_valid, s.topk, s.rows_per_pass,
                                        index_buf, ws + SL.fused_off, SL.fz.total, status, st, after_kernel, &n);
      if (r != IC_OK) return r;
      total += n;
      after_kernel = true;
    }
    g_launches = 0;
    ic_status_t r = mla_impl(y.q, y.kv, s.kv_batch_stride, s.N, index_buf, s.topk, y.sink, y.gate, s.sm_scale,
                             s.B, s.H, s.out_dtype, y.out, y.lse, ws + SL.mla_off, SL.ml.total, status, st,
                             after_kernel);
    if (r != IC_OK) return r;
    total += g_launches;
    after_kernel = true;
    if (idx_trace) {
      const size_t n = size_t(s.B) * s.topk;
      if (cudaMemcpyAsync(idx_trace + size_t(l) * n, index_buf, n * 4, cudaMemcpyDeviceToDevice, st) !=
          cudaSuccess)
        return IC_ERR_CUDA;
      after_kernel = false;
    }
  }
  g_launches = total;
  return IC_OK;
}

size_t ic_cache_append_workspace_size(void) { return kStatusBytes; }

ic_status_t ic_cache_append(const void* k_raw, const float* ln_gamma, const float* ln_beta, float ln_eps,
                            ic_dtype_t k_dtype, void* key_cache, float* key_scale, int64_t k_batch_stride,
                            int64_t scale_batch_stride, const void* kv_raw, void* kv_cache,
                            int64_t kv_batch_stride, const int64_t* pos, int T, int d_I, int64_t N,
                            float rope_base, void* q, const int64_t* q_pos, int B, int H, void* workspace,
                            size_t ws_bytes, ic_stream_t stream) {
  g_launches = 0;
  if (!workspace || ws_bytes < kStatusBytes || !aligned16(workspace)) return IC_ERR_INVALID_ARG;
  if (!k_raw || !ln_gamma || !ln_beta || !key_cache || !kv_raw || !kv_cache || !pos) return IC_ERR_INVALID_ARG;
  if (T < 1 || N < 1) return IC_ERR_INVALID_ARG;
  if (k_dtype != IC_BF16 && k_dtype != IC_FP8_E4M3) return IC_ERR_UNSUPPORTED;
  if (d_I != 64 && d_I != 128) return IC_ERR_UNSUPPORTED;
  const bool fp8 = k_dtype == IC_FP8_E4M3;
  if (fp8 != (key_scale != nullptr)) return IC_ERR_INVALID_ARG;
  if (!(ln_eps >= 0.f) || !std::isfinite(ln_eps) || !(rope_base > 0.f) || !std::isfinite(rope_base))
    return IC_ERR_INVALID_ARG;
  if (!aligned16(k_raw) || !aligned16(key_cache) || !aligned16(kv_raw) || !aligned16(kv_cache) ||
      (q && !aligned16(q)))
    return IC_ERR_INVALID_ARG;
  const int64_t esz = fp8 ? 1 : 2;
  if (k_batch_stride < 0 || scale_batch_stride < 0 || kv_batch_stride < 0) return IC_ERR_INVALID_ARG;
  // nonzero strides: token t writes cache t, which must not overlap cache t+1
  if (k_batch_stride != 0 && (k_batch_stride < N * d_I || (k_batch_stride * esz) % 16 != 0))
    return IC_ERR_INVALID_ARG;
  if (kv_batch_stride != 0 && (kv_batch_stride < N * 576 || (kv_batch_stride * 2) % 16 != 0))
    return IC_ERR_INVALID_ARG;
  if (fp8 && scale_batch_stride != 0 && scale_batch_stride < N) return IC_ERR_INVALID_ARG;
  if (q && (!q_pos || B < 1 || H < 1)) return IC_ERR_INVALID_ARG;
  if (static_cast<int64_t>(T) + (q ? B : 0) >= (int64_t(1) << 31)) return IC_ERR_INVALID_ARG;

  ic::AppendArgs a{};
  a.k_raw = static_cast<const __nv_bfloat16*>(k_raw);
  a.gamma = ln_gamma;
  a.beta = ln_beta;
  a.eps = ln_eps;
  a.fp8 = fp8 ? 1 : 0;
  a.key_cache = key_cache;
  a.key_scale = key_scale;
  a.k_bs = k_batch_stride;
  a.s_bs = fp8 ? scale_batch_stride : 0;
  a.kv_bs = kv_batch_stride;
  a.kv_raw = static_cast<const __nv_bfloat16*>(kv_raw);
  a.kv_cache = static_cast<__nv_bfloat16*>(kv_cache);
  a.pos = pos;
  a.T = T;
  a.d_I = d_I;
  a.N = N;
  a.log2_base = std::log2(static_cast<double>(rope_base));
  a.q = static_cast<__nv_bfloat16*>(q);
  a.q_pos = q_pos;
  a.B = q ? B : 0;
  a.H = q ? H : 0;
  a.status = static_cast<int*>(workspace);
  if (ic::launch_cache_append(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return IC_ERR_CUDA;
  g_launches = 1;
  return IC_OK;
}

size_t ic_decompress_gate_workspace_size(void) { return kStatusBytes; }

ic_status_t ic_decompress_gate(const void* o_latent, const void* wv_b, const void* gate, int B, int H, int d_v,
                               ic_dtype_t out_dtype, void* out, void* workspace, size_t ws_bytes,
                               ic_stream_t stream) {
  g_launches = 0;
  if (!workspace || ws_bytes < kStatusBytes || !aligned16(workspace)) return IC_ERR_INVALID_ARG;
  if (!o_latent || !wv_b || !out || B < 1 || H < 1) return IC_ERR_INVALID_ARG;
  if (d_v != 128) return IC_ERR_UNSUPPORTED;
  if (out_dtype != IC_BF16 && out_dtype != IC_F32) return IC_ERR_UNSUPPORTED;
  if (!aligned16(o_latent) || !aligned16(wv_b) || !aligned16(out) || (gate && !aligned16(gate)))
    return IC_ERR_INVALID_ARG;
  if (ceil_div<int64_t>(B, 128) * H >= (int64_t(1) << 31)) return IC_ERR_INVALID_ARG;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return IC_ERR_CUDA;
  const cuuint32_t estr[3] = {1, 1, 1};
  // wv_b (512, d_v, H): one box = 64 latent dims of a head's 128 weight rows
  CUtensorMap wmap;
  const cuuint64_t wdims[3] = {512, static_cast<cuuint64_t>(d_v), static_cast<cuuint64_t>(H)};
  const cuuint64_t wstrides[2] = {512 * 2, static_cast<cuuint64_t>(d_v) * 512 * 2};
  const cuuint32_t wbox[3] = {64, 128, 1};
  CUresult r = enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(wv_b), wdims, wstrides, wbox,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return IC_ERR_INVALID_ARG;
  // latent outputs (512, H, B): one box = 64 latent dims of one head for 128
  // queries (queries past B read as zeros)
  CUtensorMap omap;
  const cuuint64_t odims[3] = {512, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  const cuuint64_t ostrides[2] = {512 * 2, static_cast<cuuint64_t>(H) * 512 * 2};
  const cuuint32_t obox[3] = {64, 1, 128};
  r = enc(&omap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(o_latent), odims, ostrides, obox, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return IC_ERR_INVALID_ARG;
  ic::GateArgs a{};
  a.gate = static_cast<const __nv_bfloat16*>(gate);
  a.out = out;
  a.out_f32 = out_dtype == IC_F32 ? 1 : 0;
  a.B = B;
  a.H = H;
  a.status = static_cast<int*>(workspace);
  a.wait_ns = ic::wait_limit_ns();
  if (ic::launch_gate(wmap, omap, a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return IC_ERR_CUDA;
  g_launches = 1;
  return IC_OK;
}

size_t ic_cp_workspace_size(void) { return kStatusBytes; }

ic_status_t ic_cp_candidates(const float* scores, const int32_t* idx, int B, int64_t N_local, int k,
                             int64_t offset, float* cand_score, int32_t* cand_idx, void* workspace, size_t ws_bytes,
                             ic_stream_t stream) {
  g_launches = 0;
  if (!workspace || ws_bytes < kStatusBytes || !aligned16(workspace)) return IC_ERR_INVALID_ARG;
  if (!scores || !idx || !cand_score || !cand_idx) return IC_ERR_INVALID_ARG;
  if (B < 1 || k < 1 || N_local < 1 || offset < 0 || offset + N_local >= (int64_t(1) << 31)) return IC_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * k >= (int64_t(1) << 31)) return IC_ERR_INVALID_ARG;
  ic::CpCandArgs a{};
  a.scores = scores;
  a.idx = idx;
  a.B = B;
  a.k = k;
  a.N_local = N_local;
  a.offset = offset;
  a.cand_score = cand_score;
  a.cand_idx = cand_idx;
  a.status = static_cast<int*>(workspace);
  if (ic::launch_cp_candidates(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return IC_ERR_CUDA;
  g_launches = 1;
  return IC_OK;
}

ic_status_t ic_cp_merge_topk(const float* cand_score, const int32_t* cand_idx, int64_t seg_stride, int G, int B,
                             int kin, int k, int64_t lo, int64_t hi, int32_t* idx_global, int32_t* idx_local,
                             ic_stream_t stream) {
  g_launches = 0;
  if (!cand_score || !cand_idx || !idx_global) return IC_ERR_INVALID_ARG;
  if (G < 1 || B < 1 || kin < 1 || k < 1 || lo < 0 || hi < lo || hi >= (int64_t(1) << 31)) return IC_ERR_INVALID_ARG;
  if (G > 1 && seg_stride < static_cast<int64_t>(B) * kin) return IC_ERR_INVALID_ARG;
  if (static_cast<int64_t>(G) * kin > ic::kCpMaxCand) return IC_ERR_UNSUPPORTED;
  ic::CpMergeArgs a{};
  a.cand_score = cand_score;
  a.cand_idx = cand_idx;
  a.seg_stride = seg_stride;
  a.G = G;
  a.B = B;
  a.kin = kin;
  a.k = k;
  a.lo = lo;
  a.hi = hi;
  a.idx_global = idx_global;
  a.idx_local = idx_local;
  if (ic::launch_cp_merge_topk(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return IC_ERR_CUDA;
  g_launches = 1;
  return IC_OK;
}

ic_status_t ic_cp_combine(const float* part_out, int64_t out_stride, const float* part_lse, int64_t lse_stride, int G,
                          int B, int H, const float* sink, const void* gate, ic_dtype_t out_dtype, void* out,
                          float* lse, ic_stream_t stream) {
  g_launches = 0;
  if (!part_out || !part_lse || !sink || !out) return IC_ERR_INVALID_ARG;
  if (G < 1 || B < 1 || H < 1) return IC_ERR_INVALID_ARG;
  if (out_dtype != IC_BF16 && out_dtype != IC_F32) return IC_ERR_UNSUPPORTED;
  if (!aligned16(part_out) || !aligned16(out) || (gate && !aligned16(gate))) return IC_ERR_INVALID_ARG;
  const int64_t rows = static_cast<int64_t>(B) * H;
  if (rows >= (int64_t(1) << 31)) return IC_ERR_INVALID_ARG;
  // every segment holds one rank's [B, H, 512] output (16-byte aligned) and [B, H] lse
  if (G > 1 && (out_stride < rows * 512 || out_stride % 4 != 0 || lse_stride < rows)) return IC_ERR_INVALID_ARG;
  ic::CpCombineArgs a{};
  a.part_out = part_out;
  a.part_lse = part_lse;
  a.out_stride = out_stride;
  a.lse_stride = lse_stride;
  a.G = G;
  a.B = B;
  a.H = H;
  a.sink = sink;
  a.gate = static_cast<const __nv_bfloat16*>(gate);
  a.out = out;
  a.out_f32 = out_dtype == IC_F32 ? 1 : 0;
  a.lse = lse;
  if (ic::launch_cp_combine(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return IC_ERR_CUDA;
  g_launches = 1;
  return IC_OK;
}

ic_status_t ic_last_device_status(void* workspace, ic_stream_t stream) {
  if (!workspace) return IC_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return IC_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return IC_ERR_CUDA;
  if (v != 0 && cudaMemset(workspace, 0, sizeof(int)) != cudaSuccess) return IC_ERR_CUDA;
  if (v == IC_ERR_TIMEOUT || v == IC_ERR_BAD_INDEX) return static_cast<ic_status_t>(v);
  return v == 0 ? IC_OK : IC_ERR_CUDA;
}

ic_status_t ic_index_overlap(const int32_t* a, const int32_t* b, int B, int k, int64_t N, int32_t* count,
                             ic_stream_t stream) {
  g_launches = 0;
  if (!a || !b || !count || B < 1 || k < 1 || N < 1) return IC_ERR_INVALID_ARG;
  if (ic::index_overlap_smem_bytes(N) > 232448 - 1024) return IC_ERR_UNSUPPORTED;
  int n = 0;
  if (ic::launch_index_overlap(a, b, B, k, N, count, reinterpret_cast<cudaStream_t>(stream), false, &n) !=
      cudaSuccess)
    return IC_ERR_CUDA;
  g_launches = n;
  return IC_OK;
}

}  // extern "C"
