// ic_topk_noalloc: the top-k passes of ic_topk, with their scratch in a
// fixed array that ships inside this library instead of a caller workspace.
//
// Who needs this. ic_topk asks the caller for a workspace (radix histograms,
// per-CTA tie counts, counters). Some callers have no way to provide one:
//   - code that enqueues work while a CUDA graph is being captured in a mode
//     that forbids cudaMalloc (allocation is not a stream operation, so a
//     capture refuses it), and that had no chance to allocate beforehand;
//   - plugins of inference engines that plan all device memory ahead of time
//     and hand a plugin only its input and output buffers;
//   - runtimes that forbid allocation after start-up for latency or
//     fragmentation reasons.
// For them this entry point allocates nothing: it needs only the scores and
// the output index buffer. Its scratch is g_topk_scratch below, a
// __device__ array that every GPU which loads this library holds until the
// process exits (kScratchBytes, 12 MB).
//
// Limits. At most IC_TOPK_NOALLOC_MAX_ROWS rows per call (64), and the
// call's histograms and candidate buffers must fit the array (64 rows of up
// to 131072 scores do); larger calls return IC_ERR_UNSUPPORTED and launch
// nothing. The other limits are those of ic_topk (k <= 16384, N < 2^31).
//
// Sharing. Every call, from every stream and thread, uses the same array and
// each call starts by clearing the part it uses (including its status word).
// Two calls that overlap on the GPU -- in different streams, or in graphs
// replayed concurrently -- race on the array and produce garbage; serialise
// them. Device-side status is kept in the array and is not reported.
//
// Set-up. The first call on each device, with that device current, looks up
// the array's device address with cudaGetSymbolAddress (host code cannot use
// the symbol itself as a device pointer). Make that first call before any
// stream capture.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/indexcache.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = 12 * 1024 * 1024;
constexpr size_t kStatusBytes = 256;

static __device__ __align__(256) unsigned char g_topk_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[64] = {nullptr};

// Device address of g_topk_scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_topk_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" ic_status_t ic_topk_noalloc(const float* scores, int B, int64_t N, const int64_t* n_valid, int k,
                                       int32_t* idx, ic_stream_t stream) {
  if (!scores || !idx) return IC_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || N >= (int64_t(1) << 31) || k < 1 || k > 16384) return IC_ERR_INVALID_ARG;
  if (B > IC_TOPK_NOALLOC_MAX_ROWS) return IC_ERR_UNSUPPORTED;
  const ic::TopkLayout L = ic::topk_layout(B, N, k);
  if (kStatusBytes + L.total > kScratchBytes) return IC_ERR_UNSUPPORTED;
  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return IC_ERR_CUDA;
  uint8_t* scratch = static_cast<uint8_t*>(base);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the status word, the control words and the row histograms start at zero
  // on every call (a previous call that hit a device error may have left
  // them set)
  if (cudaMemsetAsync(scratch, 0, kStatusBytes + L.zero_bytes, s) != cudaSuccess) return IC_ERR_CUDA;
  return ic::topk_impl(scores, B, N, n_valid, k, idx, scratch + kStatusBytes, kScratchBytes - kStatusBytes,
                       reinterpret_cast<int*>(scratch), s, false);
}
