// Decompressed-space output gate on sm_100a tensor cores.
//
//   v[b, h, :]   = wv_b[h] @ o[b, h, :]          wv_b [H, 128, 512], o [B, H, 512]
//   out[b, h, :] = sigmoid(g[b, h, :]) * v[b, h, :]
//
// (Hy4-preview porting issue, gate bullet: the sigmoid gate multiplies the
// decompressed per-head attention output, after the value up-projection and
// before o_proj.)
//
// Mapping. One CTA per (head, tile of up to 128 queries):
//   D[128 value dims x n] = W_h[128 x 512] . O_h[n x 512]^T,  n = queries
// rounded up to 16, K = 512 in 8 slices of 64. The weights are the A (M)
// side, so each TMEM lane holds one value dim of every query in the tile and
// the epilogue thread owning it gates and stores consecutive dims (coalesced
// rows of out). At decode the 16.8 MB of weights per layer (H = 128) are the
// bytes that matter: every CTA streams its head's 128 KB once per query tile
// through a four-slice TMA ring, so the kernel is HBM-bound.
//
// Warp roles: 0 TMA producer, 1 TMEM owner and MMA issuer, 2..5 epilogue
// (one per TMEM lane quadrant). Every wait is bounded; on expiry the status
// word records IC_ERR_TIMEOUT, the epilogue writes nothing, copies in flight
// land before the CTA exits and TMEM is freed after the last MMA completes.
#include "common.cuh"
#include "kernels.h"

namespace ic {

namespace {

constexpr int kDv = 128;                  // value dims per head (MMA M)
constexpr int kDl = 512;                  // latent dims (K)
constexpr int kSlices = kDl / 64;         // 64-dim K slices
constexpr int kStages = 4;
constexpr int kSliceBytes = 128 * 128;    // 128 rows x 128 bytes
constexpr int kStageBytes = 2 * kSliceBytes;  // weight slice + query slice
constexpr int kTileQ = 128;               // queries per CTA (MMA N at most)
constexpr int kThreads = 192;
constexpr int kSmemBytes = kStages * kStageBytes + 256 + 1024;  // + barriers, alignment slack

__global__ void __launch_bounds__(kThreads, 1)
    gate_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap omap,
                const GateArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* full = bars;                // [kStages] slice landed
  uint64_t* empty = full + kStages;     // [kStages] slice consumed by the MMAs
  uint64_t* acc_full = empty + kStages; // every MMA of the tile completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = static_cast<int>(blockIdx.x % a.H);
  const int q0 = static_cast<int>(blockIdx.x / a.H) * kTileQ;
  const int nq = a.B - q0 < kTileQ ? a.B - q0 : kTileQ;
  const int n_mma = (nq + 15) & ~15;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&wmap);
    tma_prefetch_desc(&omap);
  }
  pdl_wait();  // the latent outputs come from the attention kernel
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTileQ);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      for (; s < kSlices; ++s) {
        const int st = s % kStages;
        const uint32_t ph = static_cast<uint32_t>((s / kStages) & 1);
        if (!mbar_wait(&empty[st], ph ^ 1, abort_flag, a.status, a.wait_ns)) break;
        mbar_arrive_expect_tx(&full[st], kStageBytes);
        uint8_t* base = stages + st * kStageBytes;
        tma_load_3d(base, &wmap, &full[st], s * 64, 0, h);                // W_h rows, dims [64 s, 64 s + 64)
        tma_load_3d(base + kSliceBytes, &omap, &full[st], s * 64, h, q0);  // query rows (past B: zeros)
      }
      // every copy this thread issued lands before the CTA can exit
      for (int j = (s > kStages ? s - kStages : 0); j < s; ++j)
        mbar_drain(&full[j % kStages], static_cast<uint32_t>((j / kStages) & 1));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kDv, n_mma, false, false);
      for (int s = 0; s < kSlices; ++s) {
        const int st = s % kStages;
        if (!mbar_wait(&full[st], static_cast<uint32_t>((s / kStages) & 1), abort_flag, a.status, a.wait_ns)) break;
        tc_fence_after();
        const uint32_t wa = smem_u32(stages + st * kStageBytes);
        const uint32_t ob = wa + kSliceBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(tmem_base, sw128_desc(wa + kk * 32, 16, 1024), sw128_desc(ob + kk * 32, 16, 1024), idesc,
                      (s > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[st]);
      }
      mma_commit(acc_full);  // arrives once every MMA issued above has completed
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    const int d = quad * 32 + lane;
    // The gate logits of this thread's value dim for every query of the
    // tile, requested before the accumulator wait so that their latency
    // overlaps the MMAs (one round trip instead of one per query).
    __nv_bfloat16 gl[kTileQ];
#pragma unroll
    for (int j = 0; j < kTileQ; ++j) {
      gl[j] = __float2bfloat16_rn(0.f);
      if (a.gate && j < nq) gl[j] = __ldg(a.gate + (static_cast<int64_t>(q0 + j) * a.H + h) * kDv + d);
    }
    bool got = mbar_wait(acc_full, 0u, abort_flag, a.status, a.wait_ns);
    __syncwarp();  // tcgen05.ld below is warp-collective
    got = got && !*abort_flag;
    got = __all_sync(0xffffffffu, got);
    if (got) {
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
#pragma unroll
      for (int c0 = 0; c0 < kTileQ; c0 += 32) {
        if (c0 < n_mma) {
          uint32_t r[32];
          tmem_ld32_issue(taddr + c0, r);  // columns past n_mma are allocated and ignored
          tmem_ld_wait(r);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (c0 + j < nq) {
              const int64_t o = (static_cast<int64_t>(q0 + c0 + j) * a.H + h) * kDv + d;
              float v = __uint_as_float(r[j]);
              if (a.gate) v *= 1.f / (1.f + __expf(-__bfloat162float(gl[c0 + j])));
              if (a.out_f32)
                static_cast<float*>(a.out)[o] = v;
              else
                static_cast<__nv_bfloat16*>(a.out)[o] = __float2bfloat16_rn(v);
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // every MMA issued has completed before its accumulator is freed (the
    // issuer commits acc_full on every path, including after an abort)
    if (lane == 0) mbar_drain(acc_full, 0u);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTileQ);
  }
}

}  // namespace

int gate_smem_bytes() { return kSmemBytes; }

cudaError_t launch_gate(const CUtensorMap& wmap, const CUtensorMap& omap, const GateArgs& a, cudaStream_t stream) {
  static bool done[64] = {false};  // per device
  cudaError_t e = set_smem_once(gate_kernel, kSmemBytes, done);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (a.B + kTileQ - 1) / kTileQ;
  gate_kernel<<<static_cast<unsigned>(tiles * a.H), kThreads, kSmemBytes, stream>>>(wmap, omap, a);
  return cudaGetLastError();
}

}  // namespace ic
