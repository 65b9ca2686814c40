/*
 * indexcache.h -- C ABI of the B200 (sm_100a) IndexCache decode hot path.
 *
 * The path (Hy4 IndexCache explainer, "What is IndexCache" and narrative on
 * the ticket rail; Hy4-preview porting issue, "Indexer", sink and gate
 * bullets):
 *
 *   F layer:  scores = lightning indexer over every cached token
 *             index  = top-k(scores)            -> shared index buffer
 *   S layer:  index  = the buffer as the last preceding F layer left it
 *   every layer: out = sparse MLA attention over the indexed rows, with a
 *             per-head softmax sink and a sigmoid output gate.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, owned by the caller. The
 *     library never allocates or frees device memory, never synchronises the
 *     stream it is given (except ic_last_device_status, which says so), and
 *     launches only on that stream.
 *   - Tensors are dense row-major with the shapes stated; every pointer must
 *     be 16-byte aligned.
 *   - Argument errors are detected on the host and returned before anything
 *     is launched. A failed launch returns IC_ERR_CUDA. Errors found on the
 *     device (an index outside [-1, N), a bounded wait that gave up) are
 *     recorded in a status word at the start of the caller's workspace; read
 *     it with ic_last_device_status.
 *   - Workspaces: size them with the matching *_workspace_size call and
 *     zero a new one once before its first use (the status word must start
 *     at IC_OK). The status word keeps the first device error until
 *     ic_last_device_status reads and clears it. The top-k passes keep a few
 *     control words per row in the workspace that every completed call
 *     leaves at zero; after a call that reported a device error, zero the
 *     workspace again before reusing it. Every other byte is scratch that
 *     each call initialises itself. Calls that share a workspace must not
 *     overlap in time on the device.
 */
#ifndef INDEXCACHE_H_
#define INDEXCACHE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* ic_stream_t; /* same object as cudaStream_t; NULL = legacy default stream */

typedef enum {
  IC_OK = 0,
  IC_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or schedule */
  IC_ERR_UNSUPPORTED = 2,  /* a valid shape this build has no kernel for */
  IC_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  IC_ERR_TIMEOUT = 4,      /* device: a bounded wait inside a kernel gave up */
  IC_ERR_BAD_INDEX = 5     /* device: an index outside [-1, N) was read (it was treated as -1) */
} ic_status_t;

typedef enum { IC_BF16 = 0, IC_FP8_E4M3 = 1, IC_F32 = 2 } ic_dtype_t;

/* Human-readable name of a status code (static storage). */
const char* ic_status_string(ic_status_t s);

/* ---------------------------------------------------------------------------
 * ic_indexer_score -- the lightning indexer.
 *
 * Defines (Hy4 IndexCache explainer, Jargon "Indexer": a cheap pass that
 * scores every cached position; the score form is DeepSeek's lightning
 * indexer):
 *     scores[b, s] = sum_h w[b,h] * max(0, sum_d q[b,h,d] * k_b[s,d])
 * for s < n_valid[b]; scores[b, s] = -inf for n_valid[b] <= s < N.
 *
 *   q        [B, H_I, d_I] bf16.
 *   w        [B, H_I] fp32 head weights of each query.
 *   k        key cache of query b at k + b*k_batch_stride elements, [N, d_I],
 *            bf16 (k_dtype IC_BF16) or e4m3 codes (IC_FP8_E4M3).
 *            k_batch_stride = 0: one cache shared by all B queries.
 *   k_scale  fp32 per-token scale, e4m3 keys only (NULL otherwise): the key
 *            of token s is decode(code[s,:]) * k_scale[s]; query b's scales
 *            at k_scale + b*scale_batch_stride. Scales must be >= 0.
 *   n_valid  int64 [B] causal limits (device), or NULL: every s < N valid.
 *   scores   [B, N] fp32 output, row stride N.
 *   Supported: d_I in {64, 128}; 1 <= H_I <= 128; N >= 1; B >= 1.
 *   workspace >= ic_indexer_workspace_size() bytes (holds the status word).
 *   Arithmetic: the products of q and the (decoded) keys, summed in fp32.
 *   With e4m3 keys and d_I = 128 each query head is split into two e4m3
 *   parts with a power-of-two scale, exact except that elements smaller than
 *   2^-9 of the head's largest |q| carry an error of at most 2^-17 of it;
 *   with e4m3 keys and d_I = 64 the queries are taken as f16 (|q| < 65504).
 * ------------------------------------------------------------------------- */
ic_status_t ic_indexer_score(const void* q, const float* w, const void* k, const float* k_scale,
                             ic_dtype_t k_dtype, int B, int H_I, int d_I, int64_t N,
                             int64_t k_batch_stride, int64_t scale_batch_stride,
                             const int64_t* n_valid, float* scores, void* workspace,
                             size_t ws_bytes, ic_stream_t stream);
size_t ic_indexer_workspace_size(void);

/* ---------------------------------------------------------------------------
 * ic_topk -- top-k selection (Hy4 IndexCache explainer, Jargon "Top-k
 * selection"; k = 2048 at model shape per the Hy4-preview porting issue).
 *
 * For each row b, writes to idx[b, :] the token indices of the k largest
 * scores[b, s] over s < n_valid[b] (all N when n_valid is NULL). Ties at the
 * k-th value are resolved toward the lower index. The order of the indices
 * within a row is unspecified. When fewer than k positions compete, they
 * are all written and the row is padded with -1.
 *   scores [B, N] fp32 (row stride N); idx [B, k] int32.
 *   Supported: 1 <= k <= 16384, N < 2^31.
 * ------------------------------------------------------------------------- */
ic_status_t ic_topk(const float* scores, int B, int64_t N, const int64_t* n_valid, int k,
                    int32_t* idx, void* workspace, size_t ws_bytes, ic_stream_t stream);
size_t ic_topk_workspace_size(int B, int64_t N, int k);

/* ---------------------------------------------------------------------------
 * ic_indexer_topk -- the indexer and the top-k of an F layer in one call
 * (Hy4 IndexCache explainer, Jargon "Indexer" and "Top-k selection": the
 * indexer's scores exist only to pick the k best tokens). Writes idx [B, k]
 * exactly as ic_indexer_score followed by ic_topk would; the scores never
 * leave the workspace, whose score scratch holds rows_per_pass rows at a
 * time: the rows are scored and selected in passes of that many rows
 * (rounded up to a multiple of 8; 0 = all B rows in one pass), so a long
 * prefill chunk needs rows_per_pass * N * 4 bytes of scores, not B * N * 4.
 * Arguments as for ic_indexer_score and ic_topk; the workspace must hold
 * ic_indexer_topk_workspace_size(B, N, k, rows_per_pass) bytes and follows
 * the workspace rules above (zeroed once before first use).
 * ------------------------------------------------------------------------- */
ic_status_t ic_indexer_topk(const void* q, const float* w, const void* k, const float* k_scale,
                            ic_dtype_t k_dtype, int B, int H_I, int d_I, int64_t N, int64_t k_batch_stride,
                            int64_t scale_batch_stride, const int64_t* n_valid, int topk, int rows_per_pass,
                            int32_t* idx, void* workspace, size_t ws_bytes, ic_stream_t stream);
size_t ic_indexer_topk_workspace_size(int B, int64_t N, int k, int rows_per_pass);

/* ---------------------------------------------------------------------------
 * ic_topk_noalloc -- ic_topk for callers that cannot allocate device memory.
 * The pages have no counterpart: this is an interface choice of the library.
 *
 * Same result and limits as ic_topk, but takes no workspace: its scratch is
 * a fixed array inside the library (12 MB on every GPU that loads it, held
 * until exit). Meant for code that cannot call cudaMalloc, e.g.
 * enqueueing inside a CUDA-graph capture that forbids allocation, or engine
 * plugins that only receive their input and output buffers.
 *   - At most IC_TOPK_NOALLOC_MAX_ROWS rows, and the per-row histograms and
 *     candidate buffers must fit the array (64 rows of up to 131072 scores
 *     do); otherwise IC_ERR_UNSUPPORTED with nothing launched.
 *   - All calls share the one array; calls that overlap on the GPU race.
 *   - The first call on a device looks up the array's address; make it
 *     before any stream capture. Device-side status is not reported.
 * ------------------------------------------------------------------------- */
#define IC_TOPK_NOALLOC_MAX_ROWS 64
ic_status_t ic_topk_noalloc(const float* scores, int B, int64_t N, const int64_t* n_valid, int k,
                            int32_t* idx, ic_stream_t stream);

/* ---------------------------------------------------------------------------
 * ic_sparse_mla_decode -- DSA token-level sparse attention, MLA shape,
 * with a per-head sink and a sigmoid output gate (Hy4 IndexCache explainer,
 * Jargon "DSA"; Hy4-preview porting issue: head 576 = 512 latent + 64 RoPE,
 * "learnable per-head sink (softmax-denominator bias)", "elementwise sigmoid
 * gate").
 *
 * For query b, head h, selected tokens j (idx[b,j] in [0, N)):
 *     z_j = sm_scale * sum_{d<576} q[b,h,d] * kv_b[idx_j, d]
 *     o   = sum_j exp(z_j) kv_b[idx_j, 0:512] / (exp(sink[h]) + sum_j exp(z_j))
 *     out[b,h,:] = sigmoid(gate[b,h,:]) * o     (gate NULL: out = o)
 *     lse[b,h]   = log(exp(sink[h]) + sum_j exp(z_j))   (if lse != NULL)
 * Entries equal to -1 are skipped.
 *
 *   q     [B, H, 576] bf16 (RoPE already applied to dims 512..575).
 *   kv    latent cache of query b at kv + b*kv_batch_stride elements,
 *         [N, 576] bf16; kv_batch_stride = 0: one cache shared by all.
 *   idx   [B, k] int32.   sink [H] fp32 (may be -inf: no sink term; a row
 *         with no valid selected token then gets out = 0, lse = -inf).
 *   gate  [B, H, 512] bf16 or NULL.
 *   out   [B, H, 512], bf16 (out_dtype IC_BF16) or fp32 (IC_F32).
 *   lse   [B, H] fp32 natural-log sum, or NULL.
 *   Supported: any H >= 1 (heads run in blocks of 128); k >= 1;
 *   sm_scale > 0 and finite.
 * ------------------------------------------------------------------------- */
ic_status_t ic_sparse_mla_decode(const void* q, const void* kv, int64_t kv_batch_stride, int64_t N,
                                 const int32_t* idx, int k, const float* sink, const void* gate,
                                 float sm_scale, int B, int H, ic_dtype_t out_dtype, void* out,
                                 float* lse, void* workspace, size_t ws_bytes, ic_stream_t stream);
size_t ic_sparse_mla_workspace_size(int B, int H, int k);

/* ---------------------------------------------------------------------------
 * ic_layer_stack -- the IndexCache decode step over L layers.
 *
 * Layer l with schedule[l] == 'F' runs ic_indexer_topk (the indexer and the
 * top-k) and overwrites index_buf; with 'S' it leaves index_buf as the last preceding
 * F layer wrote it (Hy4-preview porting issue, "Indexer" bullet: shared
 * layers reuse the last preceding full layer's top-k). Every layer then runs
 * ic_sparse_mla_decode reading index_buf in place. schedule[0] must be 'F'.
 *
 *   layers     [L] host array of per-layer device pointers (ic_layer_t).
 *              On S layers q_idx, w, k_idx and k_scale are ignored.
 *   schedule   host string of L characters from {'F','S'}.
 *   shape      host struct of sizes shared by every layer.
 *   index_buf  [B, topk] int32 device buffer, owned by the caller.
 *   idx_trace  optional [L, B, topk] int32 device buffer: if not NULL, the
 *              index buffer each layer attended over is copied there.
 *
 * Streaming inputs (no counterpart in the pages): a layer's wait_event, if
 * not NULL, is a cudaEvent_t (cast to void*) owned by the caller; the call
 * makes `stream` wait on it (cudaStreamWaitEvent) before the layer's first
 * kernel. A caller that uploads each layer's queries and gates on a copy
 * stream and records one event per layer lets layer l run while later
 * layers' inputs are still in flight. A failed wait returns IC_ERR_CUDA
 * (earlier layers stay enqueued).
 * ------------------------------------------------------------------------- */
typedef struct {
  int B;                       /* queries */
  int64_t N;                   /* cached tokens */
  int H_I, d_I;                /* indexer heads and dim */
  ic_dtype_t k_dtype;          /* IC_BF16 or IC_FP8_E4M3 */
  int topk;                    /* k */
  int H;                       /* attention heads */
  float sm_scale;              /* softmax scale of the 576-d logits */
  ic_dtype_t out_dtype;        /* IC_BF16 or IC_F32 */
  int64_t k_batch_stride;      /* elements between queries' key caches (0 = shared) */
  int64_t scale_batch_stride;  /* elements between queries' key scales (0 = shared) */
  int64_t kv_batch_stride;     /* elements between queries' latent caches (0 = shared) */
  const int64_t* n_valid;      /* device [B] causal limits, or NULL */
  int rows_per_pass;           /* F layers score and select this many rows at a time
                                  (ic_indexer_topk); 0 = all B rows at once */
} ic_stack_shape_t;

typedef struct {
  const void* q_idx;     /* [B, H_I, d_I] bf16 (F layers) */
  const float* w;        /* [B, H_I] fp32 (F layers) */
  const void* k_idx;     /* indexer key cache (F layers) */
  const float* k_scale;  /* e4m3 key scales or NULL (F layers) */
  const void* q;         /* [B, H, 576] bf16 */
  const void* kv;        /* latent cache */
  const float* sink;     /* [H] fp32 */
  const void* gate;      /* [B, H, 512] bf16 or NULL */
  void* out;             /* [B, H, 512] out_dtype */
  float* lse;            /* [B, H] fp32 or NULL */
  void* wait_event;      /* cudaEvent_t to wait on before the layer, or NULL */
} ic_layer_t;

ic_status_t ic_layer_stack(const ic_layer_t* layers, int L, const char* schedule,
                           const ic_stack_shape_t* shape, int32_t* index_buf, int32_t* idx_trace,
                           void* workspace, size_t ws_bytes, ic_stream_t stream);
size_t ic_layer_stack_workspace_size(const ic_stack_shape_t* shape);

/* ---------------------------------------------------------------------------
 * ic_cache_append -- the cache-append step for T new tokens, run before the
 * decode step (Hy4-preview porting issue: "Indexer" bullet, the indexer key
 * goes through a LayerNorm with bias; "RoPE is interleaved" bullet,
 * is_neox_style=False: adjacent pairs of the 64 rotary dims rotate).
 *
 * Token t writes row r = pos[t] of cache c (c = t where a batch stride is
 * nonzero, the single shared cache where it is 0):
 *   y = (k_raw[t] - mean) / sqrt(var + ln_eps) * ln_gamma + ln_beta
 *       (mean and population variance over the d_I dims)
 *   k_dtype IC_BF16:     key row = bf16(y)  (round to nearest even)
 *   k_dtype IC_FP8_E4M3: key_scale[r] = max|y| / 448 (1 if y is all zero),
 *                        key row = e4m3(y / key_scale[r]), round to nearest
 *                        even, saturating at +-448
 *   kv row  = kv_raw[t] with each rotary pair i < 32 of dims [512, 576)
 *             (a, b) = (x[512+2i], x[513+2i]) -> (a cos - b sin, a sin + b cos),
 *             angle = r * rope_base^(-2i/64), result rounded to bf16
 * If q is not NULL, the rotary dims of every head of query b < B are
 * rotated the same way in place by the angle of position q_pos[b].
 *
 *   k_raw      [T, d_I] bf16.  ln_gamma, ln_beta [d_I] fp32.
 *   key_cache  [N, d_I] bf16 or e4m3 bytes per cache, caches k_batch_stride
 *              elements apart; key_scale [N] fp32 per cache,
 *              scale_batch_stride apart (e4m3 only; NULL for bf16).
 *   kv_raw     [T, 576] bf16.  kv_cache [N, 576] bf16 per cache,
 *              kv_batch_stride elements apart.
 *   pos        [T] int64 device.  A row outside [0, N) is not written and
 *              the status word records IC_ERR_BAD_INDEX.
 *   q          [B, H, 576] bf16 or NULL.  q_pos [B] int64 device.
 *   Supported: T >= 1, N >= 1, d_I in {64, 128}; ln_eps >= 0 and
 *   rope_base > 0, both finite. Pointers 16-byte aligned. Two tokens of one
 *   call must not write the same row. The caller owns every buffer.
 *   workspace >= ic_cache_append_workspace_size() bytes (status word).
 * ------------------------------------------------------------------------- */
ic_status_t ic_cache_append(const void* k_raw, const float* ln_gamma, const float* ln_beta, float ln_eps,
                            ic_dtype_t k_dtype, void* key_cache, float* key_scale, int64_t k_batch_stride,
                            int64_t scale_batch_stride, const void* kv_raw, void* kv_cache,
                            int64_t kv_batch_stride, const int64_t* pos, int T, int d_I, int64_t N,
                            float rope_base, void* q, const int64_t* q_pos, int B, int H, void* workspace,
                            size_t ws_bytes, ic_stream_t stream);
size_t ic_cache_append_workspace_size(void);

/* ---------------------------------------------------------------------------
 * ic_decompress_gate -- the output gate in the decompressed space
 * (Hy4-preview porting issue, gate bullet: the elementwise sigmoid gate
 * multiplies the decompressed per-head attention output, after the value
 * up-projection wv_b and before o_proj).
 *
 *   v[b,h,:]   = wv_b[h] @ o_latent[b,h,:]      (512 -> d_v per head)
 *   out[b,h,:] = sigmoid(gate[b,h,:]) * v[b,h,:]   (gate NULL: out = v)
 *
 *   o_latent  [B, H, 512] bf16: the ungated sparse-attention output
 *             (ic_sparse_mla_decode with gate NULL and out_dtype IC_BF16).
 *   wv_b      [H, d_v, 512] bf16 (out x in per head).
 *   gate      [B, H, d_v] bf16 gate logits, or NULL.
 *   out       [B, H, d_v], bf16 (IC_BF16) or fp32 (IC_F32).
 *   Supported: d_v = 128; B, H >= 1. Pointers 16-byte aligned.
 *   workspace >= ic_decompress_gate_workspace_size() bytes (status word).
 * ------------------------------------------------------------------------- */
ic_status_t ic_decompress_gate(const void* o_latent, const void* wv_b, const void* gate, int B, int H, int d_v,
                               ic_dtype_t out_dtype, void* out, void* workspace, size_t ws_bytes,
                               ic_stream_t stream);
size_t ic_decompress_gate_workspace_size(void);

/* ---------------------------------------------------------------------------
 * Context-parallel decode: the N cached tokens split over G ranks, rank r
 * holding the contiguous shard [lo_r, hi_r) of the positions (Hy4 IndexCache
 * explainer, TL;DR and Jargon "Sparse attention": the indexer scores the
 * whole cached past, which is what grows with a 1M-token context). The
 * exchanges between the ranks are collectives the caller issues (NCCL); the
 * library provides the steps around them. Per F layer and rank:
 *   1. ic_indexer_score and ic_topk over the shard (local positions);
 *   2. ic_cp_candidates: (score, global position) of each local top-k entry;
 *   3. all-gather of the candidates over the ranks -> [B, G*k];
 *   4. ic_cp_merge_topk: the global top-k (every rank gets the same set: the
 *      k best of a row are among the k best of their own shard), and the
 *      row's positions inside this rank's shard;
 * and per layer:
 *   5. ic_sparse_mla_decode over the local positions with the sink -inf
 *      (no sink term), gate NULL, fp32 output and lse;
 *   6. all-gather of the partial outputs and lse over the ranks;
 *   7. ic_cp_combine: out = sum_r e^{lse_r} o_r / (e^{sink} + sum_r e^{lse_r}),
 *      then the gate -- the single-GPU result up to rounding.
 *
 * ic_cp_candidates
 *   scores [B, N_local] fp32 (the shard's scores), idx [B, k] int32 (shard
 *   positions or -1). Writes cand_score [B, k] (the score, -inf for -1) and
 *   cand_idx [B, k] (offset + position, -1 for -1). A position outside
 *   [-1, N_local) is treated as -1 and recorded as IC_ERR_BAD_INDEX in the
 *   workspace's status word (>= ic_cp_workspace_size() bytes).
 *
 * ic_cp_merge_topk
 *   Candidates of G segments (one per rank, as an all-gather lays them
 *   out), segment g at cand_score + g*seg_stride and cand_idx +
 *   g*seg_stride, each [B, kin]; G*kin <= 16384. Writes to idx_global
 *   [B, k] the global positions of the k candidates with the highest
 *   scores, ties toward the lower global position (the single-GPU tie rule),
 *   -1 padding when a row has fewer than k candidates with a position; and,
 *   if idx_local is not NULL, idx_local[b, j] = idx_global - lo when that
 *   lies in [lo, hi), else -1. Order within a row is unspecified (the same
 *   on every rank). G*kin > 16384: IC_ERR_UNSUPPORTED.
 *
 * ic_cp_combine
 *   Rank r's normalised output [B, H, 512] fp32 at part_out + r*out_stride
 *   and natural-log sum [B, H] fp32 at part_lse + r*lse_stride (-inf: no
 *   row), from step 5; when G > 1, out_stride a multiple of 4 and
 *   >= B*H*512, lse_stride >= B*H. sink [H], gate [B, H, 512] bf16 or NULL. Writes out [B, H, 512]
 *   (bf16 or fp32) and, if not NULL, lse [B, H] (log of the whole
 *   denominator).
 * ------------------------------------------------------------------------- */
ic_status_t ic_cp_candidates(const float* scores, const int32_t* idx, int B, int64_t N_local, int k,
                             int64_t offset, float* cand_score, int32_t* cand_idx, void* workspace,
                             size_t ws_bytes, ic_stream_t stream);
size_t ic_cp_workspace_size(void);
ic_status_t ic_cp_merge_topk(const float* cand_score, const int32_t* cand_idx, int64_t seg_stride, int G, int B,
                             int kin, int k, int64_t lo, int64_t hi, int32_t* idx_global, int32_t* idx_local,
                             ic_stream_t stream);
ic_status_t ic_cp_combine(const float* part_out, int64_t out_stride, const float* part_lse, int64_t lse_stride, int G,
                          int B, int H, const float* sink, const void* gate, ic_dtype_t out_dtype, void* out,
                          float* lse, ic_stream_t stream);

/* ---------------------------------------------------------------------------
 * ic_index_overlap -- per-row overlap of two index sets: the reuse diagnostic
 * of the layer stack (Hy4 IndexCache explainer: reuse is free only where
 * nearby layers want the same tokens -- the bet that sparse selections are
 * largely shared between nearby layers; Bai et al. record: cross-layer reuse
 * is not exact equality to each layer's own selection). With a = the index
 * an S layer reuses and b = the top-k it would compute itself, count / k is
 * the recall of the reused index.
 *
 *   a, b   [B, k] int32, device; entries outside [0, N) (the -1 padding)
 *          are ignored. A row of b is expected to hold distinct indices
 *          (as every top-k output does): a repeated entry is counted again.
 *   count  [B] int32, device: count[r] = number of valid b[r, :] entries
 *          that occur in a[r, :].
 *   N      1 <= N <= 1,851,392 (one bit per position in shared memory);
 *          larger N: IC_ERR_UNSUPPORTED.
 * One kernel launch on `stream`, no workspace.
 * ------------------------------------------------------------------------- */
ic_status_t ic_index_overlap(const int32_t* a, const int32_t* b, int B, int k, int64_t N, int32_t* count,
                             ic_stream_t stream);

/* ---------------------------------------------------------------------------
 * ic_last_device_status -- synchronises `stream`, then reads and clears the
 * device status word at the start of `workspace` (any of the workspaces
 * above). Returns IC_OK, IC_ERR_TIMEOUT or IC_ERR_BAD_INDEX (or IC_ERR_CUDA
 * if the synchronisation itself failed).
 * ------------------------------------------------------------------------- */
ic_status_t ic_last_device_status(void* workspace, ic_stream_t stream);

/* Number of kernels the last successful call on this host thread enqueued
 * (for launch accounting in benchmarks). */
int ic_last_launch_count(void);

/* ---------------------------------------------------------------------------
 * ic_set_wait_limit_ns / ic_wait_limit_ns -- bound of the waits inside the
 * kernels (no counterpart in the pages; part of the failure handling).
 *
 * Every wait a kernel makes on a copy, an MMA or another warp of its CTA
 * gives up after this many nanoseconds: the kernel then records
 * IC_ERR_TIMEOUT in the status word, writes no further output, lets its own
 * copies and MMAs in flight finish (each of those waits bounded by 2 s) and
 * frees its tensor memory before returning, so the context stays usable.
 * The default is 2 s. The value is process-wide and read when a call
 * enqueues its kernels (calls already enqueued keep theirs). 0 makes every
 * wait that is not already satisfied when first tested give up at once:
 * meant for tests of the failure path; outputs of such calls are undefined.
 * ------------------------------------------------------------------------- */
void ic_set_wait_limit_ns(uint64_t ns);
uint64_t ic_wait_limit_ns(void);

#ifdef __cplusplus
}
#endif
#endif /* INDEXCACHE_H_ */
