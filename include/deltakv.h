/*
 * deltakv.h -- C ABI of libdeltakv.so: the DeltaKV hot path on B200 (sm_100a).
 *
 * DeltaKV ("DeltaKV: Residual-Based KV Cache Compression via Long-Range Similarity", Hao, Huang,
 * Wang, Zhang, Yu; summaries on gist.science) stores a long-context KV cache as a strided set of
 * full "reference" tokens plus, for every other token, a low-rank code of its residual against its
 * most similar earlier reference (summary (en) §3 "Methodology": Strided Reference Selection,
 * Residual Encoding, Reconstruction).  This library provides the two data-parallel steps:
 *
 *   deltakv_compress          centre K/V (remove the shared high-norm component mu), keep every R-th
 *                             token as a reference, match each other token to its most similar earlier
 *                             reference (cosine over the whole prefix), write rank-r codes + index.
 *   deltakv_decode_attention  GQA decode attention over the compressed cache, with K and V rebuilt on
 *                             the fly as mu + reference + code * basis^T and never materialised.
 *
 * Conventions (all entry points):
 *   - Every data pointer is a caller-owned DEVICE buffer unless a comment says "host".  The library
 *     allocates no device memory and never synchronises the stream, except deltakv_get_device_error.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  All work is
 *     enqueued on it; calls return as soon as the launches are enqueued.
 *   - Invalid or unsupported arguments return a status and launch nothing.  Launch failures return
 *     DKV_ERR_CUDA (from cudaGetLastError).  Data-dependent faults that can only be seen on the device
 *     (a block id >= num_blocks, a stored reference index out of range, a length over the host bound)
 *     are not trapped: the kernel skips the offending access and records the first such event in a
 *     per-device error word that deltakv_get_device_error reads and clears.
 *   - K/V/q inputs, mu, the basis and the three cache arrays must be 16-byte aligned; the workspace must
 *     be 256-byte aligned (DKV_ERR_INVALID_ARG otherwise).
 *   - Thread safety: calls on different streams may run concurrently if they use distinct workspaces.
 *
 * Cache layout (one dkv_cache per layer; R = ref_stride = tokens per paged block):
 *   codes   [num_blocks][H_kv][R][2r]  dtype  per token: r K-code values, then r V-code values
 *   ref_idx [num_blocks][H_kv][R]      int32  reference ordinal j of each token (token t: j < ceil(t/R),
 *                                             or t/R for a reference token)
 *   refs    [num_blocks][H_kv][2][d]   dtype  centred K row then V row of the block's first token, which
 *                                             is the sequence's reference j = logical block index
 *   A block table row maps logical block b (tokens bR .. bR+R-1) to a physical block id.
 *
 * 4-bit codes (dtype DKV_BF16_Q4; the pages' 29% figure combines DeltaKV with 4-bit quantisation: summary (en)
 * §5 "Memory Efficiency").  For each token and half h (K, V) with exact code c (r values):
 *     s_h = RNE_bf16(max_i |c_i| / 7),   q_i = clamp(rint(c_i / s_h), -7, 7)  (q = 0 when s_h = 0)
 * and decode uses c'_i = s_h * q_i.  `codes` then holds, per (physical block, kv head), R*(r+4) bytes:
 *     R packed rows of r bytes (the K half's r/2 bytes, then the V half's), then R pairs of bf16 scales (K, V).
 * Inside a half, each 32-bit little-endian word holds 8 consecutive codes c_0..c_7 of two's-complement nibbles:
 * nibble k (bits 4k..4k+3, k = 0..3) holds c_{2k} and nibble k + 4 holds c_{2k+1}.
 */
#ifndef DELTAKV_H
#define DELTAKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dkv_status {
  DKV_OK = 0,
  DKV_ERR_INVALID_ARG = 1, /* null pointer, negative size, inconsistent shape                  */
  DKV_ERR_UNSUPPORTED = 2, /* valid but not built: head_dim, rank, stride, GQA ratio, too many refs */
  DKV_ERR_WORKSPACE = 3,   /* workspace smaller than the matching *_workspace query             */
  DKV_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed                                 */
  DKV_ERR_OUT_OF_BLOCKS = 5 /* the host block pool cannot supply a reservation (deltakv_pool.h)    */
} dkv_status;

/* Storage types.  DKV_BF16_Q4: K, V, q, references, basis and outputs in bf16, the residual codes as 4-bit
 * integers with one bf16 scale per token and K/V half (see "4-bit codes" below). */
typedef enum dkv_dtype { DKV_F32 = 0, DKV_BF16 = 1, DKV_BF16_Q4 = 2 } dkv_dtype;

/* Maximum references per sequence (ceil(context / R)): 524288 tokens at R = 16.  Decode keeps a softmax mass
 * per reference and query head; see deltakv_decode_attention for where it lives and the shapes whose cap is
 * lower. */
#define DKV_MAX_REFS 32768

/* Head geometry of one layer.  Supported: head_dim in {64, 128}; rank in {16, 32, 64} with
 * rank <= head_dim; ref_stride in {16, 32, 64}; num_q_heads = G * num_kv_heads with G in {1,2,4,8}
 * and G * rank <= 256; dtype DKV_F32 or DKV_BF16 (storage type of K, V, q, codes, refs, basis, out), or
 * DKV_BF16_Q4 with rank in {32, 64} (decode: G in {4, 8}, dense only).
 * Other values return DKV_ERR_UNSUPPORTED (rank 128 is a valid shape but no kernel is built for it). */
typedef struct dkv_shape {
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim; /* d */
  int32_t rank;     /* r */
  int32_t ref_stride; /* R: every R-th token is a reference; also the paged block size */
  int32_t dtype;    /* dkv_dtype */
} dkv_shape;

/* Per-layer parameters (device, read-only):
 *   mu    [H_kv][2][d] float32  shared high-norm component of K (index 0) and V (index 1)
 *   basis [H_kv][2][d][r] dtype rank-r basis B_K, B_V (orthonormal columns expected, not checked);
 *                               code = residual * B, rebuild = code * B^T                           */
typedef struct dkv_params {
  const float* mu;
  const void* basis;
} dkv_params;

/* Compressed cache of one layer (device).  See the layout above. */
typedef struct dkv_cache {
  void* codes;
  int32_t* ref_idx;
  void* refs;
  int32_t num_blocks;
} dkv_cache;

/* Human-readable name of a status (static string). */
const char* deltakv_status_string(dkv_status status);

/* Checks a shape against the supported set; DKV_OK, DKV_ERR_INVALID_ARG or DKV_ERR_UNSUPPORTED. */
dkv_status deltakv_check_shape(const dkv_shape* shape);

/* Bytes of one physical block over all kv heads (codes + ref_idx + refs); 0 for an unsupported shape.
 * Per token per kv head this is 2r*|S| + 4 + 2d*|S|/R bytes (DKV_BF16_Q4: r + 4 + 4 + 2d*2/R). */
size_t deltakv_block_bytes(const dkv_shape* shape);

/* Sizes (bytes) of the three cache arrays for `num_blocks` blocks.  Host outputs. */
dkv_status deltakv_cache_bytes(const dkv_shape* shape, int32_t num_blocks, size_t* codes_bytes,
                               size_t* ref_idx_bytes, size_t* refs_bytes);

/* Workspace needed by deltakv_compress for these host-side bounds (host output `bytes`). */
dkv_status deltakv_compress_workspace(const dkv_shape* shape, int32_t num_seqs, int64_t total_new,
                                      int32_t max_new, int32_t max_ctx, size_t* bytes);

/* Workspace needed by deltakv_decode_attention for these host-side bounds (host output `bytes`). */
dkv_status deltakv_decode_workspace(const dkv_shape* shape, int32_t num_seqs, int32_t max_ctx,
                                    size_t* bytes);

/*
 * deltakv_compress -- append new tokens of `num_seqs` sequences to the compressed cache.
 *
 * Defined by the summary (en) §3 "Methodology": Strided Reference Selection (references every R
 * tokens), Residual Encoding (z = f_c(x) - f_c(x^R) with a linear f_c(x) = x B) and §2 "Highly Shared
 * Latent Components" (the shared component mu is removed first).  Per token t of sequence s, kv head h:
 *   x~_t   = RNE_S(fp32(x_t - mu))                         (K and V halves, concatenated: 2d values)
 *   t mod R == 0:  refs[block_tables[s][t/R]][h] = x~_t;  ref_idx = t/R;  codes = 0
 *   otherwise:     j* = argmax_{j : jR < t} <x~_t, r~_j> / |r~_j|  (ties: smallest j; zero-norm ref: 0)
 *                  ref_idx = j*;  codes = RNE_S([(x~_t - r~_j*)_K B_K ; (x~_t - r~_j*)_V B_V])
 * References written by earlier calls (positions < start_pos[s]) are read from `cache`; references
 * among this call's tokens are visible to the later tokens of the same call.
 *
 *   k_new, v_new  [total_new][H_kv][d] dtype  new tokens, sequences concatenated (ragged)
 *   cu_new        [num_seqs+1] int32  prefix sums: sequence s owns rows cu_new[s] .. cu_new[s+1]-1
 *   start_pos     [num_seqs] int32    absolute position of each sequence's first new token
 *   block_tables  [num_seqs][max_blocks] int32  physical block of each logical block; every block
 *                 that holds one of the new tokens or an earlier reference must be mapped
 *   total_new, max_new, max_ctx  host-side bounds: total rows; max new tokens of one sequence;
 *                 max start_pos[s] + new tokens (so no device->host copy is needed).  max_ctx <=
 *                 DKV_MAX_REFS * R.
 *   workspace     >= deltakv_compress_workspace(shape, num_seqs, total_new, max_new, max_ctx) bytes,
 *                 256-byte aligned; contents need not be initialised and are scratch after the call.
 * Writes codes, ref_idx and refs of the new tokens only.  Floating-point: fp32 arithmetic; bf16 scores
 * come from tensor-core products of bf16 operands accumulated in fp32.
 */
dkv_status deltakv_compress(const dkv_shape* shape, const dkv_params* params, const dkv_cache* cache,
                            const void* k_new, const void* v_new, const int32_t* cu_new,
                            const int32_t* start_pos, const int32_t* block_tables, int32_t max_blocks,
                            int32_t num_seqs, int64_t total_new, int32_t max_new, int32_t max_ctx,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * deltakv_decode_attention -- one decode query per sequence and query head, over its whole cache.
 *
 * Defined by the summary (en) §3 "Reconstruction" (KV^ = f_d(z) + KV^R, f_d(z) = z B^T, plus mu) and
 * "Sparse-vLLM Integration" (tokens are rebuilt on demand inside attention, never written back).
 * For query head hq (kv head h = hq / G) of sequence s with T = context_lens[s] cached tokens:
 *   K^_t = mu_K + r~K_{ref_idx(t)} + cK_t B_K^T,  V^_t likewise
 *   out = sum_t softmax_t(scale * q.K^_t) V^_t  (rounded to dtype),  lse = log sum_t exp(scale * q.K^_t)
 * computed without forming K^ or V^: q.K^_t = q.mu_K + q.r~K_j + (q B_K).cK_t, and the V side sums
 * softmax mass per reference before one product with the reference rows.
 *
 *   q             [num_seqs][H_q][d] dtype
 *   context_lens  [num_seqs] int32, 0 <= T <= max_ctx (T = 0 gives out = 0, lse = -inf)
 *   block_tables  [num_seqs][max_blocks] int32
 *   softmax_scale <= 0 selects 1/sqrt(d)
 *   out           [num_seqs][H_q][d] dtype;  lse [num_seqs][H_q] float32 or NULL
 *   workspace     >= deltakv_decode_workspace(shape, num_seqs, max_ctx) bytes, 256-byte aligned
 *
 * The split kernel holds a mass per visible reference and query head in shared memory while it fits beside
 * the kernel's stage ring.  Past that (for example beyond 4208 references with G = 8 and r = 32, or 9200 with
 * G = 4 and r = 32), bf16 decode with r in {32, 64} keeps the masses in the workspace instead, accumulated
 * with global atomics, up to DKV_MAX_REFS.  fp32 and r = 16 (the CUDA-core split kernel), 4-bit codes, the
 * k-nearest retrieval and sparse decode keep the shared-memory cap.  Beyond a cap, this call and the matching
 * workspace query return DKV_ERR_UNSUPPORTED, before any launch.
 */
dkv_status deltakv_decode_attention(const dkv_shape* shape, const dkv_params* params,
                                    const dkv_cache* cache, const void* q, const int32_t* context_lens,
                                    const int32_t* block_tables, int32_t max_blocks, int32_t num_seqs,
                                    int32_t max_ctx, float softmax_scale, void* out, float* lse,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* Workspace needed by deltakv_decode_attention_sparse for these host-side bounds (host output `bytes`). */
dkv_status deltakv_decode_sparse_workspace(const dkv_shape* shape, int32_t num_seqs, int32_t max_ctx,
                                           int32_t max_sel, size_t* bytes);

/*
 * deltakv_decode_attention_sparse -- decode attention over a caller-given subset of each sequence's tokens.
 *
 * Defined by the summary (en) §3 "Sparse-vLLM Integration" (also summary (pt) §2 and summary (fr) §2): DeltaKV
 * is combined with a sparse attention that keeps only some tokens per step, and only those tokens are
 * reconstructed, on demand, so that memory traffic is spent on them alone.  The selection policy itself (the
 * pages use an OmniKV-style one) is the caller's; this call takes its result.  For query head hq (kv head
 * h = hq / G) of sequence s with selected positions P_s = token_idx[cu_tokens[s] .. cu_tokens[s+1]-1]:
 *   out = sum_{t in P_s} softmax_t(scale * q.K^_t) V^_t,   lse = log sum_{t in P_s} exp(scale * q.K^_t)
 * with K^_t, V^_t rebuilt as in deltakv_decode_attention (never materialised).  Only the listed tokens' codes
 * and indices are read; the reference rows are read for the whole context, since a listed token may point at
 * any earlier reference.
 *
 *   token_idx     [cu_tokens[num_seqs]] int32  positions in [0, context_lens[s]); any order (a position
 *                 listed twice counts twice).  A position outside the context is replaced by 0 and recorded
 *                 as DKV_DEVERR_BOUNDS.  May be NULL when every list is empty.
 *   cu_tokens     [num_seqs+1] int32 prefix sums of the list lengths; every length <= max_sel (host bound)
 *   other arguments as in deltakv_decode_attention; an empty list gives out = 0, lse = -inf.
 *   workspace     >= deltakv_decode_sparse_workspace(shape, num_seqs, max_ctx, max_sel) bytes, 256-aligned
 */
dkv_status deltakv_decode_attention_sparse(const dkv_shape* shape, const dkv_params* params,
                                           const dkv_cache* cache, const void* q, const int32_t* context_lens,
                                           const int32_t* block_tables, int32_t max_blocks,
                                           const int32_t* token_idx, const int32_t* cu_tokens, int32_t max_sel,
                                           int32_t num_seqs, int32_t max_ctx, float softmax_scale, void* out,
                                           float* lse, void* workspace, size_t workspace_bytes, void* stream);

/*
 * deltakv_compress_topk -- deltakv_compress with the pages' own retrieval: the k nearest references by L2
 * distance, the residual taken against their mean.
 *
 * Defined by the summary (en) §3 "Methodology" ("Strided Reference Selection": the k nearest reference tokens by
 * L2 distance; "Residual Encoding": the compressor's difference against the mean of those references) and the
 * summary (fr) §2.  Per non-reference token t of sequence s, kv head h, with x~_t as in deltakv_compress:
 *   J_t  = the k visible references (j R < t) nearest to x~_t in L2 distance on the 2d-wide [k~ ; v~], i.e.
 *          the k largest 2<x~_t, r~_j> - |r~_j|^2 (ties: the smaller j); all of them if fewer than k are visible
 *   m_t  = mean of r~_j over J_t;   codes = RNE_S([(x~_t - m_t)_K B_K ; (x~_t - m_t)_V B_V])
 * A reference token t keeps t / R in every slot and a zero code.  The cache is as for deltakv_compress except
 * `ref_idx`, which holds k slots per token: ref_idx [num_blocks][H_kv][R][k] int32, the chosen ordinals in
 * ascending order, -1 in unfilled slots.  Decode such a cache with deltakv_decode_attention_topk and the same k.
 *   k          1, 2 or 4 (others: DKV_ERR_UNSUPPORTED); dtype DKV_BF16 with rank 32 or 64
 *   other arguments and the workspace (deltakv_compress_workspace) as for deltakv_compress
 * The GPU ranks candidates by fp32 tensor-core products whose 6 lowest mantissa bits carry the column, so
 * candidates whose scores agree to about 2^-17 of their magnitude may be ranked either way.
 */
dkv_status deltakv_compress_topk(const dkv_shape* shape, int32_t k, const dkv_params* params, const dkv_cache* cache,
                                 const void* k_new, const void* v_new, const int32_t* cu_new,
                                 const int32_t* start_pos, const int32_t* block_tables, int32_t max_blocks,
                                 int32_t num_seqs, int64_t total_new, int32_t max_new, int32_t max_ctx,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* Workspace needed by deltakv_decode_attention_topk for these host-side bounds (host output `bytes`). */
dkv_status deltakv_decode_topk_workspace(const dkv_shape* shape, int32_t k, int32_t num_seqs, int32_t max_ctx,
                                         size_t* bytes);

/*
 * deltakv_decode_attention_topk -- decode attention over a cache written by deltakv_compress_topk with the same k.
 *
 * As deltakv_decode_attention, with each token rebuilt against the mean of its filled slots' references
 * (summary (en) §3 "Reconstruction"): K^_t = mu_K + mean_{j in J_t} r~K_j + cK_t B_K^T, and likewise V.  k = 1
 * is deltakv_decode_attention.  k in {2, 4}: dtype DKV_BF16, rank 32 or 64, G in {4, 8}
 * (DKV_ERR_UNSUPPORTED otherwise).  Workspace: deltakv_decode_topk_workspace with the same k.
 */
dkv_status deltakv_decode_attention_topk(const dkv_shape* shape, int32_t k, const dkv_params* params,
                                         const dkv_cache* cache, const void* q, const int32_t* context_lens,
                                         const int32_t* block_tables, int32_t max_blocks, int32_t num_seqs,
                                         int32_t max_ctx, float softmax_scale, void* out, float* lse,
                                         void* workspace, size_t workspace_bytes, void* stream);

/* Kernel ids for deltakv_profile_kernel. */
#define DKV_KERNEL_CENTER 0          /* compress: centring                                   */
#define DKV_KERNEL_REFPREP 1         /* compress: reference copy, norms, projections         */
#define DKV_KERNEL_SEARCH 2          /* compress: similarity search + codes (tensor cores)   */
#define DKV_KERNEL_DECODE_PROLOGUE 3 /* decode: q.B_K, q.mu_K, q.r~K_j                        */
#define DKV_KERNEL_DECODE_SPLIT 4    /* decode: split-K stream over the codes                */
#define DKV_KERNEL_DECODE_COMBINE 5  /* decode: merge splits, reference rows, output         */
#define DKV_NUM_KERNELS 6

/* Timing hook.  After this call, the next `n` launches of kernel `kernel_id` (in any entry point, on
 * its stream) are bracketed by cudaEventRecord(start_events[i]) / cudaEventRecord(stop_events[i]), i =
 * 0, 1, ...; later launches record nothing.  The arrays hold cudaEvent_t handles created by the caller
 * and must stay valid while recording.  n = 0 (or NULL arrays) switches the hook off for that kernel.
 * Host-global state, not thread safe; meant for benchmarks.  deltakv_profile_count returns in *n (host)
 * how many launches were recorded so far. */
dkv_status deltakv_profile_kernel(int32_t kernel_id, void* const* start_events, void* const* stop_events,
                                  int32_t n);
dkv_status deltakv_profile_count(int32_t kernel_id, int32_t* n);

/*
 * deltakv_decode_attention_noalloc -- deltakv_decode_attention without a caller-provided workspace.
 *
 * No counterpart on the DeltaKV pages: this is a library convenience.  It is meant for callers that may
 * not allocate device memory themselves, for example a plug-in running inside an inference engine
 * whose device memory is owned by that engine's own allocator, or a latency-critical serving loop in
 * which a cudaMalloc / cudaFree (which can synchronise the whole device) is not acceptable.
 *
 * Arguments, layout and results are those of deltakv_decode_attention minus `workspace` and
 * `workspace_bytes`.  The scratch memory comes from one fixed array of DKV_NOALLOC_SCRATCH_BYTES
 * (16 MiB) that lives in the library's device image: every GPU that loads the library keeps it until
 * the process exits.  Calls whose scratch need (deltakv_decode_workspace for the same shape, num_seqs
 * and max_ctx) exceeds it return DKV_ERR_WORKSPACE and launch nothing.  This entry point never calls
 * cudaMalloc, cudaFree or any other allocating routine.
 *
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with that
 *     device current and caches it; make that first call before any stream capture.  The cached address
 *     belongs to the device's primary context (the one the CUDA runtime uses): do not call this entry
 *     point after cudaDeviceReset, or with a driver-API context current that is not the primary one.
 *   - Arguments are checked in the order of deltakv_decode_attention (DKV_ERR_INVALID_ARG, then
 *     DKV_ERR_UNSUPPORTED) before the scratch size, so only a supported call can return DKV_ERR_WORKSPACE.
 *   - All calls share the one array and it keeps the contents the last call left; the parts that must
 *     start from zero are cleared on the stream by every call.  Calls that overlap on the GPU (other
 *     streams, other host threads) race on the array: serialise them.
 */
#define DKV_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
dkv_status deltakv_decode_attention_noalloc(const dkv_shape* shape, const dkv_params* params,
                                            const dkv_cache* cache, const void* q, const int32_t* context_lens,
                                            const int32_t* block_tables, int32_t max_blocks, int32_t num_seqs,
                                            int32_t max_ctx, float softmax_scale, void* out, float* lse,
                                            void* stream);

/* Error word codes recorded by kernels (see deltakv_get_device_error). */
#define DKV_DEVERR_NONE 0
#define DKV_DEVERR_BLOCK_ID 1    /* block table entry outside [0, num_blocks)               */
#define DKV_DEVERR_REF_IDX 2     /* stored reference index outside [0, ceil(T/R))           */
#define DKV_DEVERR_BOUNDS 3      /* a device length exceeds its host-side bound              */
#define DKV_DEVERR_TIMEOUT 4     /* a pipeline wait exceeded its time limit; the kernel quit  */

/* Synchronises `stream`, then returns in *code (host) the first error recorded on the current device
 * since the last call (DKV_DEVERR_*), and clears it. */
dkv_status deltakv_get_device_error(void* stream, int32_t* code);

/* Self-test of the kernels' bounded waits (failure detection without a fault).  Launches, on `stream`, one
 * thread that waits with the kernels' own wait loop, but a limit of limit_ns (1 us .. 2 s) of global time, on
 * an mbarrier phase that nothing completes.  When the limit runs out, the wait records DKV_DEVERR_TIMEOUT in
 * the device error word and the kernel returns: the context stays usable.
 *   result  device pointer to 2 uint64 (8-byte aligned): [0] = 1 if the phase completed (never), [1] = the
 *           wait's duration in ns.  Owned by the caller; written when the kernel runs.
 * Returns DKV_ERR_INVALID_ARG for a limit outside the range or a misaligned or NULL result, before any launch.
 */
dkv_status deltakv_selftest_wait_timeout(uint64_t limit_ns, uint64_t* result, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DELTAKV_H */
