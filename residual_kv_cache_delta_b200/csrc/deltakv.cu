// libdeltakv.so: the C ABI declared in include/deltakv.h.  This is the library's single translation
// unit: it pulls in the compress and decode kernels, validates arguments on the host and enqueues the
// launches.  No device memory is allocated here and no stream is synchronised (except in
// deltakv_get_device_error).
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "compress.cuh"
#include "decode.cuh"
#include "layout.h"
#include "launch.h"

namespace dkv {

// Self-test of the kernels' bounded waits: one thread waits, with the same wait loop the kernels use and a
// caller-given limit, on an mbarrier phase that nothing completes (count 1, no arrival, no copy armed).
// out[0] = 1 if the phase completed, out[1] = the wait's duration in ns of global time.
__global__ void selftest_wait_kernel(uint64_t limit_ns, unsigned long long* out) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(smem_u32(&bar), 1);
  abort_flag = 0;
  fence_barrier_init();
  const uint64_t t0 = global_timer_ns();
  const bool done = mbar_wait_for(smem_u32(&bar), 0, &abort_flag, limit_ns);
  out[1] = global_timer_ns() - t0;
  out[0] = done ? 1ull : 0ull;
}


struct ProfSlot {
  cudaEvent_t* start = nullptr;
  cudaEvent_t* stop = nullptr;
  int n = 0, i = 0;
};
static ProfSlot g_prof[DKV_NUM_KERNELS];

// Inside a stream capture an event record must be marked external to become a real node of the graph
// (otherwise it only expresses a dependency and the event is never recorded when the graph runs).
static void record_event(cudaEvent_t e, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cs);
  if (cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
  else
    cudaEventRecord(e, st);
}

void prof_begin(int id, cudaStream_t st) {
  ProfSlot& p = g_prof[id];
  if (p.i < p.n) record_event(p.start[p.i], st);
}
void prof_end(int id, cudaStream_t st) {
  ProfSlot& p = g_prof[id];
  if (p.i < p.n) record_event(p.stop[p.i++], st);
}

}  // namespace dkv

// Scratch of deltakv_decode_attention_noalloc: one fixed array in the device image (per device that loads
// the library).  Host code only ever uses its device address, looked up per device with
// cudaGetSymbolAddress; the symbol itself is a host-side stand-in and is never passed to a kernel.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DKV_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoallocMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
dkv_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DKV_ERR_CUDA;
  if (dev < 0 || dev >= kNoallocMaxDevices) return DKV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return DKV_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return DKV_OK;
}

using dkv::elem_bytes;

bool pow2_in(int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

dkv_status check_shape(const dkv_shape* s) {
  if (s == nullptr) return DKV_ERR_INVALID_ARG;
  if (s->num_q_heads <= 0 || s->num_kv_heads <= 0 || s->head_dim <= 0 || s->rank <= 0 || s->ref_stride <= 0)
    return DKV_ERR_INVALID_ARG;
  if (s->dtype != DKV_F32 && s->dtype != DKV_BF16 && s->dtype != DKV_BF16_Q4) return DKV_ERR_INVALID_ARG;
  if (s->num_q_heads % s->num_kv_heads != 0) return DKV_ERR_INVALID_ARG;
  if (s->rank > s->head_dim) return DKV_ERR_INVALID_ARG;
  const int G = s->num_q_heads / s->num_kv_heads;
  if (s->head_dim != 64 && s->head_dim != 128) return DKV_ERR_UNSUPPORTED;
  if (!pow2_in(s->rank, 16, 128)) return DKV_ERR_UNSUPPORTED;
  if (!pow2_in(s->ref_stride, 16, 64)) return DKV_ERR_UNSUPPORTED;
  if (!pow2_in(G, 1, 8) || G * s->rank > 256) return DKV_ERR_UNSUPPORTED;
  if (s->dtype == DKV_BF16 && s->rank > 64) return DKV_ERR_UNSUPPORTED;  // projection tile is 2r <= 128 wide
  if (s->dtype == DKV_F32 && s->rank > 64) return DKV_ERR_UNSUPPORTED;
  if (s->dtype == DKV_BF16_Q4 && s->rank != 32 && s->rank != 64) return DKV_ERR_UNSUPPORTED;  // nibble words
  return DKV_OK;
}

// 16-byte alignment: kernels use 128-bit vector accesses and bulk copies on these arrays.
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Code rows of the cache are addressed with 32-bit row coordinates (tensor maps, packed row ids): the pool may
// hold at most 2^31 - 1 rows of R tokens per kv head in total.
bool cache_rows_fit(const dkv_shape* s, const dkv_cache* c) {
  return static_cast<int64_t>(c->num_blocks) * s->num_kv_heads * s->ref_stride <= INT32_MAX;
}

dkv_status check_bounds(const dkv_shape* s, int num_seqs, int max_ctx) {
  if (num_seqs < 0 || max_ctx < 0) return DKV_ERR_INVALID_ARG;
  if (dkv::max_refs(max_ctx, s->ref_stride) > DKV_MAX_REFS) return DKV_ERR_UNSUPPORTED;
  return DKV_OK;
}

dkv_status compress_impl(const dkv_shape* shape, int topk, const dkv_params* params, const dkv_cache* cache,
                         const void* k_new, const void* v_new, const int32_t* cu_new, const int32_t* start_pos,
                         const int32_t* block_tables, int32_t max_blocks, int32_t num_seqs, int64_t total_new,
                         int32_t max_new, int32_t max_ctx, void* workspace, size_t workspace_bytes, void* stream);
dkv_status decode_impl(const dkv_shape* shape, int topk, const dkv_params* params, const dkv_cache* cache,
                       const void* q, const int32_t* context_lens, const int32_t* block_tables, int32_t max_blocks,
                       int32_t num_seqs, int32_t max_ctx, float softmax_scale, void* out, float* lse, void* workspace,
                       size_t workspace_bytes, void* stream);

}  // namespace

extern "C" {

const char* deltakv_status_string(dkv_status status) {
  switch (status) {
    case DKV_OK: return "ok";
    case DKV_ERR_INVALID_ARG: return "invalid argument";
    case DKV_ERR_UNSUPPORTED: return "unsupported shape or size";
    case DKV_ERR_WORKSPACE: return "workspace too small";
    case DKV_ERR_CUDA: return "CUDA error";
    case DKV_ERR_OUT_OF_BLOCKS: return "block pool exhausted";
  }
  return "unknown status";
}

dkv_status deltakv_check_shape(const dkv_shape* shape) { return check_shape(shape); }

size_t deltakv_block_bytes(const dkv_shape* s) {
  if (check_shape(s) != DKV_OK) return 0;
  const size_t es = elem_bytes(*s), H = s->num_kv_heads, R = s->ref_stride;
  return H * (R * dkv::code_row_bytes(*s) + R * 4 + 2 * s->head_dim * es);
}

dkv_status deltakv_cache_bytes(const dkv_shape* s, int32_t num_blocks, size_t* codes_bytes,
                               size_t* ref_idx_bytes, size_t* refs_bytes) {
  const dkv_status st = check_shape(s);
  if (st != DKV_OK) return st;
  if (num_blocks < 0 || codes_bytes == nullptr || ref_idx_bytes == nullptr || refs_bytes == nullptr)
    return DKV_ERR_INVALID_ARG;
  const size_t es = elem_bytes(*s), H = s->num_kv_heads, R = s->ref_stride, nb = num_blocks;
  *codes_bytes = nb * H * R * dkv::code_row_bytes(*s);
  *ref_idx_bytes = nb * H * R * 4;
  *refs_bytes = nb * H * 2 * s->head_dim * es;
  return DKV_OK;
}

dkv_status deltakv_compress_workspace(const dkv_shape* s, int32_t num_seqs, int64_t total_new, int32_t max_new,
                                      int32_t max_ctx, size_t* bytes) {
  dkv_status st = check_shape(s);
  if (st != DKV_OK) return st;
  if (bytes == nullptr || total_new < 0 || max_new < 0) return DKV_ERR_INVALID_ARG;
  if ((st = check_bounds(s, num_seqs, max_ctx)) != DKV_OK) return st;
  *bytes = dkv::compress_ws_layout(*s, num_seqs, total_new, max_ctx).total;
  return DKV_OK;
}

dkv_status deltakv_decode_workspace(const dkv_shape* s, int32_t num_seqs, int32_t max_ctx, size_t* bytes) {
  dkv_status st = check_shape(s);
  if (st != DKV_OK) return st;
  if (bytes == nullptr) return DKV_ERR_INVALID_ARG;
  if ((st = check_bounds(s, num_seqs, max_ctx)) != DKV_OK) return st;
  if ((st = dkv::decode_supported(*s, num_seqs, max_ctx)) != DKV_OK) return st;
  *bytes = dkv::decode_layout(*s, num_seqs, max_ctx).total;
  return DKV_OK;
}

dkv_status deltakv_compress(const dkv_shape* shape, const dkv_params* params, const dkv_cache* cache,
                            const void* k_new, const void* v_new, const int32_t* cu_new, const int32_t* start_pos,
                            const int32_t* block_tables, int32_t max_blocks, int32_t num_seqs, int64_t total_new,
                            int32_t max_new, int32_t max_ctx, void* workspace, size_t workspace_bytes,
                            void* stream) {
  return compress_impl(shape, 0, params, cache, k_new, v_new, cu_new, start_pos, block_tables, max_blocks, num_seqs,
                       total_new, max_new, max_ctx, workspace, workspace_bytes, stream);
}

dkv_status deltakv_compress_topk(const dkv_shape* shape, int32_t k, const dkv_params* params, const dkv_cache* cache,
                                 const void* k_new, const void* v_new, const int32_t* cu_new,
                                 const int32_t* start_pos, const int32_t* block_tables, int32_t max_blocks,
                                 int32_t num_seqs, int64_t total_new, int32_t max_new, int32_t max_ctx,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  if (k != 1 && k != 2 && k != 4) return DKV_ERR_UNSUPPORTED;
  return compress_impl(shape, k, params, cache, k_new, v_new, cu_new, start_pos, block_tables, max_blocks, num_seqs,
                       total_new, max_new, max_ctx, workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace {

dkv_status compress_impl(const dkv_shape* shape, int topk, const dkv_params* params, const dkv_cache* cache,
                         const void* k_new, const void* v_new, const int32_t* cu_new, const int32_t* start_pos,
                         const int32_t* block_tables, int32_t max_blocks, int32_t num_seqs, int64_t total_new,
                         int32_t max_new, int32_t max_ctx, void* workspace, size_t workspace_bytes, void* stream) {
  dkv_status st = check_shape(shape);
  if (st != DKV_OK) return st;
  if (params == nullptr || cache == nullptr) return DKV_ERR_INVALID_ARG;
  if ((st = check_bounds(shape, num_seqs, max_ctx)) != DKV_OK) return st;
  if (total_new < 0 || max_new < 0 || max_blocks < 0) return DKV_ERR_INVALID_ARG;
  if (num_seqs == 0 || total_new == 0 || max_new == 0) return DKV_OK;
  if (max_new > max_ctx || total_new > static_cast<int64_t>(num_seqs) * max_new) return DKV_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_blocks) * shape->ref_stride < max_ctx) return DKV_ERR_INVALID_ARG;
  if (static_cast<int64_t>(shape->num_kv_heads) * total_new > INT32_MAX) return DKV_ERR_UNSUPPORTED;
  if (params->mu == nullptr || params->basis == nullptr || cache->codes == nullptr || cache->ref_idx == nullptr ||
      cache->refs == nullptr || cache->num_blocks <= 0 || k_new == nullptr || v_new == nullptr ||
      cu_new == nullptr || start_pos == nullptr || block_tables == nullptr || workspace == nullptr)
    return DKV_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return DKV_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(params->mu) || !aligned16(params->basis) ||
      !aligned16(cache->codes) || !aligned16(cache->ref_idx) || !aligned16(cache->refs))
    return DKV_ERR_INVALID_ARG;
  if (!cache_rows_fit(shape, cache)) return DKV_ERR_UNSUPPORTED;
  if (workspace_bytes < dkv::compress_ws_layout(*shape, num_seqs, total_new, max_ctx).total)
    return DKV_ERR_WORKSPACE;
  // the k-nearest retrieval runs on the tensor-core search with r in {32, 64}, bf16 codes
  if (topk > 0 && (shape->dtype != DKV_BF16 || (shape->rank != 32 && shape->rank != 64))) return DKV_ERR_UNSUPPORTED;
  dkv::CompressArgs a{shape,     params,       cache,      k_new,    v_new,     cu_new, start_pos,
                      block_tables, max_blocks, num_seqs, total_new, max_new, max_ctx, topk};
  return dkv::launch_compress(a, workspace, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

dkv_status deltakv_decode_attention(const dkv_shape* shape, const dkv_params* params, const dkv_cache* cache,
                                    const void* q, const int32_t* context_lens, const int32_t* block_tables,
                                    int32_t max_blocks, int32_t num_seqs, int32_t max_ctx, float softmax_scale,
                                    void* out, float* lse, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  return decode_impl(shape, 1, params, cache, q, context_lens, block_tables, max_blocks, num_seqs, max_ctx,
                     softmax_scale, out, lse, workspace, workspace_bytes, stream);
}

dkv_status deltakv_decode_topk_workspace(const dkv_shape* s, int32_t k, int32_t num_seqs, int32_t max_ctx,
                                         size_t* bytes) {
  dkv_status st = check_shape(s);
  if (st != DKV_OK) return st;
  if (bytes == nullptr) return DKV_ERR_INVALID_ARG;
  if (k != 1 && k != 2 && k != 4) return DKV_ERR_UNSUPPORTED;
  if ((st = check_bounds(s, num_seqs, max_ctx)) != DKV_OK) return st;
  if ((st = dkv::decode_supported(*s, num_seqs, max_ctx, -1, k)) != DKV_OK) return st;
  *bytes = dkv::decode_layout(*s, num_seqs, max_ctx, -1, k).total;
  return DKV_OK;
}

dkv_status deltakv_decode_attention_topk(const dkv_shape* shape, int32_t k, const dkv_params* params,
                                         const dkv_cache* cache, const void* q, const int32_t* context_lens,
                                         const int32_t* block_tables, int32_t max_blocks, int32_t num_seqs,
                                         int32_t max_ctx, float softmax_scale, void* out, float* lse,
                                         void* workspace, size_t workspace_bytes, void* stream) {
  if (k != 1 && k != 2 && k != 4) return DKV_ERR_UNSUPPORTED;
  return decode_impl(shape, k, params, cache, q, context_lens, block_tables, max_blocks, num_seqs, max_ctx,
                     softmax_scale, out, lse, workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace {

dkv_status decode_impl(const dkv_shape* shape, int topk, const dkv_params* params, const dkv_cache* cache,
                       const void* q, const int32_t* context_lens, const int32_t* block_tables, int32_t max_blocks,
                       int32_t num_seqs, int32_t max_ctx, float softmax_scale, void* out, float* lse, void* workspace,
                       size_t workspace_bytes, void* stream) {
  dkv_status st = check_shape(shape);
  if (st != DKV_OK) return st;
  if (params == nullptr || cache == nullptr) return DKV_ERR_INVALID_ARG;
  if ((st = check_bounds(shape, num_seqs, max_ctx)) != DKV_OK) return st;
  if (max_blocks < 0) return DKV_ERR_INVALID_ARG;
  if (num_seqs == 0) return DKV_OK;
  if (static_cast<int64_t>(max_blocks) * shape->ref_stride < max_ctx) return DKV_ERR_INVALID_ARG;
  if (params->mu == nullptr || params->basis == nullptr || cache->codes == nullptr || cache->ref_idx == nullptr ||
      cache->refs == nullptr || cache->num_blocks <= 0 || q == nullptr || context_lens == nullptr ||
      block_tables == nullptr || out == nullptr || workspace == nullptr)
    return DKV_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return DKV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(params->mu) || !aligned16(params->basis) || !aligned16(cache->codes) ||
      !aligned16(cache->ref_idx) || !aligned16(cache->refs))
    return DKV_ERR_INVALID_ARG;
  if (!cache_rows_fit(shape, cache)) return DKV_ERR_UNSUPPORTED;
  if ((st = dkv::decode_supported(*shape, num_seqs, max_ctx, -1, topk)) != DKV_OK) return st;
  if (workspace_bytes < dkv::decode_layout(*shape, num_seqs, max_ctx, -1, topk).total) return DKV_ERR_WORKSPACE;
  dkv::DecodeArgs a{shape, params, cache, q, context_lens, block_tables, max_blocks, num_seqs, max_ctx,
                    softmax_scale, out, lse};
  a.topk = topk;
  return dkv::launch_decode(a, workspace, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

dkv_status deltakv_decode_sparse_workspace(const dkv_shape* s, int32_t num_seqs, int32_t max_ctx, int32_t max_sel,
                                           size_t* bytes) {
  dkv_status st = check_shape(s);
  if (st != DKV_OK) return st;
  if (bytes == nullptr || max_sel < 0) return DKV_ERR_INVALID_ARG;
  if (dkv::is_q4(*s)) return DKV_ERR_UNSUPPORTED;
  if ((st = check_bounds(s, num_seqs, max_ctx)) != DKV_OK) return st;
  if ((st = dkv::decode_supported(*s, num_seqs, max_ctx, max_sel)) != DKV_OK) return st;
  *bytes = dkv::decode_layout(*s, num_seqs, max_ctx, max_sel).total;
  return DKV_OK;
}

dkv_status deltakv_decode_attention_sparse(const dkv_shape* shape, const dkv_params* params, const dkv_cache* cache,
                                           const void* q, const int32_t* context_lens, const int32_t* block_tables,
                                           int32_t max_blocks, const int32_t* token_idx, const int32_t* cu_tokens,
                                           int32_t max_sel, int32_t num_seqs, int32_t max_ctx, float softmax_scale,
                                           void* out, float* lse, void* workspace, size_t workspace_bytes,
                                           void* stream) {
  dkv_status st = check_shape(shape);
  if (st != DKV_OK) return st;
  if (params == nullptr || cache == nullptr) return DKV_ERR_INVALID_ARG;
  if ((st = check_bounds(shape, num_seqs, max_ctx)) != DKV_OK) return st;
  if (max_blocks < 0 || max_sel < 0) return DKV_ERR_INVALID_ARG;
  if (dkv::is_q4(*shape)) return DKV_ERR_UNSUPPORTED;  // sparse decode reads bf16 or fp32 codes
  if (num_seqs == 0) return DKV_OK;
  if (static_cast<int64_t>(max_blocks) * shape->ref_stride < max_ctx) return DKV_ERR_INVALID_ARG;
  if (params->mu == nullptr || params->basis == nullptr || cache->codes == nullptr || cache->ref_idx == nullptr ||
      cache->refs == nullptr || cache->num_blocks <= 0 || q == nullptr || context_lens == nullptr ||
      block_tables == nullptr || out == nullptr || workspace == nullptr || cu_tokens == nullptr ||
      (max_sel > 0 && token_idx == nullptr))
    return DKV_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return DKV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(params->mu) || !aligned16(params->basis) || !aligned16(cache->codes) ||
      !aligned16(cache->ref_idx) || !aligned16(cache->refs))
    return DKV_ERR_INVALID_ARG;
  if (!cache_rows_fit(shape, cache)) return DKV_ERR_UNSUPPORTED;
  if ((st = dkv::decode_supported(*shape, num_seqs, max_ctx, max_sel)) != DKV_OK) return st;
  if (workspace_bytes < dkv::decode_layout(*shape, num_seqs, max_ctx, max_sel).total) return DKV_ERR_WORKSPACE;
  dkv::DecodeArgs a{shape, params, cache, q, context_lens, block_tables, max_blocks, num_seqs, max_ctx,
                    softmax_scale, out, lse, token_idx, cu_tokens, max_sel};
  // an empty list array is never read (every sequence's list is empty), but the kernels take a valid pointer
  static const int32_t kNoTokens[1] = {0};
  if (a.sel == nullptr) a.sel = kNoTokens;
  return dkv::launch_decode(a, workspace, static_cast<cudaStream_t>(stream));
}

dkv_status deltakv_profile_kernel(int32_t kernel_id, void* const* start_events, void* const* stop_events,
                                  int32_t n) {
  if (kernel_id < 0 || kernel_id >= DKV_NUM_KERNELS || n < 0) return DKV_ERR_INVALID_ARG;
  dkv::ProfSlot& p = dkv::g_prof[kernel_id];
  const bool on = n > 0 && start_events != nullptr && stop_events != nullptr;
  p.start = on ? reinterpret_cast<cudaEvent_t*>(const_cast<void**>(start_events)) : nullptr;
  p.stop = on ? reinterpret_cast<cudaEvent_t*>(const_cast<void**>(stop_events)) : nullptr;
  p.n = on ? n : 0;
  p.i = 0;
  return DKV_OK;
}

dkv_status deltakv_profile_count(int32_t kernel_id, int32_t* n) {
  if (kernel_id < 0 || kernel_id >= DKV_NUM_KERNELS || n == nullptr) return DKV_ERR_INVALID_ARG;
  *n = dkv::g_prof[kernel_id].i;
  return DKV_OK;
}

dkv_status deltakv_decode_attention_noalloc(const dkv_shape* shape, const dkv_params* params,
                                            const dkv_cache* cache, const void* q, const int32_t* context_lens,
                                            const int32_t* block_tables, int32_t max_blocks, int32_t num_seqs,
                                            int32_t max_ctx, float softmax_scale, void* out, float* lse,
                                            void* stream) {
  dkv_status st = check_shape(shape);
  if (st != DKV_OK) return st;
  if (params == nullptr || cache == nullptr) return DKV_ERR_INVALID_ARG;
  if ((st = check_bounds(shape, num_seqs, max_ctx)) != DKV_OK) return st;
  if (max_blocks < 0) return DKV_ERR_INVALID_ARG;
  if (num_seqs == 0) return DKV_OK;
  if (static_cast<int64_t>(max_blocks) * shape->ref_stride < max_ctx) return DKV_ERR_INVALID_ARG;
  if (params->mu == nullptr || params->basis == nullptr || cache->codes == nullptr || cache->ref_idx == nullptr ||
      cache->refs == nullptr || cache->num_blocks <= 0 || q == nullptr || context_lens == nullptr ||
      block_tables == nullptr || out == nullptr)
    return DKV_ERR_INVALID_ARG;
  if ((st = dkv::decode_supported(*shape, num_seqs, max_ctx)) != DKV_OK) return st;
  if (dkv::decode_layout(*shape, num_seqs, max_ctx).total > DKV_NOALLOC_SCRATCH_BYTES) return DKV_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != DKV_OK) return st;
  return deltakv_decode_attention(shape, params, cache, q, context_lens, block_tables, max_blocks, num_seqs, max_ctx,
                                  softmax_scale, out, lse, scratch, DKV_NOALLOC_SCRATCH_BYTES, stream);
}

dkv_status deltakv_selftest_wait_timeout(uint64_t limit_ns, uint64_t* result, void* stream) {
  if (result == nullptr || (reinterpret_cast<uintptr_t>(result) & 7u) != 0) return DKV_ERR_INVALID_ARG;
  if (limit_ns < 1000ull || limit_ns > dkv::kWaitLimitNs) return DKV_ERR_INVALID_ARG;
  dkv::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      limit_ns, reinterpret_cast<unsigned long long*>(result));
  return cudaGetLastError() == cudaSuccess ? DKV_OK : DKV_ERR_CUDA;
}

dkv_status deltakv_get_device_error(void* stream, int32_t* code) {
  if (code == nullptr) return DKV_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DKV_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, dkv::g_error_word, sizeof(int)) != cudaSuccess) return DKV_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(dkv::g_error_word, &zero, sizeof(int)) != cudaSuccess) return DKV_ERR_CUDA;
  *code = v;
  return DKV_OK;
}

}  // extern "C"
