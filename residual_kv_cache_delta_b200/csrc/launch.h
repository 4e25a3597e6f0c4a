// Launch entry points of the compress and decode paths (host side, called by the C ABI in deltakv.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <utility>

#include "../../include/deltakv.h"

namespace dkv {

// Raises a kernel's dynamic shared-memory limit to the device's opt-in maximum (less its static shared
// memory), once per (kernel, device) and safely from several host threads.  The attribute belongs to the
// current device's context, so a process that drives several devices sets it on each of them.
// CTAs of `Kernel` resident per SM at `threads` threads and `smem` bytes of dynamic shared memory (at least
// 1), from the occupancy calculator; cached per device and shared-memory size.
template <auto Kernel>
inline int resident_ctas(int threads, size_t smem) {
  static std::mutex mu;
  struct Entry {
    int dev;
    size_t smem;
    int n;
  };
  static Entry cache[16];
  static int used = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 1;
  }
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].dev == dev && cache[i].smem == smem) return cache[i].n;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kernel, threads, smem) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = 1;
  }
  if (used < 16) cache[used++] = Entry{dev, smem, n};
  return n;
}

template <auto Kernel, bool kMaxCarveout = false>
inline bool ensure_max_dynamic_smem() {
  static std::mutex mu;
  static uint64_t done = 0;  // one bit per device ordinal below 64
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 64 && ((done >> dev) & 1u)) return true;
  int optin = 0;
  cudaFuncAttributes fa;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
  if (cudaFuncGetAttributes(&fa, Kernel) != cudaSuccess) return false;
  if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           optin - static_cast<int>(fa.sharedSizeBytes)) != cudaSuccess)
    return false;
  // kMaxCarveout: ask for the largest shared-memory share of the L1 (two CTAs of a persistent kernel per SM)
  if (kMaxCarveout && cudaFuncSetAttribute(Kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                           cudaSharedmemCarveoutMaxShared) != cudaSuccess)
    return false;
  if (dev < 64) done |= uint64_t(1) << dev;
  return true;
}

// Launches `kernel` with programmatic stream serialization: it may be scheduled before the previous kernel of
// the stream has completed (once that kernel's CTAs have all triggered griddepcontrol.launch_dependents) and
// must execute griddepcontrol.wait before it reads anything that kernel writes.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_programmatic(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

struct CompressArgs {
  const dkv_shape* shape;
  const dkv_params* params;
  const dkv_cache* cache;
  const void* k_new;
  const void* v_new;
  const int* cu_new;
  const int* start_pos;
  const int* block_tables;
  int max_blocks;
  int num_seqs;
  int64_t total_new;
  int max_new;
  int max_ctx;
  int topk = 0;  // 0: cosine top-1 search; 1, 2, 4: the k nearest by L2, residual against their mean
};

struct DecodeArgs {
  const dkv_shape* shape;
  const dkv_params* params;
  const dkv_cache* cache;
  const void* q;
  const int* context_lens;
  const int* block_tables;
  int max_blocks;
  int num_seqs;
  int max_ctx;
  float softmax_scale;
  void* out;
  float* lse;
  // sparse decode: the tokens of sequence s are sel[cu_sel[s] .. cu_sel[s+1]-1] (cu_sel == nullptr: dense)
  const int* sel = nullptr;
  const int* cu_sel = nullptr;
  int max_sel = 0;
  int topk = 1;  // reference slots per token (k-nearest retrieval: 1, 2 or 4)
};

dkv_status launch_compress(const CompressArgs& a, void* workspace, cudaStream_t stream);

// Timing hook (deltakv_profile_kernel): records the caller's events around a kernel launch.
void prof_begin(int kernel_id, cudaStream_t stream);
void prof_end(int kernel_id, cudaStream_t stream);
dkv_status launch_decode(const DecodeArgs& a, void* workspace, cudaStream_t stream);
// DKV_OK, or DKV_ERR_UNSUPPORTED when the decode kernels' shared memory cannot hold this shape and bound
// (max_sel >= 0: sparse decode over lists of at most max_sel tokens).
// topk: reference slots per token (1; 2 or 4 after the k-nearest compress).
dkv_status decode_supported(const dkv_shape& shape, int num_seqs, int max_ctx, int max_sel = -1, int topk = 1);
// Workspace layout of a decode call (max_sel >= 0: sparse), with the split plan the launch will use.
struct DecodeWs;
DecodeWs decode_layout(const dkv_shape& shape, int num_seqs, int max_ctx, int max_sel = -1, int topk = 1);

}  // namespace dkv
