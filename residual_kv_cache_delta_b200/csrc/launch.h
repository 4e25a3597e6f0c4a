// Launch entry points of the compress and decode paths (host side, called by the C ABI in api.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/deltakv.h"

namespace dkv {

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
};

dkv_status launch_compress(const CompressArgs& a, void* workspace, cudaStream_t stream);

// Timing hook (deltakv_profile_kernel): records the caller's events around a kernel launch.
void prof_begin(int kernel_id, cudaStream_t stream);
void prof_end(int kernel_id, cudaStream_t stream);
dkv_status launch_decode(const DecodeArgs& a, void* workspace, cudaStream_t stream);

}  // namespace dkv
