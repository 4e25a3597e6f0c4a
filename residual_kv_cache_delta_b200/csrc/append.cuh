// Small appends of the compress path on sm_100a (bf16 cosine search, at most kAppendMaxNew new tokens per
// sequence): search and codes on CUDA cores over the reference rows of the paged cache.
// Summary (en) §3, "for a new token, it retrieves the most similar reference among the preceding ones": a
// decoding step appends one token per sequence, so the per-call cost should follow the references it reads,
// not the 256-row tiles of the tensor-core search.
// Included by compress.cuh after its device code (it uses SeqRange, load_seq, lookup_block, ceil_div_i).
#pragma once

namespace dkv {

// ------------------------------------------------------------------------------------------------
// 4. Appends (bf16 cosine search, at most kAppendMaxNew new tokens per sequence): search and codes on CUDA
//    cores, reading every reference row straight from the paged cache.  No contiguous copy, inverse norm or
//    projection of the stored references is made, so the cost of a call is one read of each visible reference
//    row per kv head, with the norm formed beside the dot products, instead of the whole reference prep and a
//    256-row tensor-core unit per (sequence, kv head).
//  append_search_kernel  CTA = (kAppendRefs references, kv head, sequence), one reference per thread.  The new
//    tokens' centred rows x~ = RNE_S(fp32(x - mu)) are staged in shared memory as fp32.  Each thread forms
//    |r~_j|^2 and x~_t . r~_j for every new token t that sees reference j (j < ceil(t / R)), scores
//    s = (x~_t . r~_j) * (1 / sqrt(|r~_j|^2)) in fp32, and the CTA's best (score, j) per token goes to a
//    64-bit atomic maximum in the workspace: key = order(score) << 32 | (0xffffffff - j), so equal scores go
//    to the smallest j, as in the other searches.
//  append_codes_kernel  CTA = (new token, kv head, sequence): reference tokens take their own index and zero
//    codes; the others stage B_K, B_V, x~ and the winning reference row r~_j in shared memory, and thread o
//    forms the code P_o - PR_j,o with P = x~ . blockdiag(B_K, B_V) and
//    PR_j = r~_j . blockdiag(B_K, B_V) in fp32 (the same products as the tensor-core path's fp32 accumulators),
//    rounded to bf16 once.
// ------------------------------------------------------------------------------------------------
constexpr int kAppendMaxNew = 16;   // new tokens per sequence up to which a call takes this path
constexpr int kAppendRefs = 256;    // references per search CTA

// Order-preserving map of fp32 bits to unsigned (larger float -> larger unsigned).
__device__ __forceinline__ uint32_t order_f32(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int D>
__global__ void __launch_bounds__(kAppendRefs) append_search_kernel(
    const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new,
    const float* __restrict__ mu, const __nv_bfloat16* __restrict__ refs, const int* __restrict__ cu_new,
    const int* __restrict__ start_pos, const int* __restrict__ block_tables, int max_blocks, int num_blocks,
    int H, int R, int64_t total_new, int max_new, int max_ctx, unsigned long long* __restrict__ keys) {
  __shared__ float xs[kAppendMaxNew][2 * D];
  const int s = blockIdx.z, h = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31;
  SeqRange sr;
  if (!load_seq(cu_new, start_pos, s, total_new, max_new, max_ctx, sr)) return;  // recorded by center_kernel
  const int n = sr.n_new;
  if (n <= 0) return;
  const int jmax = ceil_div_i(sr.start + n - 1, R);  // references the call's last token sees
  const int j0 = blockIdx.x * kAppendRefs;
  if (j0 >= jmax) return;  // CTA-uniform
  for (int e = tid; e < n * 2 * D; e += kAppendRefs) {
    const int i = e / (2 * D), c = e % (2 * D), kv = c / D, cc = c % D;
    const int64_t trow = sr.base + i;
    const float x = __bfloat162float((kv ? v_new : k_new)[(trow * H + h) * D + cc]);
    xs[i][c] = __bfloat162float(__float2bfloat16_rn(__fsub_rn(x, __ldg(mu + (h * 2 + kv) * D + cc))));
  }
  __syncthreads();
  const int j = j0 + tid;
  float dot[kAppendMaxNew];
#pragma unroll
  for (int i = 0; i < kAppendMaxNew; ++i) dot[i] = 0.f;
  float nrm = 0.f;
  bool have = false;
  if (j < jmax) {
    const int pb = lookup_block(block_tables, max_blocks, num_blocks, s, j);
    if (pb >= 0) {
      have = true;
      const uint4* row = reinterpret_cast<const uint4*>(refs + (static_cast<int64_t>(pb) * H + h) * 2 * D);
#pragma unroll 8
      for (int c = 0; c < 2 * D / 8; ++c) {
        float f[8];
        unpack16(__ldg(row + c), f, static_cast<__nv_bfloat16*>(nullptr));
#pragma unroll
        for (int e = 0; e < 8; ++e) nrm = fmaf(f[e], f[e], nrm);
#pragma unroll
        for (int i = 0; i < kAppendMaxNew; ++i) {
          if (i < n) {
            const float4 xa = *reinterpret_cast<const float4*>(&xs[i][c * 8]);
            const float4 xb = *reinterpret_cast<const float4*>(&xs[i][c * 8 + 4]);
            float d = dot[i];
            d = fmaf(f[0], xa.x, d);
            d = fmaf(f[1], xa.y, d);
            d = fmaf(f[2], xa.z, d);
            d = fmaf(f[3], xa.w, d);
            d = fmaf(f[4], xb.x, d);
            d = fmaf(f[5], xb.y, d);
            d = fmaf(f[6], xb.z, d);
            d = fmaf(f[7], xb.w, d);
            dot[i] = d;
          }
        }
      }
    }
  }
  const float inv = nrm > 0.f ? 1.0f / sqrtf(nrm) : 0.f;
#pragma unroll
  for (int i = 0; i < kAppendMaxNew; ++i) {
    if (i >= n) break;  // uniform
    const int t = sr.start + i;
    if (t % R == 0) continue;  // reference tokens do not search (uniform)
    const bool vis = have && j < ceil_div_i(t, R);
    unsigned long long key = vis ? (static_cast<unsigned long long>(order_f32(dot[i] * inv)) << 32) |
                                       static_cast<unsigned long long>(0xffffffffu - static_cast<uint32_t>(j))
                                 : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, o);
      key = other > key ? other : key;
    }
    if (lane == 0 && key != 0ull) atomicMax(keys + (static_cast<int64_t>(s) * H + h) * max_new + i, key);
  }
}

constexpr int kAppendCodeThreads = 128;

template <int D, int RK>
__global__ void __launch_bounds__(kAppendCodeThreads) append_codes_kernel(
    const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new,
    const float* __restrict__ mu, const __nv_bfloat16* __restrict__ basis, const __nv_bfloat16* __restrict__ refs,
    const int* __restrict__ cu_new, const int* __restrict__ start_pos, const int* __restrict__ block_tables,
    int max_blocks, int num_blocks, int H, int R, int64_t total_new, int max_new, int max_ctx,
    const unsigned long long* __restrict__ keys, __nv_bfloat16* __restrict__ codes, int* __restrict__ ref_idx) {
  static_assert(2 * RK <= kAppendCodeThreads, "one thread per code dimension");
  // B_K and B_V [2][D][RK] (as stored), the token's x~ and the winning reference row r~_j [2D] (fp32)
  __shared__ __align__(16) __nv_bfloat16 bs[2 * D * RK];
  __shared__ float xsh[2 * D], rsh[2 * D];
  const int i = blockIdx.x, h = blockIdx.y, s = blockIdx.z, tid = threadIdx.x;
  SeqRange sr;
  if (!load_seq(cu_new, start_pos, s, total_new, max_new, max_ctx, sr)) return;  // recorded by center_kernel
  if (i >= sr.n_new) return;
  const __nv_bfloat16* bsrc = basis + static_cast<int64_t>(h) * 2 * D * RK;
  {
    const int t = sr.start + i;
    const int pb_t = lookup_block(block_tables, max_blocks, num_blocks, s, t / R);
    if (pb_t < 0) return;  // uniform
    const int64_t cell = (static_cast<int64_t>(pb_t) * H + h) * R + t % R;  // row of token t in codes / ref_idx
    __nv_bfloat16* crow = codes + cell * 2 * RK;
    if (t % R == 0) {  // a reference token: its own index, zero codes
      if (tid < 2 * RK) crow[tid] = __float2bfloat16_rn(0.f);
      if (tid == 0) ref_idx[cell] = t / R;
      return;
    }
    const unsigned long long key = keys[(static_cast<int64_t>(s) * H + h) * max_new + i];
    const int j = static_cast<int>(0xffffffffu - static_cast<uint32_t>(key & 0xffffffffull));
    int jj = j;
    if (key == 0ull || j < 0 || j >= ceil_div_i(t, R)) {
      if (tid == 0) record_error(DKV_DEVERR_REF_IDX);
      jj = 0;
    }
    const int pb_j = lookup_block(block_tables, max_blocks, num_blocks, s, jj);
    const __nv_bfloat16* rrow = refs + (static_cast<int64_t>(pb_j < 0 ? 0 : pb_j) * H + h) * 2 * D;
    const int64_t trow = sr.base + i;
    for (int e = tid; e < 2 * D * RK / 8; e += kAppendCodeThreads)
      reinterpret_cast<uint4*>(bs)[e] = __ldg(reinterpret_cast<const uint4*>(bsrc) + e);
    for (int c = tid; c < 2 * D; c += kAppendCodeThreads) {
      const int kv = c / D, cc = c % D;
      const float x = __bfloat162float((kv ? v_new : k_new)[(trow * H + h) * D + cc]);
      xsh[c] = __bfloat162float(__float2bfloat16_rn(__fsub_rn(x, __ldg(mu + (h * 2 + kv) * D + cc))));
      rsh[c] = __bfloat162float(rrow[c]);
    }
    __syncthreads();
    if (tid < 2 * RK) {
      const int kv = tid / RK, oc = tid % RK;
      const __nv_bfloat16* bcol = bs + kv * D * RK + oc;  // B[k][oc], stride RK
      float p = 0.f, q = 0.f;
#pragma unroll 8
      for (int k = 0; k < D; ++k) {
        const float b = __bfloat162float(bcol[k * RK]);
        p = fmaf(xsh[kv * D + k], b, p);
        q = fmaf(rsh[kv * D + k], b, q);
      }
      crow[tid] = __float2bfloat16_rn(p - q);
    }
    if (tid == 0) ref_idx[cell] = jj;
  }
}

}  // namespace dkv
