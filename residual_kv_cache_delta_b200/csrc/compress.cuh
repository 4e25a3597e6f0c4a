// DeltaKV compress on sm_100a.
//
// Three launches per call (summary (en) §3 "Methodology": strided references, residual encoding with a
// linear compressor; §2: removal of the shared high-norm component):
//   1. center_kernel   x~ = RNE_S(fp32(x - mu)) for every new token; reference rows go to the paged cache.
//   2. refprep_kernel  for every visible reference j of every (seq, kv head): a contiguous copy of r~_j,
//                      1/|r~_j| and the projection PR_j = r~_j . blockdiag(B_K, B_V).
//   3. search          score every (token, earlier reference) pair, keep the argmax, and emit
//                      code = RNE_S(P_t - PR_j*) with P_t = x~_t . blockdiag(B_K, B_V)  (f_c is linear, so
//                      f_c(x) - f_c(x^R) = P_t - PR_j).
//      bf16: search_tc_kernel -- tcgen05 tensor-core tiles fed by TMA, warp-specialised, accumulators in
//            tensor memory, argmax and code epilogue on CUDA cores.
//      fp32: search_simt_kernel -- CUDA-core fp32 (the tensor cores have no fp32-exact mode).
#include <cstdio>

#include "common.cuh"
#include "launch.h"
#include "layout.h"

namespace dkv {

// ------------------------------------------------------------------------------------------------
// 16-byte vector I/O in storage precision.
// ------------------------------------------------------------------------------------------------
template <typename T>
struct V16;
template <>
struct V16<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void load(const float* p, float (&f)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    f[0] = v.x, f[1] = v.y, f[2] = v.z, f[3] = v.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&f)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  }
};
template <>
struct V16<__nv_bfloat16> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&f)[8]) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    unpack16(v, f, static_cast<__nv_bfloat16*>(nullptr));
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&f)[8]) {
    uint4 v;
    v.x = pack_bf16x2(f[0], f[1]);
    v.y = pack_bf16x2(f[2], f[3]);
    v.z = pack_bf16x2(f[4], f[5]);
    v.w = pack_bf16x2(f[6], f[7]);
    *reinterpret_cast<uint4*>(p) = v;
  }
};

__device__ __forceinline__ int ceil_div_i(int a, int b) { return (a + b - 1) / b; }

// Reads and validates one sequence's new-token range; false (and an error record) if it breaks the
// host-side bounds.
struct SeqRange {
  int base, n_new, start;
};
__device__ __forceinline__ bool load_seq(const int* cu_new, const int* start_pos, int s, int64_t total_new,
                                         int max_new, int max_ctx, SeqRange& sr) {
  sr.base = __ldg(cu_new + s);
  sr.n_new = __ldg(cu_new + s + 1) - sr.base;
  sr.start = __ldg(start_pos + s);
  const bool ok = sr.base >= 0 && sr.n_new >= 0 && sr.n_new <= max_new && sr.start >= 0 &&
                  static_cast<int64_t>(sr.base) + sr.n_new <= total_new &&
                  static_cast<int64_t>(sr.start) + sr.n_new <= max_ctx;
  return ok;
}

__device__ __forceinline__ int lookup_block(const int* block_tables, int max_blocks, int num_blocks, int s, int lb) {
  const int pb = __ldg(block_tables + static_cast<int64_t>(s) * max_blocks + lb);
  if (pb < 0 || pb >= num_blocks) {
    record_error(DKV_DEVERR_BLOCK_ID);
    return -1;
  }
  return pb;
}

// ------------------------------------------------------------------------------------------------
// 1. Centre the new tokens.  One thread per 16-byte vector of a (token, kv head) K|V row pair; the
//    (token, head) decomposition costs one 32-bit division per thread.  REFS_ONLY: only the reference
//    tokens of the call (written to the paged cache); the tensor-core search centres its own token tiles.
// ------------------------------------------------------------------------------------------------
template <typename T, int D>
struct CenterCfg {
  static constexpr int V = V16<T>::N;
  static constexpr int VPR = 2 * D / V;    // vectors per (token, head): K row then V row
  static constexpr int ROWS = 256 / VPR;   // (token, head) rows per CTA
};

template <typename T, int D, bool REFS_ONLY>
__global__ void __launch_bounds__(256) center_kernel(const T* __restrict__ k_new, const T* __restrict__ v_new,
                                                     const float* __restrict__ mu, const int* __restrict__ cu_new,
                                                     const int* __restrict__ start_pos,
                                                     const int* __restrict__ block_tables, int max_blocks,
                                                     int num_blocks, int H, int R, int64_t total_new, int max_new,
                                                     int max_ctx, T* __restrict__ xt, T* __restrict__ refs) {
  using C = CenterCfg<T, D>;
  constexpr int V = C::V, HALF = C::VPR / 2;
  const int s = blockIdx.y;
  SeqRange sr;
  if (!load_seq(cu_new, start_pos, s, total_new, max_new, max_ctx, sr)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_error(DKV_DEVERR_BOUNDS);
    return;
  }
  const int row = blockIdx.x * C::ROWS + threadIdx.x / C::VPR;
  const int vi = threadIdx.x % C::VPR;
  const int i_local = row / H, h = row - (row / H) * H;
  // REFS_ONLY: row i_local is the call's i-th reference token (positions that are multiples of R)
  const int n_local = REFS_ONLY ? ceil_div_i(sr.start, R) * R + i_local * R - sr.start : i_local;
  if (n_local >= sr.n_new) return;
  const int kv = vi / HALF, c = vi % HALF;
  const int64_t trow = sr.base + n_local;
  const int pos = sr.start + n_local;
  float x[V], m[V];
  V16<T>::load((kv ? v_new : k_new) + (trow * H + h) * D + c * V, x);
  const float4* mp = reinterpret_cast<const float4*>(mu + (h * 2 + kv) * D + c * V);
#pragma unroll
  for (int e = 0; e < V / 4; ++e) {
    const float4 q = __ldg(mp + e);
    m[4 * e] = q.x, m[4 * e + 1] = q.y, m[4 * e + 2] = q.z, m[4 * e + 3] = q.w;
  }
#pragma unroll
  for (int e = 0; e < V; ++e) x[e] = __fsub_rn(x[e], m[e]);  // IEEE fp32 subtract; rounding to S in store
  if (!REFS_ONLY) V16<T>::store(xt + (static_cast<int64_t>(h) * total_new + trow) * (2 * D) + kv * D + c * V, x);
  if (pos % R == 0) {
    const int pb = lookup_block(block_tables, max_blocks, num_blocks, s, pos / R);
    if (pb >= 0) V16<T>::store(refs + ((static_cast<int64_t>(pb) * H + h) * 2 + kv) * D + c * V, x);
  }
}

// ------------------------------------------------------------------------------------------------
// 2. Reference prep: contiguous copy, inverse norm and projection of every visible reference.
//    CTA = (64 references, kv head, sequence), 256 threads.  CTAs (0, h, 0) also write the bf16
//    blockdiag(B_K, B_V)^T operand of the projection MMA.
// ------------------------------------------------------------------------------------------------
constexpr int kPrepRefs = 64;

template <typename T, int D, int RK>
struct PrepCfg {
  static constexpr int V = V16<T>::N;
  static constexpr int VPR = 2 * D / V;  // 16-byte vectors per reference row
  static constexpr int RS = 2 * D + 1;   // padded fp32 row stride in shared memory
  static constexpr size_t SMEM = (static_cast<size_t>(kPrepRefs) * RS + 2 * D * RK + 4 * kPrepRefs) * sizeof(float);
};

template <typename T, int D, int RK>
__global__ void __launch_bounds__(256) refprep_kernel(const T* __restrict__ refs, const T* __restrict__ basis,
                                                      const int* __restrict__ cu_new,
                                                      const int* __restrict__ start_pos,
                                                      const int* __restrict__ block_tables, int max_blocks,
                                                      int num_blocks, int H, int R, int64_t total_new,
                                                      int max_new, int max_ctx, int64_t max_ref_pad,
                                                      T* __restrict__ refc, float* __restrict__ invn,
                                                      float* __restrict__ pr, __nv_bfloat16* __restrict__ bd) {
  using C = PrepCfg<T, D, RK>;
  constexpr int V = C::V, RS = C::RS;
  extern __shared__ float sm_prep[];
  float* rs = sm_prep;                      // [64][2D+1]
  float* bs = rs + kPrepRefs * RS;          // [2][D][RK]
  float* ssp = bs + 2 * D * RK;             // [4][64] partial sums of squares
  const int s = blockIdx.z, h = blockIdx.y, j0 = blockIdx.x * kPrepRefs;
  const int tid = threadIdx.x;
  const T* bsrc = basis + static_cast<int64_t>(h) * 2 * D * RK;
  const bool write_bd = bd != nullptr && blockIdx.x == 0 && s == 0;
  SeqRange sr;
  if (!load_seq(cu_new, start_pos, s, total_new, max_new, max_ctx, sr)) {  // recorded by center_kernel
    if (!write_bd) return;
    sr.start = sr.n_new = 0;
  }
  const int n_ref = ceil_div_i(sr.start + sr.n_new, R);
  if (j0 >= n_ref && !write_bd) return;
  const int64_t rowbase = (static_cast<int64_t>(s) * H + h) * max_ref_pad;

  // Every load of this CTA is issued before any is used (one round trip for the block id, one for the
  // rows and the basis).  A thread stages one reference row: 16-byte vectors c = tid/64 + 4i of row
  // j0 + tid%64 (consecutive lanes take consecutive rows, so the padded-stride shared-memory writes fall in
  // distinct banks).
  constexpr int NIT = kPrepRefs * C::VPR / 256;
  constexpr int NBI = 2 * D * RK / V / 256;
  const int jj_s = tid % kPrepRefs, c_s = tid / kPrepRefs;
  const int j_s = j0 + jj_s;
  const int pb = j_s < n_ref ? lookup_block(block_tables, max_blocks, num_blocks, s, j_s) : -1;
  float xs[NIT][V];
  float xb[NBI][V];
#pragma unroll
  for (int i = 0; i < NIT; ++i) {
    if (pb >= 0) {
      V16<T>::load(refs + (static_cast<int64_t>(pb) * H + h) * 2 * D + (c_s + 4 * i) * V, xs[i]);
    } else {
#pragma unroll
      for (int q = 0; q < V; ++q) xs[i][q] = 0.f;
    }
  }
#pragma unroll
  for (int i = 0; i < NBI; ++i) V16<T>::load(bsrc + (tid + 256 * i) * V, xb[i]);
  // basis of this kv head as fp32: bs[kv][k][o]
#pragma unroll
  for (int i = 0; i < NBI; ++i) {
#pragma unroll
    for (int q = 0; q < V; q += 4)
      *reinterpret_cast<float4*>(bs + (tid + 256 * i) * V + q) =
          make_float4(xb[i][q], xb[i][q + 1], xb[i][q + 2], xb[i][q + 3]);
  }
#pragma unroll
  for (int i = 0; i < NIT; ++i) {
    const int c = c_s + 4 * i;
    if (pb >= 0) V16<T>::store(refc + (rowbase + j_s) * 2 * D + c * V, xs[i]);
#pragma unroll
    for (int q = 0; q < V; ++q) rs[jj_s * RS + c * V + q] = xs[i][q];
  }
  __syncthreads();
  if (write_bd) {
    // blockdiag(B_K, B_V)^T: row o < r holds B_K[:, o] in columns 0..D-1, row o >= r holds B_V[:, o-r]
    // in columns D..2D-1, zeros elsewhere (built from the staged fp32 basis, 8 columns per store;
    // consecutive threads take consecutive rows o, so the shared-memory reads are conflict-free)
    __nv_bfloat16* dst = bd + static_cast<int64_t>(h) * 2 * RK * 2 * D;
    for (int e = tid; e < 2 * RK * 2 * D / 8; e += 256) {
      const int o = e % (2 * RK), k0 = (e / (2 * RK)) * 8;
      const int kv = o / RK;
      uint32_t wv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int k = k0 + 2 * q + u;
          v2[u] = (k >= D) == (kv == 1) ? bs[(kv * D + (k - kv * D)) * RK + (o - kv * RK)] : 0.f;
        }
        wv[q] = pack_bf16x2(v2[0], v2[1]);
      }
      *reinterpret_cast<uint4*>(dst + o * 2 * D + k0) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
    if (j0 >= n_ref) return;
  }

  const int jj = tid % kPrepRefs, part = tid / kPrepRefs;  // 4 parts per reference
  const int j = j0 + jj;
  // inverse norm: each part sums a quarter of the 2D values
  {
    float ss = 0.f;
    const float* xr = rs + jj * RS + part * (D / 2);
#pragma unroll 8
    for (int k = 0; k < D / 2; ++k) ss = fmaf(xr[k], xr[k], ss);
    ssp[part * kPrepRefs + jj] = ss;
  }
  // projection: part = (K|V half, which half of the r outputs)
  {
    constexpr int NO = RK / 2;
    const int og = part >> 1, oh = part & 1;
    float acc[NO];
#pragma unroll
    for (int m = 0; m < NO; ++m) acc[m] = 0.f;
    const float* xr = rs + jj * RS + og * D;
    const float* bk = bs + og * D * RK + oh * NO;
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      const float xv = xr[k];
      const float4* b4 = reinterpret_cast<const float4*>(bk + k * RK);
#pragma unroll
      for (int m4 = 0; m4 < NO / 4; ++m4) {
        const float4 b = b4[m4];
        acc[4 * m4 + 0] = fmaf(xv, b.x, acc[4 * m4 + 0]);
        acc[4 * m4 + 1] = fmaf(xv, b.y, acc[4 * m4 + 1]);
        acc[4 * m4 + 2] = fmaf(xv, b.z, acc[4 * m4 + 2]);
        acc[4 * m4 + 3] = fmaf(xv, b.w, acc[4 * m4 + 3]);
      }
    }
    if (j < n_ref) {
      float4* dst = reinterpret_cast<float4*>(pr + (rowbase + j) * 2 * RK + og * RK + oh * NO);
#pragma unroll
      for (int m4 = 0; m4 < NO / 4; ++m4)
        dst[m4] = make_float4(acc[4 * m4], acc[4 * m4 + 1], acc[4 * m4 + 2], acc[4 * m4 + 3]);
    }
  }
  __syncthreads();
  if (tid < kPrepRefs && j < n_ref) {
    const float ss = (ssp[jj] + ssp[kPrepRefs + jj]) + (ssp[2 * kPrepRefs + jj] + ssp[3 * kPrepRefs + jj]);
    invn[rowbase + j] = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
  }
}

// ------------------------------------------------------------------------------------------------
// 2b. Reference prep, bf16: the projection PR_j = r~_j . blockdiag(B_K, B_V) on the tensor cores.
//     CTA = (64 references, kv head, sequence), 256 threads.  The reference rows and the basis are staged
//     in shared memory as bf16 with padded rows (conflict-free ldmatrix); warp w computes the 16 references
//     16(w % 4) .. 16(w % 4) + 15 against B_K (w < 4) or B_V (w >= 4) with mma.sync m16n8k16 (bf16 products
//     are exact in fp32, accumulation in fp32).  Contiguous copy, 1/|r~_j| and the bf16 blockdiag operand
//     of the search kernel as in the CUDA-core variant.
// ------------------------------------------------------------------------------------------------
template <int D, int RK>
struct PrepTcCfg {
  static constexpr int XS = 2 * D + 8;    // padded bf16 row stride of the staged references
  static constexpr int BS = RK + 8;       // padded bf16 row stride of the staged basis [kv][k][n]
  static constexpr size_t SMEM = (static_cast<size_t>(kPrepRefs) * XS + 2 * D * BS) * 2 + 4 * kPrepRefs * 4;
};

template <int D, int RK>
__global__ void __launch_bounds__(256) refprep_tc_kernel(const __nv_bfloat16* __restrict__ refs,
                                                         const __nv_bfloat16* __restrict__ basis,
                                                         const int* __restrict__ cu_new,
                                                         const int* __restrict__ start_pos,
                                                         const int* __restrict__ block_tables, int max_blocks,
                                                         int num_blocks, int H, int R, int64_t total_new,
                                                         int max_new, int max_ctx, int64_t max_ref_pad,
                                                         __nv_bfloat16* __restrict__ refc, float* __restrict__ invn,
                                                         float* __restrict__ pr, __nv_bfloat16* __restrict__ bd,
                                                         int l2) {
  // l2 = 0: invn_j = 1/|r~_j| (cosine search); l2 = 1: invn_j = -|r~_j|^2 (nearest-by-L2 search)
  using C = PrepTcCfg<D, RK>;
  constexpr int XS = C::XS, BS = C::BS;
  constexpr int VPR = 2 * D / 8;                      // 16-byte vectors per reference row
  constexpr int NIT = kPrepRefs * VPR / 256;          // row vectors per thread
  constexpr int NBI = 2 * D * RK / 8 / 256 > 0 ? 2 * D * RK / 8 / 256 : 1;  // basis vectors per thread
  extern __shared__ __align__(16) unsigned char sm_preptc[];
  __nv_bfloat16* sx = reinterpret_cast<__nv_bfloat16*>(sm_preptc);   // [64][XS]
  __nv_bfloat16* sb = sx + kPrepRefs * XS;                             // [2][D][BS]
  float* ssp = reinterpret_cast<float*>(sb + 2 * D * BS);              // [4][64]
  const int s = blockIdx.z, h = blockIdx.y, j0 = blockIdx.x * kPrepRefs;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const __nv_bfloat16* bsrc = basis + static_cast<int64_t>(h) * 2 * D * RK;
  const bool write_bd = bd != nullptr && blockIdx.x == 0 && s == 0;
  SeqRange sr;
  if (!load_seq(cu_new, start_pos, s, total_new, max_new, max_ctx, sr)) {  // recorded by center_kernel
    if (!write_bd) return;
    sr.start = sr.n_new = 0;
  }
  const int n_ref = ceil_div_i(sr.start + sr.n_new, R);
  if (j0 >= n_ref && !write_bd) return;
  const int64_t rowbase = (static_cast<int64_t>(s) * H + h) * max_ref_pad;

  // stage: thread takes vectors c = tid/64 + 4i of reference j0 + tid%64, and basis vectors tid + 256i
  const int jj_s = tid % kPrepRefs, c_s = tid / kPrepRefs;
  const int j_s = j0 + jj_s;
  const int pb = j_s < n_ref ? lookup_block(block_tables, max_blocks, num_blocks, s, j_s) : -1;
  uint4 xs[NIT], xb[NBI];
#pragma unroll
  for (int i = 0; i < NIT; ++i)
    xs[i] = pb >= 0 ? __ldg(reinterpret_cast<const uint4*>(refs + (static_cast<int64_t>(pb) * H + h) * 2 * D) + c_s + 4 * i)
                    : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int i = 0; i < NBI; ++i)
    if (tid + 256 * i < 2 * D * RK / 8) xb[i] = __ldg(reinterpret_cast<const uint4*>(bsrc) + tid + 256 * i);
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NIT; ++i) {
    const int c = c_s + 4 * i;
    if (pb >= 0) reinterpret_cast<uint4*>(refc + (rowbase + j_s) * 2 * D)[c] = xs[i];
    *reinterpret_cast<uint4*>(sx + jj_s * XS + c * 8) = xs[i];
    float f[8];
    unpack16(xs[i], f, static_cast<__nv_bfloat16*>(nullptr));
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
  }
  ssp[c_s * kPrepRefs + jj_s] = ss;
#pragma unroll
  for (int i = 0; i < NBI; ++i) {
    const int e = tid + 256 * i;  // vector e of basis [kv][k][n]: 8 consecutive n of one (kv, k)
    if (e < 2 * D * RK / 8) {
      const int kvk = (e * 8) / RK, n0 = (e * 8) % RK;
      *reinterpret_cast<uint4*>(sb + kvk * BS + n0) = xb[i];
    }
  }
  __syncthreads();
  if (write_bd) {
    // blockdiag(B_K, B_V)^T: row o < r holds B_K[:, o] in columns 0..D-1, row o >= r holds B_V[:, o-r]
    // in columns D..2D-1, zeros elsewhere (8 columns per store; consecutive threads take consecutive rows)
    __nv_bfloat16* dst = bd + static_cast<int64_t>(h) * 2 * RK * 2 * D;
    for (int e = tid; e < 2 * RK * 2 * D / 8; e += 256) {
      const int o = e % (2 * RK), k0 = (e / (2 * RK)) * 8;
      const int kv = o / RK;
      uint32_t wv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t lo = 0, hi = 0;
        const int ka = k0 + 2 * q, kb = ka + 1;
        if ((ka >= D) == (kv == 1))
          lo = __bfloat16_as_ushort(sb[(kv * D + (ka - kv * D)) * BS + (o - kv * RK)]);
        if ((kb >= D) == (kv == 1))
          hi = __bfloat16_as_ushort(sb[(kv * D + (kb - kv * D)) * BS + (o - kv * RK)]);
        wv[q] = lo | (hi << 16);
      }
      *reinterpret_cast<uint4*>(dst + o * 2 * D + k0) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
    if (j0 >= n_ref) return;
  }
  // inverse norms
  if (tid < kPrepRefs && j0 + tid < n_ref) {
    const float t2 = (ssp[tid] + ssp[kPrepRefs + tid]) + (ssp[2 * kPrepRefs + tid] + ssp[3 * kPrepRefs + tid]);
    invn[rowbase + j0 + tid] = l2 ? -t2 : (t2 > 0.f ? 1.0f / sqrtf(t2) : 0.f);
  }
  // projection: warp -> (kv half, 16 references)
  const int kv = warp >> 2, mt = warp & 3;
  float acc[RK / 8][4];
#pragma unroll
  for (int n = 0; n < RK / 8; ++n)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[n][q] = 0.f;
  const uint32_t xa = smem_u32(sx + (mt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1)) * XS + kv * D + 8 * (lane >> 4));
  // B as [k][n]: matrices (k 0-7, n), (k 8-15, n), (k 0-7, n+8), (k 8-15, n+8), transposed on load
  const uint32_t xb0 = smem_u32(sb + (kv * D + (lane & 7) + 8 * ((lane >> 3) & 1)) * BS + 8 * (lane >> 4));
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    uint32_t a0, a1, a2, a3;
    ldsm_x4(xa + ks * 32, a0, a1, a2, a3);
#pragma unroll
    for (int np = 0; np < RK / 16; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(xb0 + (ks * 16 * BS + np * 16) * 2, b0, b1, b2, b3);
      mma_bf16_16816_a4(acc[2 * np], a0, a1, a2, a3, b0, b1);
      mma_bf16_16816_a4(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
    }
  }
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int n = 0; n < RK / 8; ++n) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int j = j0 + mt * 16 + g + 8 * half;
      if (j < n_ref)
        *reinterpret_cast<float2*>(pr + (rowbase + j) * 2 * RK + kv * RK + n * 8 + 2 * t) =
            make_float2(acc[n][2 * half], acc[n][2 * half + 1]);
    }
  }
}

// ------------------------------------------------------------------------------------------------
// 3a. SIMT search + codes (fp32 storage).  CTA = 64 new tokens of one (seq, kv head); thread = token.
// ------------------------------------------------------------------------------------------------
constexpr int kSimtTok = 64;
constexpr int kSimtRefs = 32;

template <typename T>
__global__ void __launch_bounds__(kSimtTok) search_simt_kernel(
    const T* __restrict__ xt, const T* __restrict__ refc, const float* __restrict__ invn,
    const T* __restrict__ basis, const int* __restrict__ cu_new, const int* __restrict__ start_pos,
    const int* __restrict__ block_tables, int max_blocks, int num_blocks, int H, int d, int r, int R,
    int64_t total_new, int max_new, int max_ctx, int64_t max_ref_pad, T* __restrict__ codes,
    int* __restrict__ ref_idx) {
  extern __shared__ float sm_simt[];
  const int d2 = 2 * d;
  float* xs = sm_simt;                        // [2d][64] transposed tokens
  float* rsm = xs + d2 * kSimtTok;       // [32][2d] references
  float* isv = rsm + kSimtRefs * d2;     // [32] inverse norms
  const int s = blockIdx.z, h = blockIdx.y, tid = threadIdx.x;
  SeqRange sr;
  if (!load_seq(cu_new, start_pos, s, total_new, max_new, max_ctx, sr)) return;
  const int i0 = blockIdx.x * kSimtTok;
  if (i0 >= sr.n_new) return;
  const int n_here = min(kSimtTok, sr.n_new - i0);
  const int i = i0 + tid;
  const bool valid = tid < n_here;
  const int t = sr.start + i;
  const int64_t xrow0 = static_cast<int64_t>(h) * total_new + sr.base + i0;
  for (int e = tid; e < kSimtTok * d2; e += kSimtTok) {
    const int tok = e / d2, k = e % d2;
    xs[k * kSimtTok + tok] = tok < n_here ? Elem<T>::to_f(xt[(xrow0 + tok) * d2 + k]) : 0.f;
  }
  const int jlim = valid ? ceil_div_i(t, R) : 0;
  const int jmax = ceil_div_i(sr.start + i0 + n_here - 1, R);
  const int64_t rowbase = (static_cast<int64_t>(s) * H + h) * max_ref_pad;
  float best = -INFINITY;
  int bj = 0;
  for (int jc = 0; jc < jmax; jc += kSimtRefs) {
    __syncthreads();
    for (int e = tid; e < kSimtRefs * d2; e += kSimtTok) {
      const int jj = e / d2, k = e % d2;
      rsm[e] = jc + jj < jmax ? Elem<T>::to_f(refc[(rowbase + jc + jj) * d2 + k]) : 0.f;
    }
    if (tid < kSimtRefs) isv[tid] = jc + tid < jmax ? invn[rowbase + jc + tid] : 0.f;
    __syncthreads();
    for (int jj = 0; jj < kSimtRefs && jc + jj < jlim; ++jj) {
      float dot = 0.f;
      for (int k = 0; k < d2; ++k) dot = fmaf(xs[k * kSimtTok + tid], rsm[jj * d2 + k], dot);
      const float sc = dot * isv[jj];
      if (sc > best) {
        best = sc;
        bj = jc + jj;
      }
    }
  }
  if (!valid) return;
  const bool isref = (t % R) == 0;
  if (isref) bj = t / R;
  const int pb = lookup_block(block_tables, max_blocks, num_blocks, s, t / R);
  if (pb < 0) return;
  T* cdst = codes + ((static_cast<int64_t>(pb) * H + h) * R + t % R) * (2 * r);
  const T* ref = refc + (rowbase + bj) * d2;
  const T* b = basis + static_cast<int64_t>(h) * 2 * d * r;
  for (int o = 0; o < 2 * r; ++o) {
    const int kv = o >= r ? 1 : 0, oo = o - kv * r;
    float c = 0.f;
    if (!isref) {
      for (int k = 0; k < d; ++k) {
        const float res = __fsub_rn(xs[(kv * d + k) * kSimtTok + tid], Elem<T>::to_f(ref[kv * d + k]));
        c = fmaf(res, Elem<T>::to_f(b[(kv * d + k) * r + oo]), c);
      }
    }
    cdst[o] = Elem<T>::from_f(c);
  }
  ref_idx[(static_cast<int64_t>(pb) * H + h) * R + t % R] = bj;
}

// ------------------------------------------------------------------------------------------------
// 3b. tcgen05 search + codes (bf16 storage), on pairs of SMs.
//
// Persistent two-CTA clusters.  A work unit is 256 new tokens of one (seq, kv head); CTA k of the pair
// owns token rows 128k .. 128k+127 of it (operand A, K-major, 128-byte swizzle; double-buffered, so the
// next unit's tokens load under the current unit's MMAs).  A reference tile is 256 references: each CTA
// streams its half (128 references in 64-column K-chunks) through a ring, and the leader CTA issues one
// 256 x 256 x 16 pair MMA (cta_group::2) per K step.  Each SM then reads only its own A rows and its own
// half of B from shared memory: half the shared-memory bytes per flop of a one-SM 128 x 128 MMA.
//   warp 0      TMA producer (one lane) of each CTA: loads its A rows, its half of every reference chunk
//               and of the projection basis, counting bytes on the leader's barriers.  The leader's
//               producer is also the scheduler: it takes the next unit from a global counter (units are
//               numbered longest first: a greedy longest-processing-time schedule) and publishes it to
//               both CTAs.
//   warp 1      tensor-memory owner (both CTAs) and MMA issuer (leader, one lane): per reference tile,
//               D[tok][ref] over K = 2d into one of two 256-column accumulators; the last item of a unit is
//               the projection P = x~ . blockdiag(B_K, B_V) (N = 2r).
//   warps 2..9  epilogue (both CTAs): warps 2-5 take columns 0-127 of a tile, warps 6-9 columns 128-255,
//               for the 128 rows of their CTA; scale by 1/|r_j|, running maximum; when a 64-column part
//               raises it, a second pass over the same registers finds the smallest j attaining it (ties
//               go to the smallest j); causal mask j*R < t on the boundary tile.  The two column halves
//               are merged per unit; then code = RNE(P - PR_j*), scattered to the cache.
// Accumulator double-buffering lets the epilogue of tile i overlap the MMAs of tile i+1.
// ------------------------------------------------------------------------------------------------
constexpr int kTcEpiWarps = 8;
constexpr int kTcConvWarps = 2;                  // centre the raw token tile in shared memory
constexpr int kTcThreads = (2 + kTcEpiWarps + kTcConvWarps) * 32;
constexpr int kTcTileM = 128;                    // token rows per CTA
constexpr int kTcUnit = 2 * kTcTileM;            // tokens per unit (pair)
constexpr int kTcHalfRefs = kRefTile / 2;        // references per CTA per tile
constexpr int kTcStageBytes = 16384;             // 128 rows x 64 bf16
constexpr int kTcSched = 4;                      // published-unit ring depth
// per unit: leader MMA + peer producer, and the epilogue and converter warps of both CTAs
constexpr int kTcSchConsumers = 2 * (1 + kTcEpiWarps + kTcConvWarps);

// KT: 0 = cosine argmax; 1, 2, 4 = the KT nearest by L2 (the two column halves' lists merge in kMrg).
template <int CH, int KT = 0>
struct TcConfig {
  static constexpr int kABytes = 2 * CH * kTcStageBytes;                  // two A buffers
  static constexpr int kStages = CH == 4 ? 5 : 8;
  static constexpr int kInvOffset = kABytes + kStages * kTcStageBytes;    // [2][256] fp32
  static constexpr int kMrgOffset = kInvOffset + 2 * kRefTile * 4;        // [2][128][KT] fp32 + int32
  static constexpr int kBarOffset = kMrgOffset + 4 * kTcTileM * 4 * (KT > 1 ? KT : 1);
  static constexpr int kNumBars = 6 + 2 * kStages + 4 + 2 * kTcSched;
  static constexpr int kSmemBytes = kBarOffset + kNumBars * 8 + 16 + kTcSched * 4 + 1024;  // + alignment slack
};

// 32 lanes x 64 consecutive fp32 columns.
__device__ __forceinline__ void tmem_ld_32x32b_x64(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}

// 32 lanes x 16 consecutive fp32 columns (into the first 16 entries of r).
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// Maximum over one 64-column part of a row of scaled scores s_e = v_e * inv_e (e < nv visible), with the
// column index carried in the result: each product's 6 lowest mantissa bits are replaced by 63 - e before
// the maximum is taken, so the maximum names its own column and, among products equal in the remaining
// bits, the smallest e (for positive scores).  The truncation changes a score by less than 2^-17 of its
// magnitude.  Returns the tagged fp32 bits; -inf bits (no tag) when nothing is visible.
__device__ __forceinline__ uint32_t part_max_tagged(const uint32_t (&v)[64], const float4* iv4, int nv) {
  float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  const bool full = nv >= 64;
#pragma unroll
  for (int e8 = 0; e8 < 8; ++e8) {
    const float4 ia = iv4[2 * e8], ib = iv4[2 * e8 + 1];
    const float ivs[8] = {ia.x, ia.y, ia.z, ia.w, ib.x, ib.y, ib.z, ib.w};
    float t[8];
#pragma unroll
    for (int h = 0; h < 4; ++h) {  // two products per packed multiply
      uint64_t pa, pb, pp;
      asm("mov.b64 %0, {%1, %2};" : "=l"(pa) : "r"(v[8 * e8 + 2 * h]), "r"(v[8 * e8 + 2 * h + 1]));
      asm("mov.b64 %0, {%1, %2};" : "=l"(pb) : "f"(ivs[2 * h]), "f"(ivs[2 * h + 1]));
      asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(pp) : "l"(pa), "l"(pb));
      uint32_t lo, hi;
      asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(pp));
      const int e = 8 * e8 + 2 * h;
      t[2 * h] = __uint_as_float((lo & ~63u) | static_cast<uint32_t>(63 - e));
      t[2 * h + 1] = __uint_as_float((hi & ~63u) | static_cast<uint32_t>(62 - e));
      if (!full) {
        if (e >= nv) t[2 * h] = -INFINITY;
        if (e + 1 >= nv) t[2 * h + 1] = -INFINITY;
      }
    }
    // four running maxima, two three-input maxima per 8 columns each
    float r0, r1;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r0) : "f"(m[(2 * e8) & 3]), "f"(t[0]), "f"(t[1]));
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r1) : "f"(m[(2 * e8 + 1) & 3]), "f"(t[2]), "f"(t[3]));
    m[(2 * e8) & 3] = r0;
    m[(2 * e8 + 1) & 3] = r1;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r0) : "f"(m[(2 * e8 + 2) & 3]), "f"(t[4]), "f"(t[5]));
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r1) : "f"(m[(2 * e8 + 3) & 3]), "f"(t[6]), "f"(t[7]));
    m[(2 * e8 + 2) & 3] = r0;
    m[(2 * e8 + 3) & 3] = r1;
  }
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(m[0]), "f"(m[1]), "f"(m[2]));
  r = fmaxf(r, m[3]);
  return __float_as_uint(r);
}

// Unit u (0-based, longest first) -> (token pair p, sequence s, kv head h).
struct TcUnit {
  int p, s, h;
};
__device__ __forceinline__ TcUnit decode_unit(int u, int num_seqs, int H, int num_pairs) {
  const int sh = num_seqs * H;
  TcUnit x;
  x.p = num_pairs - 1 - u / sh;
  const int rem = u % sh;
  x.s = rem / H;
  x.h = rem % H;
  return x;
}

// Per-unit geometry shared by every role.
struct TcGeom {
  SeqRange sr;
  int t0, n_here, nrt;
};
__device__ __forceinline__ TcGeom unit_geom(const TcUnit& x, const int* cu_new, const int* start_pos,
                                            int64_t total_new, int max_new, int max_ctx, int R) {
  TcGeom g;
  load_seq(cu_new, start_pos, x.s, total_new, max_new, max_ctx, g.sr);
  g.t0 = g.sr.start + x.p * kTcUnit;
  g.n_here = min(kTcUnit, g.sr.n_new - x.p * kTcUnit);
  g.nrt = ceil_div_i(ceil_div_i(g.t0 + g.n_here - 1, R), kRefTile);
  return g;
}
// The KT largest of one 64-column part of a row of nearness scores s_e = 2 v_e - |r_e|^2 (e < nv visible;
// nr holds -|r_e|^2), sorted descending, each carrying its column as 63 - e in the 6 lowest mantissa bits (as in
// part_max_tagged); -inf where fewer than KT columns are visible.  Two scores per packed fused multiply-add.
template <int KT>
__device__ __forceinline__ void part_topk_tagged(const uint32_t (&v)[64], const float4* nr4, int nv, float (&t)[KT]) {
#pragma unroll
  for (int k = 0; k < KT; ++k) t[k] = -INFINITY;
  const bool full = nv >= 64;
  const uint64_t two = 0x4000000040000000ull;  // {2.0f, 2.0f}
#pragma unroll
  for (int e8 = 0; e8 < 8; ++e8) {
    const float4 na = nr4[2 * e8], nb = nr4[2 * e8 + 1];
    const float ns[8] = {na.x, na.y, na.z, na.w, nb.x, nb.y, nb.z, nb.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      uint64_t pa, pc, pp;
      asm("mov.b64 %0, {%1, %2};" : "=l"(pa) : "r"(v[8 * e8 + 2 * h]), "r"(v[8 * e8 + 2 * h + 1]));
      asm("mov.b64 %0, {%1, %2};" : "=l"(pc) : "f"(ns[2 * h]), "f"(ns[2 * h + 1]));
      asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(pp) : "l"(pa), "l"(two), "l"(pc));
      uint32_t lo, hi;
      asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(pp));
      const int e = 8 * e8 + 2 * h;
      float x[2] = {__uint_as_float((lo & ~63u) | static_cast<uint32_t>(63 - e)),
                    __uint_as_float((hi & ~63u) | static_cast<uint32_t>(62 - e))};
      if (!full) {
        if (e >= nv) x[0] = -INFINITY;
        if (e + 1 >= nv) x[1] = -INFINITY;
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {  // insertion into the sorted list
        float y = x[u];
#pragma unroll
        for (int k = 0; k < KT; ++k) {
          const float hiv = fmaxf(t[k], y);
          y = fminf(t[k], y);
          t[k] = hiv;
        }
      }
    }
  }
}

// Inserts (cv, cj) into the list (bv, bj), sorted by value descending and, for equal values, by j ascending.
template <int KT>
__device__ __forceinline__ void topk_insert(float (&bv)[KT], int (&bj)[KT], float cv, int cj) {
#pragma unroll
  for (int k = 0; k < KT; ++k) {
    const bool b = cv > bv[k] || (cv == bv[k] && cj < bj[k]);
    const float tv = b ? bv[k] : cv;
    const int tj = b ? bj[k] : cj;
    bv[k] = b ? cv : bv[k];
    bj[k] = b ? cj : bj[k];
    cv = tv;
    cj = tj;
  }
}

// One 4-bit level of code c at scale s: clamp(rint(c / s), -7, 7) as a two's-complement nibble (0 when s = 0).
__device__ __forceinline__ uint32_t q4_nibble(float c, float s) {
  if (!(s > 0.f)) return 0u;
  const float q = fminf(fmaxf(rintf(__fdiv_rn(c, s)), -7.f), 7.f);
  return static_cast<uint32_t>(static_cast<int>(q)) & 15u;
}

template <int CH, bool Q4, int KT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcThreads, 1) search_tc_kernel(
    const __grid_constant__ CUtensorMap k_map, const __grid_constant__ CUtensorMap v_map,
    const __grid_constant__ CUtensorMap refc_map, const __grid_constant__ CUtensorMap bd_map,
    const float* __restrict__ mu, const float* __restrict__ invn, const float* __restrict__ pr,
    const int* __restrict__ cu_new, const int* __restrict__ start_pos, const int* __restrict__ block_tables,
    int max_blocks, int num_blocks, int num_seqs, int H, int R, int r, int64_t total_new, int64_t max_ref_pad,
    int max_new, int max_ctx, int num_pairs, int* __restrict__ work_counter, __nv_bfloat16* __restrict__ codes,
    int* __restrict__ ref_idx) {
  using C = TcConfig<CH, KT>;
  static_assert(!(Q4 && KT > 0), "4-bit codes with the cosine search only");
  constexpr int KTm = KT > 0 ? KT : 1;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_shared<1024>(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kABytes;
  float* sInv = reinterpret_cast<float*>(smem + C::kInvOffset);       // [2][kRefTile]
  float* sBest = reinterpret_cast<float*>(smem + C::kMrgOffset);      // [2][128][KTm]
  int* sBj = reinterpret_cast<int*>(sBest + 2 * kTcTileM * KTm);      // [2][128][KTm]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* a_full = bars + 0;            // [2] both: this CTA's raw token rows landed
  uint64_t* a_empty = bars + 2;           // [2] both: pair-MMA commit
  uint64_t* a_conv = bars + 4;            // [2] leader: converter warps of both CTAs finished centring
  uint64_t* b_full = bars + 6;            // [NS] leader
  uint64_t* b_empty = bars + 6 + NS;      // [NS] both
  uint64_t* acc_full = bars + 6 + 2 * NS; // [2] both
  uint64_t* acc_empty = acc_full + 2;     // [2] leader: every epilogue warp of both CTAs
  uint64_t* sch_full = acc_full + 4;      // [kTcSched] both
  uint64_t* sch_empty = sch_full + kTcSched;  // [kTcSched] leader
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sTmem + 1);
  volatile int* sUnit = reinterpret_cast<volatile int*>(sTmem + 4);  // [kTcSched]

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(a_full + i), 1);
      mbar_init(smem_u32(a_empty + i), 1);
      mbar_init(smem_u32(a_conv + i), 2 * kTcConvWarps);
      mbar_init(smem_u32(acc_full + i), 1);
      mbar_init(smem_u32(acc_empty + i), 2 * kTcEpiWarps);
    }
    for (int i = 0; i < NS; ++i) {
      mbar_init(smem_u32(b_full + i), 1);
      mbar_init(smem_u32(b_empty + i), 1);
    }
    for (int i = 0; i < kTcSched; ++i) {
      mbar_init(smem_u32(sch_full + i), 1);
      mbar_init(smem_u32(sch_empty + i), kTcSchConsumers);
    }
    *sAbort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&k_map);
    prefetch_tensormap(&v_map);
    prefetch_tensormap(&refc_map);
    prefetch_tensormap(&bd_map);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(sTmem), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem_base = *sTmem;

  const int r2 = 2 * r;
  const int total_units = num_pairs * num_seqs * H;
  // the leader's copies of the pair-wide barriers, as cluster addresses
  const uint32_t lead_a_conv = mapa_shared(smem_u32(a_conv), 0);
  const uint32_t lead_b_full = mapa_shared(smem_u32(b_full), 0);
  const uint32_t lead_acc_empty = mapa_shared(smem_u32(acc_empty), 0);
  const uint32_t lead_sch_empty = mapa_shared(smem_u32(sch_empty), 0);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- scheduler (leader) + producer (both) ----------------
      // next_unit(k): the leader takes a unit from the counter and publishes it as ring entry k to both
      // CTAs; the peer reads ring entry k.  -1 ends the work (and is published too).
      auto next_unit = [&](uint32_t k, int& u) -> bool {
        const uint32_t q = k % kTcSched;
        u = -1;
        if (leader) {
          for (;;) {
            const int c = atomicAdd(work_counter, 1);
            if (c >= total_units) break;
            const TcUnit x = decode_unit(c, num_seqs, H, num_pairs);
            SeqRange sr;
            if (!load_seq(cu_new, start_pos, x.s, total_new, max_new, max_ctx, sr)) continue;  // recorded by centre
            if (x.p * kTcUnit >= sr.n_new) continue;
            u = c;
            break;
          }
          if (!mbar_wait(smem_u32(sch_empty + q), ((k / kTcSched) & 1) ^ 1, sAbort)) return false;
          sUnit[q] = u;
          st_shared_cluster_u32(mapa_shared(smem_u32(const_cast<int*>(sUnit + q)), 1), static_cast<uint32_t>(u));
          mbar_arrive(smem_u32(sch_full + q));
          mbar_arrive_cluster(mapa_shared(smem_u32(sch_full + q), 1));  // release: orders the store above
        } else {
          if (!mbar_wait_cluster(smem_u32(sch_full + q), (k / kTcSched) & 1, sAbort)) return false;
          u = sUnit[q];
          mbar_arrive_cluster(lead_sch_empty + q * 8);  // release: the read above is done before the leader rewrites
        }
        return true;
      };
      // load_a(k, u): this CTA's 128 raw token rows of unit u (K columns, then V columns, of its kv head) into
      // A buffer k & 1; the converter warps centre them in place
      auto load_a = [&](uint32_t k, int u) -> bool {
        const TcUnit x = decode_unit(u, num_seqs, H, num_pairs);
        SeqRange sr;
        load_seq(cu_new, start_pos, x.s, total_new, max_new, max_ctx, sr);
        const int trow0 = static_cast<int>(sr.base + x.p * kTcUnit) + static_cast<int>(rank) * kTcTileM;
        const uint32_t abuf = k & 1;
        if (!mbar_wait(smem_u32(a_empty + abuf), ((k >> 1) & 1) ^ 1, sAbort)) return false;
        mbar_arrive_expect_tx(smem_u32(a_full + abuf), CH * kTcStageBytes);
        for (int c = 0; c < CH; ++c)
          tma_load_2d(smem_u32(sA + (abuf * CH + c) * kTcStageBytes), c < CH / 2 ? &k_map : &v_map,
                      x.h * (CH / 2) * 64 + (c % (CH / 2)) * 64, trow0, smem_u32(a_full + abuf));
        return true;
      };
      uint32_t stage = 0;
      int u = -1;
      bool ok = next_unit(0, u) && (u < 0 || load_a(0, u));
      for (uint32_t k = 0; ok && u >= 0; ++k) {
        const TcUnit x = decode_unit(u, num_seqs, H, num_pairs);
        const TcGeom g = unit_geom(x, cu_new, start_pos, total_new, max_new, max_ctx, R);
        const int64_t refrow0 = (static_cast<int64_t>(x.s) * H + x.h) * max_ref_pad;
        int u_next = -1;
        bool have_next = false, a_next = false;
        for (int rt = 0; rt <= g.nrt && ok; ++rt) {
          for (int c = 0; c < CH; ++c, ++stage) {
            const uint32_t slot = stage % NS;
            if (!mbar_wait(smem_u32(b_empty + slot), ((stage / NS) & 1) ^ 1, sAbort)) { ok = false; break; }
            if (rt < g.nrt) {
              if (leader) mbar_arrive_expect_tx(smem_u32(b_full + slot), 2 * kTcStageBytes);
              tma_load_2d_pair(smem_u32(sB + slot * kTcStageBytes), &refc_map, c * 64,
                               static_cast<int>(refrow0 + rt * kRefTile) + static_cast<int>(rank) * kTcHalfRefs,
                               lead_b_full + slot * 8);
            } else {
              if (leader) mbar_arrive_expect_tx(smem_u32(b_full + slot), 2 * (r2 / 2) * 128);
              tma_load_2d_pair(smem_u32(sB + slot * kTcStageBytes), &bd_map, c * 64,
                               x.h * r2 + static_cast<int>(rank) * (r2 / 2), lead_b_full + slot * 8);
            }
            // the next unit's tokens load (and are centred) under this unit's MMAs: its id is taken once
            // the first tile is queued, its rows are loaded as soon as their buffer is free
            if (have_next && !a_next && u_next >= 0 &&
                mbar_try_wait(smem_u32(a_empty + ((k + 1) & 1)), (((k + 1) >> 1) & 1) ^ 1)) {
              a_next = true;
              ok = load_a(k + 1, u_next);
              if (!ok) break;
            }
          }
          if (ok && !have_next) {
            have_next = true;
            ok = next_unit(k + 1, u_next);
          }
        }
        if (ok && u_next >= 0 && !a_next) ok = load_a(k + 1, u_next);
        u = u_next;
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (leader) ----------------
      uint32_t stage = 0, item = 0;
      for (uint32_t k = 0;; ++k) {
        const uint32_t q = k % kTcSched;
        if (!mbar_wait(smem_u32(sch_full + q), (k / kTcSched) & 1, sAbort)) break;
        const int u = sUnit[q];
        mbar_arrive(smem_u32(sch_empty + q));
        if (u < 0) break;
        const TcUnit x = decode_unit(u, num_seqs, H, num_pairs);
        const TcGeom g = unit_geom(x, cu_new, start_pos, total_new, max_new, max_ctx, R);
        const uint32_t abuf = k & 1;
        bool failed = false;
        if (!mbar_wait(smem_u32(a_conv + abuf), (k >> 1) & 1, sAbort)) break;
        tc_fence_after();
        for (int rt = 0; rt <= g.nrt && !failed; ++rt, ++item) {
          const uint32_t buf = item & 1;
          if (!mbar_wait(smem_u32(acc_empty + buf), ((item >> 1) & 1) ^ 1, sAbort)) { failed = true; break; }
          tc_fence_after();
          const uint32_t idesc = idesc_bf16_f32(kTcUnit, rt < g.nrt ? kRefTile : r2);
          for (int c = 0; c < CH; ++c, ++stage) {
            const uint32_t slot = stage % NS;
            if (!mbar_wait(smem_u32(b_full + slot), (stage / NS) & 1, sAbort)) { failed = true; break; }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(sA + (abuf * CH + c) * kTcStageBytes);
            const uint32_t b_addr = smem_u32(sB + slot * kTcStageBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_pair(tmem_base + buf * kRefTile, sw128_kmajor_desc(a_addr + kk * 32),
                             sw128_kmajor_desc(b_addr + kk * 32), idesc, (c | kk) != 0 ? 1u : 0u);
            umma_commit_pair(smem_u32(b_empty + slot), 0x3);
          }
          if (failed) break;
          umma_commit_pair(smem_u32(acc_full + buf), 0x3);
        }
        if (failed) break;
        umma_commit_pair(smem_u32(a_empty + abuf), 0x3);
      }
    }
  } else if (warp >= 2 + kTcEpiWarps) {
    // ---------------- converters (both CTAs): x~ = RNE_bf16(fp32(x) - mu) on this CTA's token rows ----------------
    const int cidx = (warp - 2 - kTcEpiWarps) * 32 + lane;  // 0..63
    const int qc = cidx & 7;   // logical 16-byte chunk (8 columns) within a 64-column K-chunk
    const int r0 = cidx >> 3;  // rows r0, r0 + 8, ..., r0 + 120
    for (uint32_t k = 0;; ++k) {
      const uint32_t q = k % kTcSched;
      const bool got = mbar_wait_cluster(smem_u32(sch_full + q), (k / kTcSched) & 1, sAbort);
      const int u = got ? sUnit[q] : -1;
      __syncwarp();
      if (got && lane == 0) mbar_arrive_cluster(lead_sch_empty + q * 8);  // release: orders the read above
      if (u < 0) break;
      const TcUnit x = decode_unit(u, num_seqs, H, num_pairs);
      const uint32_t abuf = k & 1;
      // mu of this lane's 8 columns in every K-chunk: [K columns | V columns] of kv head h
      const float4* muh4 = reinterpret_cast<const float4*>(mu + static_cast<int64_t>(x.h) * CH * 64);
      float m[CH][8];
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const float4 a = __ldg(muh4 + c * 16 + qc * 2), b = __ldg(muh4 + c * 16 + qc * 2 + 1);
        m[c][0] = a.x, m[c][1] = a.y, m[c][2] = a.z, m[c][3] = a.w;
        m[c][4] = b.x, m[c][5] = b.y, m[c][6] = b.z, m[c][7] = b.w;
      }
      if (!mbar_wait(smem_u32(a_full + abuf), (k >> 1) & 1, sAbort)) break;
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        uint8_t* tile = sA + (abuf * CH + c) * kTcStageBytes;
#pragma unroll 4
        for (int i = 0; i < kTcTileM / 8; ++i) {
          const int rr = r0 + 8 * i;
          uint4* p = reinterpret_cast<uint4*>(tile + rr * 128 + ((qc ^ (rr & 7)) << 4));  // 128-byte swizzle
          float f[8];
          unpack16(*p, f, static_cast<__nv_bfloat16*>(nullptr));
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = __fsub_rn(f[e], m[c][e]);  // IEEE fp32 subtract, then RNE to bf16
          *p = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                          pack_bf16x2(f[6], f[7]));
        }
      }
      fence_proxy_async_shared();  // the tensor cores read the tile through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_a_conv + abuf * 8);
    }
  } else {
    // ---------------- epilogue (both CTAs) ----------------
    const int ew = warp - 2;
    const int ch = ew >> 2;   // column half of each 256-column tile
    const int qd = warp & 3;  // tensor-memory lane quarter this warp may access
    const int row = qd * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(qd * 32) << 16);
    const int etid = ew * 32 + lane;  // 0..255: one 1/|r| value of each tile per thread
    uint32_t item = 0, ib = 0;
    for (uint32_t k = 0;; ++k) {
      const uint32_t q = k % kTcSched;
      // every exit of the epilogue loop is decided by an OR over all epilogue threads (uniform)
      const bool got = mbar_wait_cluster(smem_u32(sch_full + q), (k / kTcSched) & 1, sAbort);
      const int u = got ? sUnit[q] : -1;
      __syncwarp();
      if (got && lane == 0) mbar_arrive_remote(lead_sch_empty + q * 8);
      if (named_bar_or(1, kTcEpiWarps * 32, u < 0 || *sAbort)) break;
      const TcUnit x = decode_unit(u, num_seqs, H, num_pairs);
      const TcGeom g = unit_geom(x, cu_new, start_pos, total_new, max_new, max_ctx, R);
      const int nrt = g.nrt;
      const int64_t refrow0 = (static_cast<int64_t>(x.s) * H + x.h) * max_ref_pad;
      const int i = static_cast<int>(rank) * kTcTileM + row;
      const bool valid = i < g.n_here;
      const int t = g.t0 + i;
      const int jlim = valid ? ceil_div_i(t, R) : 0;
      float best = -INFINITY;
      int bj = 0;
      float tkv[KTm];  // KT > 0: the row's nearest references so far (value descending, then j ascending)
      int tkj[KTm];
#pragma unroll
      for (int k = 0; k < KTm; ++k) {
        tkv[k] = -INFINITY;
        tkj[k] = 0x7fffffff;
      }
      bool failed = false;
      // 1/|r_j| slices live in a two-slot shared buffer filled by the epilogue threads themselves, one tile
      // ahead, so the producer never waits on the epilogue.
      if (nrt > 0) {
        sInv[ib * kRefTile + etid] = __ldg(invn + refrow0 + etid);
        named_bar_sync(1, kTcEpiWarps * 32);
      }
      for (int rt = 0; rt < nrt; ++rt, ++item) {
        const uint32_t buf = item & 1;
        const float inv_next = rt + 1 < nrt ? __ldg(invn + refrow0 + (rt + 1) * kRefTile + etid) : 0.f;
        if (!mbar_wait(smem_u32(acc_full + buf), (item >> 1) & 1, sAbort)) failed = true;
        failed = __any_sync(0xffffffffu, failed);  // warp-uniform: tensor-memory loads are warp-collective
        tc_fence_after();
        const int jb = rt * kRefTile + ch * kTcHalfRefs;
        const int nval = min(kTcHalfRefs, max(jlim - jb, 0));  // visible columns of this half for this row
        const float4* inv4 = reinterpret_cast<const float4*>(sInv + ib * kRefTile + ch * kTcHalfRefs);
#pragma unroll 1
        for (int half = 0; half < 2 && !failed; ++half) {
          uint32_t v[64];
          tmem_ld_32x32b_x64(lane_base + buf * kRefTile + ch * kTcHalfRefs + half * 64, v);
          tmem_ld_wait();
          if (half == 1) {
            // the last read of this accumulator is done: release it before the arithmetic (the leader
            // counts both CTAs' warps)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(lead_acc_empty + buf * 8);
          }
          const int nv = nval - half * 64;  // visible columns in this part (may be <= 0 or >= 64)
          if (nv > 0) {
            if constexpr (KT == 0) {
              const uint32_t cm = part_max_tagged(v, inv4 + half * 16, nv);
              // compare without the tag: equal truncated scores keep the earlier part (smaller j)
              const float cmt = __uint_as_float(cm & ~63u);
              if (cmt > best) {
                best = cmt;
                bj = jb + half * 64 + (63 - static_cast<int>(cm & 63u));
              }
            } else {
              float cand[KTm];
              part_topk_tagged<KTm>(v, inv4 + half * 16, nv, cand);
#pragma unroll
              for (int c = 0; c < KTm; ++c) {
                if (cand[c] == -INFINITY) break;
                const uint32_t cb = __float_as_uint(cand[c]);
                topk_insert<KTm>(tkv, tkj, __uint_as_float(cb & ~63u), jb + half * 64 + (63 - static_cast<int>(cb & 63u)));
              }
            }
          }
        }
        // (the accumulator buffer was released after its last read above)
        // publish the next slice; the barrier also retires every warp's reads of the current slot
        if (rt + 1 < nrt) sInv[(ib ^ 1) * kRefTile + etid] = inv_next;
        ib ^= 1;
        if (named_bar_or(1, kTcEpiWarps * 32, failed || *sAbort)) {
          failed = true;
          break;
        }
      }
      if (failed) break;  // uniform (decided by the barrier above)
      // merge the two column halves: the larger score wins, equal scores go to the smaller index
      int jsl[KTm];  // KT > 0: chosen ordinals, ascending; nslot of them are filled
      int nslot = 1;
      if constexpr (KT == 0) {
        sBest[ch * kTcTileM + row] = best;
        sBj[ch * kTcTileM + row] = bj;
        named_bar_sync(1, kTcEpiWarps * 32);
        {
          const float b0 = sBest[row], b1 = sBest[kTcTileM + row];
          const int j0 = sBj[row], j1 = sBj[kTcTileM + row];
          bj = (b1 > b0 || (b1 == b0 && j1 < j0)) ? j1 : j0;
        }
        named_bar_sync(1, kTcEpiWarps * 32);  // merge slots are free for the next unit
      } else {
#pragma unroll
        for (int k = 0; k < KT; ++k) {
          sBest[(ch * kTcTileM + row) * KT + k] = tkv[k];
          sBj[(ch * kTcTileM + row) * KT + k] = tkj[k];
        }
        named_bar_sync(1, kTcEpiWarps * 32);
#pragma unroll
        for (int k = 0; k < KT; ++k) {  // both halves' threads form the same merged list
          const float ov = sBest[((ch ^ 1) * kTcTileM + row) * KT + k];
          if (ov != -INFINITY) topk_insert<KTm>(tkv, tkj, ov, sBj[((ch ^ 1) * kTcTileM + row) * KT + k]);
        }
        named_bar_sync(1, kTcEpiWarps * 32);  // merge slots are free for the next unit
        // the filled slots in ascending ordinal order (unfilled ones sort last as the largest key)
        nslot = 0;
#pragma unroll
        for (int k = 0; k < KT; ++k) {
          jsl[k] = tkv[k] != -INFINITY ? tkj[k] : 0x7fffffff;
          nslot += tkv[k] != -INFINITY;
        }
#pragma unroll
        for (int a2 = 0; a2 < KT; ++a2)
#pragma unroll
          for (int b2 = 0; b2 + 1 < KT - a2; ++b2) {
            const int lo = min(jsl[b2], jsl[b2 + 1]), hi = max(jsl[b2], jsl[b2 + 1]);
            jsl[b2] = lo;
            jsl[b2 + 1] = hi;
          }
      }
      // projection item: codes.  Column half ch writes the K (ch = 0) or V (ch = 1) code of its row; the
      // PR row loads are issued before the wait.  A failed wait only skips the work; the next loop head
      // leaves uniformly.
      const bool isref = valid && (t % R) == 0;
      const int js = isref ? t / R : bj;
      if constexpr (KT > 0) {
        if (isref) {
          nslot = KT;
#pragma unroll
          for (int k = 0; k < KT; ++k) jsl[k] = t / R;
        }
      }
      constexpr int kMaxR4 = 16;  // r <= 64: at most two 32-column chunks
      float4 prv[8];              // PR values of the current 32-column chunk (the first is loaded ahead)
      const float4* prow4 = reinterpret_cast<const float4*>(pr + (refrow0 + js) * r2 + ch * r);
      // KT > 0: the chunk's PR values are the mean over the filled slots (r >= 32)
      auto load_mean_pr = [&](int cc) {
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) prv[e4] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < KTm; ++k) {
          if (k >= nslot) break;
          const float4* p4 = reinterpret_cast<const float4*>(pr + (refrow0 + jsl[k]) * r2 + ch * r + cc * 32);
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 x4 = __ldg(p4 + e4);
            prv[e4].x += x4.x;
            prv[e4].y += x4.y;
            prv[e4].z += x4.z;
            prv[e4].w += x4.w;
          }
        }
        const float inv = nslot > 0 ? 1.f / static_cast<float>(nslot) : 0.f;
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          prv[e4].x *= inv;
          prv[e4].y *= inv;
          prv[e4].z *= inv;
          prv[e4].w *= inv;
        }
      };
      if constexpr (KT == 0) {
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4)
          if (e4 < r / 4 && valid) prv[e4] = __ldg(prow4 + e4);
      } else {
        if (valid) load_mean_pr(0);
      }
      const int pb = valid ? lookup_block(block_tables, max_blocks, num_blocks, x.s, t / R) : -1;
      const uint32_t buf = item & 1;
      ++item;
      if (__any_sync(0xffffffffu, !mbar_wait(smem_u32(acc_full + buf), ((item - 1) >> 1) & 1, sAbort))) continue;
      tc_fence_after();
      if constexpr (Q4) {
        // 4-bit codes: the half's r codes are collected first (their largest magnitude sets the scale
        // s = RNE_bf16(max / 7)), then quantised to levels -7..7, packed into nibble words (nibble k of a word
        // holds code 2k, nibble k + 4 code 2k + 1) and stored with the scale.
        float cq[kMaxR4 * 4];
#pragma unroll
        for (int cc = 0; cc < kMaxR4 / 8; ++cc) {
          if (cc * 32 >= r) break;  // warp-uniform; r >= 32 with 4-bit codes
          uint32_t pv[32];
          tmem_ld_32x32b_x32(lane_base + buf * kRefTile + ch * r + cc * 32, pv);
          tmem_ld_wait();
          if ((cc + 1) * 32 >= r) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(lead_acc_empty + buf * 8);
          }
          if (cc > 0 && pb >= 0) {
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) prv[e4] = __ldg(prow4 + cc * 8 + e4);
          }
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 p4 = prv[e4];
            const int e = cc * 32 + e4 * 4;
            cq[e + 0] = isref ? 0.f : __fsub_rn(__uint_as_float(pv[e4 * 4 + 0]), p4.x);
            cq[e + 1] = isref ? 0.f : __fsub_rn(__uint_as_float(pv[e4 * 4 + 1]), p4.y);
            cq[e + 2] = isref ? 0.f : __fsub_rn(__uint_as_float(pv[e4 * 4 + 2]), p4.z);
            cq[e + 3] = isref ? 0.f : __fsub_rn(__uint_as_float(pv[e4 * 4 + 3]), p4.w);
          }
        }
        if (pb >= 0) {
          float mx = 0.f;
#pragma unroll
          for (int e = 0; e < kMaxR4 * 4; ++e)
            if (e < r) mx = fmaxf(mx, fabsf(cq[e]));
          const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(mx, 7.0f));
          const float sc = __bfloat162float(sb);
          uint8_t* cell = reinterpret_cast<uint8_t*>(codes) + (static_cast<int64_t>(pb) * H + x.h) * R * (r + 4);
          uint32_t wq[kMaxR4 / 2];  // r / 8 nibble words of this half
#pragma unroll
          for (int w = 0; w < kMaxR4 / 2; ++w) {
            wq[w] = 0u;
            if (w * 8 < r) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                wq[w] |= (q4_nibble(cq[8 * w + 2 * k], sc) << (4 * k)) |
                         (q4_nibble(cq[8 * w + 2 * k + 1], sc) << (4 * k + 16));
            }
          }
          uint4* dst = reinterpret_cast<uint4*>(cell + (t % R) * r + ch * (r / 2));
#pragma unroll
          for (int u = 0; u < kMaxR4 / 8; ++u)
            if (u * 16 < r / 2) dst[u] = make_uint4(wq[4 * u], wq[4 * u + 1], wq[4 * u + 2], wq[4 * u + 3]);
          reinterpret_cast<__nv_bfloat16*>(cell + R * r)[(t % R) * 2 + ch] = sb;
        }
      } else {
        __nv_bfloat16* cdst = pb >= 0 ? codes + ((static_cast<int64_t>(pb) * H + x.h) * R + t % R) * r2 + ch * r : nullptr;
        // the accumulator is released right after its last read, before the last chunk's subtraction and stores
  #pragma unroll
        for (int cc = 0; cc < kMaxR4 / 8; ++cc) {
          if (cc * 32 >= r) break;  // warp-uniform
          uint32_t pv[32];
          if (r >= 32) {
            tmem_ld_32x32b_x32(lane_base + buf * kRefTile + ch * r + cc * 32, pv);
          } else {
            tmem_ld_32x32b_x16(lane_base + buf * kRefTile + ch * r, pv);
          }
          tmem_ld_wait();
          if ((cc + 1) * 32 >= r) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(lead_acc_empty + buf * 8);
          }
          if (cc > 0 && pb >= 0) {
            if constexpr (KT > 0) {
              load_mean_pr(cc);
            } else {
  #pragma unroll
              for (int e4 = 0; e4 < 8; ++e4) prv[e4] = __ldg(prow4 + cc * 8 + e4);
            }
          }
          if (pb >= 0) {
            const int nc = r < 32 ? r : 32;
            uint4* dst4 = reinterpret_cast<uint4*>(cdst + cc * 32);
  #pragma unroll
            for (int e8 = 0; e8 < 4; ++e8) {  // 8 codes per 16-byte store
              if (e8 * 8 >= nc) break;
              uint32_t w[4];
  #pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                const float4 p4 = prv[e8 * 2 + h2];
                const int e = e8 * 8 + h2 * 4;
                const float c0 = isref ? 0.f : __fsub_rn(__uint_as_float(pv[e + 0]), p4.x);
                const float c1 = isref ? 0.f : __fsub_rn(__uint_as_float(pv[e + 1]), p4.y);
                const float c2 = isref ? 0.f : __fsub_rn(__uint_as_float(pv[e + 2]), p4.z);
                const float c3 = isref ? 0.f : __fsub_rn(__uint_as_float(pv[e + 3]), p4.w);
                w[h2 * 2] = pack_bf16x2(c0, c1);
                w[h2 * 2 + 1] = pack_bf16x2(c2, c3);
              }
              dst4[e8] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
      if constexpr (KT == 0) {
        if (ch == 0 && pb >= 0) ref_idx[(static_cast<int64_t>(pb) * H + x.h) * R + t % R] = js;
      } else {
        if (ch == 0 && pb >= 0) {
          int* dst = ref_idx + ((static_cast<int64_t>(pb) * H + x.h) * R + t % R) * KT;
#pragma unroll
          for (int k = 0; k < KT; ++k) dst[k] = k < nslot ? jsl[k] : -1;
        }
      }
    }
  }

  // No role of either CTA touches the other's shared memory or the pair's tensor memory past this point.
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// ------------------------------------------------------------------------------------------------
// Host side.
// ------------------------------------------------------------------------------------------------
}  // namespace dkv
#include "append.cuh"
namespace dkv {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 map over a row-major [rows][cols] array; boxes of [box_rows][64] with the 128-byte swizzle.
static bool make_map_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int CH, bool Q4, int KT>
static dkv_status launch_tc(const CompressArgs& a, const CompressWs& L, uint8_t* ws, cudaStream_t st) {
  const dkv_shape& sh = *a.shape;
  const int H = sh.num_kv_heads, d2 = 2 * sh.head_dim, r2 = 2 * sh.rank;
  CUtensorMap k_map, v_map, refc_map, bd_map;
  // raw new tokens as [total_new rows][H_kv * d columns]; a box is 128 tokens x 64 columns of one head
  if (!make_map_bf16(&k_map, a.k_new, static_cast<uint64_t>(H) * sh.head_dim, static_cast<uint64_t>(a.total_new),
                     kTcTileM) ||
      !make_map_bf16(&v_map, a.v_new, static_cast<uint64_t>(H) * sh.head_dim, static_cast<uint64_t>(a.total_new),
                     kTcTileM) ||
      !make_map_bf16(&refc_map, ws + L.refc, d2, static_cast<uint64_t>(a.num_seqs) * H * L.max_ref_pad,
                     kTcHalfRefs) ||
      !make_map_bf16(&bd_map, ws + L.bd, d2, static_cast<uint64_t>(H) * r2, r2 / 2))
    return DKV_ERR_CUDA;
  const int smem = TcConfig<CH, KT>::kSmemBytes;
  // once per device (no attribute calls or occupancy queries inside stream captures): the shared-memory
  // limit, and how many two-CTA clusters of this kernel fit on the device at once
  static std::mutex mc_mu;
  static int mc_dev[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DKV_ERR_CUDA;
  int max_clusters = 0;
  {
    std::lock_guard<std::mutex> lock(mc_mu);
    if (dev < 64) max_clusters = mc_dev[dev];
  }
  if (max_clusters == 0) {
    if (!ensure_max_dynamic_smem<search_tc_kernel<CH, Q4, KT>>()) return DKV_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, search_tc_kernel<CH, Q4, KT>, &cfg) != cudaSuccess || n <= 0) return DKV_ERR_CUDA;
    max_clusters = n;
    std::lock_guard<std::mutex> lock(mc_mu);
    if (dev < 64) mc_dev[dev] = n;
  }
  const int num_pairs = static_cast<int>(ceil_div64(a.max_new, kTcUnit));
  const int64_t units = static_cast<int64_t>(num_pairs) * a.num_seqs * H;
  if (units > INT32_MAX / 2) return DKV_ERR_UNSUPPORTED;
  const int grid = 2 * static_cast<int>(units < max_clusters ? units : max_clusters);
  int* counter = reinterpret_cast<int*>(ws + L.counter);
  if (cudaMemsetAsync(counter, 0, sizeof(int), st) != cudaSuccess) return DKV_ERR_CUDA;
  prof_begin(DKV_KERNEL_SEARCH, st);
    search_tc_kernel<CH, Q4, KT><<<grid, kTcThreads, smem, st>>>(
      k_map, v_map, refc_map, bd_map, a.params->mu, reinterpret_cast<const float*>(ws + L.invn),
      reinterpret_cast<const float*>(ws + L.pr), a.cu_new, a.start_pos, a.block_tables, a.max_blocks,
      a.cache->num_blocks, a.num_seqs, H, sh.ref_stride, sh.rank, a.total_new, L.max_ref_pad, a.max_new,
      a.max_ctx, num_pairs, counter, static_cast<__nv_bfloat16*>(a.cache->codes), a.cache->ref_idx);
    prof_end(DKV_KERNEL_SEARCH, st);
  return DKV_OK;
}

template <typename T, int D, int RK>
static dkv_status launch_compress_t(const CompressArgs& a, uint8_t* ws, cudaStream_t st) {
  const dkv_shape& sh = *a.shape;
  const int H = sh.num_kv_heads, R = sh.ref_stride;
  const CompressWs L = compress_ws_layout(sh, a.num_seqs, a.total_new, a.max_ctx);
  T* xt = reinterpret_cast<T*>(ws + L.xt);
  T* refc = reinterpret_cast<T*>(ws + L.refc);
  float* invn = reinterpret_cast<float*>(ws + L.invn);
  float* pr = reinterpret_cast<float*>(ws + L.pr);
  constexpr bool kTensorCores = sizeof(T) == 2;
  // 1. centre
  {
    using CC = CenterCfg<T, D>;
    // the tensor-core path centres its token tiles inside the search kernel: only reference rows here
    const int64_t rows = kTensorCores ? ceil_div64(a.max_new, R) : a.max_new;
    dim3 grid(static_cast<unsigned>(ceil_div64(rows * H, CC::ROWS)), a.num_seqs);
    prof_begin(DKV_KERNEL_CENTER, st);
    center_kernel<T, D, kTensorCores><<<grid, 256, 0, st>>>(
        static_cast<const T*>(a.k_new), static_cast<const T*>(a.v_new), a.params->mu, a.cu_new, a.start_pos,
        a.block_tables, a.max_blocks, a.cache->num_blocks, H, R, a.total_new, a.max_new, a.max_ctx, xt,
        static_cast<T*>(a.cache->refs));
    prof_end(DKV_KERNEL_CENTER, st);
  }
  // 2'. small appends (bf16 cosine search, at most kAppendMaxNew new tokens per sequence): search and codes
  //     over the paged reference rows on CUDA cores, with no reference prep
  if constexpr (kTensorCores) {
    if (!is_q4(sh) && a.topk == 0 && a.max_new <= kAppendMaxNew) {
      // one 64-bit (score, index) key per (sequence, kv head, new token) over the inverse-norm area, which
      // this path does not use (it holds at least kRefTile floats per (sequence, kv head))
      unsigned long long* keys = reinterpret_cast<unsigned long long*>(ws + L.invn);
      const size_t kbytes = static_cast<size_t>(a.num_seqs) * H * a.max_new * sizeof(unsigned long long);
      if (a.max_new > 0) {
        if (cudaMemsetAsync(keys, 0, kbytes, st) != cudaSuccess) return DKV_ERR_CUDA;
        const int64_t nref = max_refs(a.max_ctx, R);
        prof_begin(DKV_KERNEL_SEARCH, st);
        if (nref > 0) {
          dim3 g1(static_cast<unsigned>(ceil_div64(nref, kAppendRefs)), H, a.num_seqs);
          append_search_kernel<D><<<g1, kAppendRefs, 0, st>>>(
              static_cast<const __nv_bfloat16*>(a.k_new), static_cast<const __nv_bfloat16*>(a.v_new), a.params->mu,
              static_cast<const __nv_bfloat16*>(a.cache->refs), a.cu_new, a.start_pos, a.block_tables, a.max_blocks,
              a.cache->num_blocks, H, R, a.total_new, a.max_new, a.max_ctx, keys);
        }
        dim3 g2(static_cast<unsigned>(a.max_new), H, a.num_seqs);
        append_codes_kernel<D, RK><<<g2, kAppendCodeThreads, 0, st>>>(
            static_cast<const __nv_bfloat16*>(a.k_new), static_cast<const __nv_bfloat16*>(a.v_new), a.params->mu,
            static_cast<const __nv_bfloat16*>(a.params->basis), static_cast<const __nv_bfloat16*>(a.cache->refs),
            a.cu_new, a.start_pos, a.block_tables, a.max_blocks, a.cache->num_blocks, H, R, a.total_new, a.max_new,
            a.max_ctx, keys, static_cast<__nv_bfloat16*>(a.cache->codes), a.cache->ref_idx);
        prof_end(DKV_KERNEL_SEARCH, st);
      }
      return DKV_OK;
    }
  }
  // 2. reference prep (+ the blockdiag basis operand on the tensor-core path)
  {
    const int nref = max_refs(a.max_ctx, R);
    dim3 grid(static_cast<unsigned>(ceil_div64(nref, kPrepRefs)), H, a.num_seqs);
    if (kTensorCores ? !ensure_max_dynamic_smem<refprep_tc_kernel<D, RK>>()
                     : !ensure_max_dynamic_smem<refprep_kernel<T, D, RK>>())
      return DKV_ERR_CUDA;
    prof_begin(DKV_KERNEL_REFPREP, st);
    if constexpr (kTensorCores) {
      refprep_tc_kernel<D, RK><<<grid, 256, PrepTcCfg<D, RK>::SMEM, st>>>(
          static_cast<const __nv_bfloat16*>(a.cache->refs), static_cast<const __nv_bfloat16*>(a.params->basis),
          a.cu_new, a.start_pos, a.block_tables, a.max_blocks, a.cache->num_blocks, H, R, a.total_new, a.max_new,
          a.max_ctx, L.max_ref_pad, reinterpret_cast<__nv_bfloat16*>(refc), invn, pr,
          reinterpret_cast<__nv_bfloat16*>(ws + L.bd), a.topk > 0 ? 1 : 0);
    } else {
      refprep_kernel<T, D, RK><<<grid, 256, PrepCfg<T, D, RK>::SMEM, st>>>(
          static_cast<const T*>(a.cache->refs), static_cast<const T*>(a.params->basis), a.cu_new, a.start_pos,
          a.block_tables, a.max_blocks, a.cache->num_blocks, H, R, a.total_new, a.max_new, a.max_ctx, L.max_ref_pad,
          refc, invn, pr, nullptr);
    }
    prof_end(DKV_KERNEL_REFPREP, st);
  }
  // 3. search + codes
  if constexpr (kTensorCores) {
    constexpr int CH = D == 64 ? 2 : 4;
    if (is_q4(*a.shape)) return launch_tc<CH, true, 0>(a, L, ws, st);
    switch (a.topk) {
      case 0: return launch_tc<CH, false, 0>(a, L, ws, st);
      case 1: return launch_tc<CH, false, 1>(a, L, ws, st);
      case 2: return launch_tc<CH, false, 2>(a, L, ws, st);
      case 4: return launch_tc<CH, false, 4>(a, L, ws, st);
    }
    return DKV_ERR_UNSUPPORTED;
  } else {
    const int d = D, r = RK;
    dim3 grid(static_cast<unsigned>(ceil_div64(a.max_new, kSimtTok)), H, a.num_seqs);
    const size_t smem = (static_cast<size_t>(2 * d) * kSimtTok + kSimtRefs * 2 * d + kSimtRefs) * sizeof(float);
    if (!ensure_max_dynamic_smem<search_simt_kernel<T>>()) return DKV_ERR_CUDA;
    prof_begin(DKV_KERNEL_SEARCH, st);
    search_simt_kernel<T><<<grid, kSimtTok, smem, st>>>(
        xt, refc, invn, static_cast<const T*>(a.params->basis), a.cu_new, a.start_pos, a.block_tables,
        a.max_blocks, a.cache->num_blocks, H, d, r, R, a.total_new, a.max_new, a.max_ctx, L.max_ref_pad,
        static_cast<T*>(a.cache->codes), a.cache->ref_idx);
    prof_end(DKV_KERNEL_SEARCH, st);
  }
  return DKV_OK;
}

template <typename T, int D>
static dkv_status launch_compress_d(const CompressArgs& a, uint8_t* ws, cudaStream_t st) {
  switch (a.shape->rank) {
    case 16: return launch_compress_t<T, D, 16>(a, ws, st);
    case 32: return launch_compress_t<T, D, 32>(a, ws, st);
    case 64: return launch_compress_t<T, D, 64>(a, ws, st);
  }
  return DKV_ERR_UNSUPPORTED;
}

template <typename T>
static dkv_status launch_compress_dt(const CompressArgs& a, uint8_t* ws, cudaStream_t st) {
  return a.shape->head_dim == 64 ? launch_compress_d<T, 64>(a, ws, st) : launch_compress_d<T, 128>(a, ws, st);
}

dkv_status launch_compress(const CompressArgs& a, void* workspace, cudaStream_t st) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const dkv_status s = a.shape->dtype == DKV_F32 ? launch_compress_dt<float>(a, ws, st)
                                                 : launch_compress_dt<__nv_bfloat16>(a, ws, st);
  if (s != DKV_OK) return s;
  return cudaGetLastError() == cudaSuccess ? DKV_OK : DKV_ERR_CUDA;
}

}  // namespace dkv
