// DeltaKV decode attention over the compressed, paged cache on sm_100a.
//
// Summary (en) §3 "Reconstruction": KV^ = f_d(z) + KV^R with a linear decompressor f_d(z) = z B^T, plus
// the shared component mu; "Sparse-vLLM Integration": tokens are rebuilt on demand inside attention.
// Here nothing is rebuilt in memory at all.  For kv head h, query head g and token t with reference
// j = ref_idx(t) and codes (cK, cV):
//     q.K^_t   = q.mu_K + q.r~K_j + (q B_K).cK_t
//     sum_t p_t V^_t = (sum p) mu_V + sum_j w_j r~V_j + (sum_t p_t cV_t) B_V^T,   w_j = sum_{t: ref(t)=j} p_t
// so the per-token work is two r-wide dot products on the codes (HBM-bound stream of 2r values + one
// index per token) and one add into the per-reference mass w_j.
//
//   decode_prologue_kernel  qp = q B_K, qmu = q.mu_K, sref_j = q.r~K_j  (all scaled by scale*log2 e)
//   decode_split_kernel     split-K over tokens: bulk copies of whole paged blocks into a shared-memory
//                           ring (one producer warp), 8 consumer warps with 4 lanes per token; per stage
//                           the scores are formed, the CTA-wide running max is raised only when a stage
//                           exceeds it by more than 2^4 (then acc, l and the mass bins are rescaled), and
//                           p, l, acc = sum p cV and bins[j] += p are accumulated.  For bf16 with r in
//                           {32, 64} decode_split_mma_kernel does the same with the two per-token
//                           contractions on the tensor cores.
//   decode_combine_kernel   merges the splits (max / sum-exp), forms sum_j w_j r~V_j per chunk of
//                           references; the last chunk CTA of a (seq, kv head) adds acc B_V^T and mu,
//                           divides by the softmax mass and writes out and lse.
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "layout.h"

namespace dkv {

__device__ __forceinline__ int ceil_div_d(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ int checked_ctx(const int* context_lens, int s, int max_ctx) {
  const int T = __ldg(context_lens + s);
  if (T < 0 || T > max_ctx) {
    record_error(DKV_DEVERR_BOUNDS);
    return 0;
  }
  return T;
}

// Extent of one sequence for the split kernels.  Dense decode runs its splits over the context's positions
// 0 .. ctx-1; sparse decode (a caller-given token list per sequence) runs them over the list's entries
// sel[sel0 .. sel0 + n - 1], whose tokens may point at any of the context's references.
struct SeqExtent {
  int ctx;   // cached tokens of the sequence
  int n;     // entries the splits run over: ctx (dense) or the length of the selected list (sparse)
  int sel0;  // first list entry of the sequence (sparse)
};

template <bool SPARSE>
__device__ __forceinline__ SeqExtent seq_extent(const int* context_lens, const int* cu_sel, int s, int max_ctx,
                                                int max_sel) {
  SeqExtent e;
  e.ctx = checked_ctx(context_lens, s, max_ctx);
  e.n = e.ctx;
  e.sel0 = 0;
  if constexpr (SPARSE) {
    const int a = __ldg(cu_sel + s), b = __ldg(cu_sel + s + 1);
    e.n = b - a;
    e.sel0 = a;
    if (a < 0 || e.n < 0 || e.n > max_sel) {
      record_error(DKV_DEVERR_BOUNDS);
      e.n = 0;
      e.sel0 = 0;
    }
  }
  return e;
}

// References a split's tokens may index: those before its last token (dense), or all of the context's
// (sparse, where a split's listed tokens may lie anywhere in the context).
template <bool SPARSE>
__device__ __forceinline__ int split_jcap(const SeqExtent& e, int t_end, int R) {
  return SPARSE ? ceil_div_d(e.ctx, R) : ceil_div_d(t_end, R);
}

// Position of list entry `e` of a sparse item, range-checked against the context (an entry outside it is
// recorded and replaced by position 0).
__device__ __forceinline__ int checked_pos(const int* list, int e, int ctx) {
  int p = __ldg(list + e);
  if (p < 0 || p >= ctx) {
    record_error(DKV_DEVERR_BOUNDS);
    p = 0;
  }
  return p;
}

__device__ __forceinline__ int checked_block(const int* block_tables, int max_blocks, int num_blocks, int s,
                                             int lb) {
  const int pb = __ldg(block_tables + static_cast<int64_t>(s) * max_blocks + lb);
  if (pb < 0 || pb >= num_blocks) {
    record_error(DKV_DEVERR_BLOCK_ID);
    return 0;  // read a valid block instead; the error word reports the bad table
  }
  return pb;
}

// Loads N consecutive storage elements (N * sizeof(T) a multiple of 8 bytes, 8-byte aligned) as fp32.
template <typename T, int N>
__device__ __forceinline__ void load_elems(const T* p, float (&f)[N]) {
  constexpr int BYTES = N * static_cast<int>(sizeof(T));
  if constexpr (BYTES % 16 == 0) {
    const uint4* p4 = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int u = 0; u < BYTES / 16; ++u) {
      const uint4 v = p4[u];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if constexpr (sizeof(T) == 2) {
          f[u * 8 + 2 * q] = __uint_as_float(w[q] << 16);
          f[u * 8 + 2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
        } else {
          f[u * 4 + q] = __uint_as_float(w[q]);
        }
      }
    }
  } else {
    const uint2* p2 = reinterpret_cast<const uint2*>(p);
#pragma unroll
    for (int u = 0; u < BYTES / 8; ++u) {
      const uint2 v = p2[u];
      const uint32_t w[2] = {v.x, v.y};
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if constexpr (sizeof(T) == 2) {
          f[u * 4 + 2 * q] = __uint_as_float(w[q] << 16);
          f[u * 4 + 2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
        } else {
          f[u * 2 + q] = __uint_as_float(w[q]);
        }
      }
    }
  }
}

// ------------------------------------------------------------------------------------------------
// Prologue, fp32.  CTA = (128 references, kv head, sequence), 128 threads.  Each warp takes 32 references,
// whose K rows are read as coalesced 16-byte vectors (D / V lanes per row), all issued before any is used;
// every lane forms the G partial dot products of its vector with the staged queries and a shuffle
// reduction over the row's lanes finishes them.  CTA 0 of each (seq, kv head) also forms q B_K and
// q . mu_K, with B_K staged through shared memory.  (bf16 has its own kernel below.)
// ------------------------------------------------------------------------------------------------
constexpr int kProRefs = 128;

template <typename T, int D, int G>
__global__ void __launch_bounds__(kProRefs) decode_prologue_kernel(
    const T* __restrict__ q, const float* __restrict__ mu, const T* __restrict__ basis, const T* __restrict__ refs,
    const int* __restrict__ context_lens, const int* __restrict__ block_tables, int max_blocks, int num_blocks,
    int Hq, int H, int r, int R, int max_ctx, int max_ref, float scale2, float* __restrict__ qp,
    float* __restrict__ qmu, float* __restrict__ sref) {
  static_assert(sizeof(T) == 4, "fp32 storage");
  constexpr int V = 16 / sizeof(T);
  constexpr int TPR = D / V;      // lanes per K row: 8, 16 or 32
  constexpr int RPW = 32 / TPR;   // rows per warp-wide load
  constexpr int NIT = 32 / RPW;   // loads per lane for the warp's 32 references
  extern __shared__ float sm_pro[];
  // the split kernel may start now: its code stream does not depend on this kernel's outputs
  griddep_launch_dependents();
  {
    // fp32: the K rows stay in registers and every lane forms partial dot products with the staged queries
    float* qs = sm_pro;        // [G][D]
    float* bks = qs + G * D;   // [D][r] then mu_K [D] (CTA 0 only)
    const int s = blockIdx.z, h = blockIdx.y, j0 = blockIdx.x * kProRefs;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ctx = checked_ctx(context_lens, s, max_ctx);
    const int n_ref = ceil_div_d(ctx, R);
    if (blockIdx.x != 0 && j0 >= n_ref) return;
    const int wj0 = j0 + warp * 32;  // this warp's first reference
    const int pbl = wj0 + lane < n_ref ? checked_block(block_tables, max_blocks, num_blocks, s, wj0 + lane) : 0;
    const int sub = lane % TPR;      // this lane's 16-byte vector within a row
    uint4 xv[NIT];
#pragma unroll
    for (int it = 0; it < NIT; ++it) {
      const int rr = it * RPW + lane / TPR;  // reference wj0 + rr
      const int pb = __shfl_sync(0xffffffffu, pbl, rr);
      const uint4* src = reinterpret_cast<const uint4*>(refs + (static_cast<int64_t>(pb) * H + h) * 2 * D) + sub;
      if (wj0 + rr < n_ref) xv[it] = __ldg(src);
    }
    const T* qsrc = q + (static_cast<int64_t>(s) * Hq + h * G) * D;
    for (int e = tid; e < G * D / V; e += kProRefs) {
      float x[V];
      load_elems<T, V>(qsrc + e * V, x);
#pragma unroll
      for (int c = 0; c < V; ++c) qs[e * V + c] = x[c];
    }
    if (blockIdx.x == 0) {
      // B_K [D][r] and mu_K staged with all loads in flight (at most 64 / 128 + 1 per thread)
      constexpr int NBK = (D * 64 / V + kProRefs - 1) / kProRefs;
      const uint4* bk4 = reinterpret_cast<const uint4*>(basis + static_cast<int64_t>(h) * 2 * D * r);
      const int nbk = D * r / V;
      uint4 xb[NBK];
#pragma unroll
      for (int u = 0; u < NBK; ++u)
        if (tid + u * kProRefs < nbk) xb[u] = __ldg(bk4 + tid + u * kProRefs);
      const float mk = __ldg(mu + static_cast<int64_t>(h) * 2 * D + (tid % D));
#pragma unroll
      for (int u = 0; u < NBK; ++u) {
        if (tid + u * kProRefs < nbk) {
          float x[V];
          unpack16(xb[u], x, static_cast<T*>(nullptr));
#pragma unroll
          for (int c = 0; c < V; ++c) bks[(tid + u * kProRefs) * V + c] = x[c];
        }
      }
      if (tid < D) bks[D * r + tid] = mk;
    }
    __syncthreads();
    if (blockIdx.x == 0) {
      for (int e = tid; e < G * r; e += kProRefs) {
        const int g = e / r, o = e % r;
        float a = 0.f;
#pragma unroll 8
        for (int k = 0; k < D; ++k) a = fmaf(qs[g * D + k], bks[k * r + o], a);
        qp[(static_cast<int64_t>(s) * Hq + h * G + g) * r + o] = a * scale2;
      }
      if (tid < G) {
        const float* mks = bks + D * r;
        float a = 0.f;
#pragma unroll 8
        for (int k = 0; k < D; ++k) a = fmaf(qs[tid * D + k], mks[k], a);
        qmu[static_cast<int64_t>(s) * Hq + h * G + tid] = a * scale2;
      }
    }
    if (wj0 >= n_ref) return;  // warp-uniform
    float* dst0 = sref + ((static_cast<int64_t>(s) * H + h) * max_ref) * G;
#pragma unroll
    for (int it = 0; it < NIT; ++it) {
      const int rr = it * RPW + lane / TPR;
      const bool ok = wj0 + rr < n_ref;
      float x[V];
      if (ok) {
        unpack16(xv[it], x, static_cast<T*>(nullptr));
      } else {
#pragma unroll
        for (int c = 0; c < V; ++c) x[c] = 0.f;
      }
      float part[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float4* q4 = reinterpret_cast<const float4*>(qs + g * D + sub * V);
        float a = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < V / 4; ++c4) {
          const float4 qq = q4[c4];
          a = fmaf(x[4 * c4 + 0], qq.x, a);
          a = fmaf(x[4 * c4 + 1], qq.y, a);
          a = fmaf(x[4 * c4 + 2], qq.z, a);
          a = fmaf(x[4 * c4 + 3], qq.w, a);
        }
#pragma unroll
        for (int o = TPR / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        part[g] = a;
      }
      if (ok && sub == 0) {
        float* dst = dst0 + static_cast<int64_t>(wj0 + rr) * G;
#pragma unroll
        for (int g = 0; g < G; ++g) dst[g] = part[g] * scale2;
      }
    }
  }
}

// ------------------------------------------------------------------------------------------------
// Prologue, bf16.  One launch, two kinds of CTA (128 threads each):
//   blockIdx.x <  S * H_kv   q B_K and q . mu_K of one (sequence, kv head).  q, B_K and mu_K are staged in
//                            shared memory by cp.async; each thread forms whole outputs with fp32 FMAs in
//                            dimension order.
//   blockIdx.x >= S * H_kv   q . r~K_j on 16-reference tiles.  A warp task is kProTaskTiles consecutive
//                            tiles of one (sequence, kv head); warps take tasks grid-stride and keep two
//                            tiles' K rows in flight while they multiply.
// No K row passes through shared memory.  Lane (g, t) of the m16n8k16 fragment loads, as 16-byte vectors,
// the 8-dimension chunks c = t, t + 4, ... of rows g and g + 8 of the tile.  Chunk c = t + 4m holds the A
// values of k-steps 2m and 2m + 1 under the dimension order
//     k-step 2m + e, k-values {2t, 2t+1, 2t+8, 2t+9}  <->  dimensions 8(t + 4m) + 4e + {0, 1, 2, 3}.
// q (exact in bf16, heads as the 8 columns of B) is laid out in the same order, so the contraction is the
// plain dot product over all dimensions, with the MMA's fp32 accumulation.
// ------------------------------------------------------------------------------------------------
constexpr int kProThreads = 128;
constexpr int kProTaskTiles = 4;  // 16-reference tiles per warp task of the bf16 prologue

template <int D, int G>
__global__ void __launch_bounds__(kProThreads) decode_prologue_tc_kernel(
    const __nv_bfloat16* __restrict__ q, const float* __restrict__ mu, const __nv_bfloat16* __restrict__ basis,
    const __nv_bfloat16* __restrict__ refs, const int* __restrict__ context_lens,
    const int* __restrict__ block_tables, int max_blocks, int num_blocks, int num_seqs, int Hq, int H, int r,
    int R, int max_ctx, int max_ref, float scale2, float* __restrict__ qp,
    float* __restrict__ qmu, float* __restrict__ sref) {
  static_assert(G <= 8, "the query heads of a group are the 8 columns of the B fragment");
  constexpr int NCH = D / 32;  // 16-byte chunks per lane and row (D / 8 chunks over the 4 lanes of a row)
  constexpr int NKS = D / 16;  // k-steps
  extern __shared__ __align__(16) unsigned char sm_pro_tc[];
  // the split kernel may start now: its code stream does not depend on this kernel's outputs
  griddep_launch_dependents();
  const int units = num_seqs * H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (static_cast<int>(blockIdx.x) < units) {
    // ---- q B_K [G][r] and q . mu_K [G] of one (sequence, kv head) ----
    const int s = blockIdx.x / H, h = blockIdx.x % H;
    __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(sm_pro_tc);  // [G][D]
    __nv_bfloat16* bks = qs + G * D;                                   // [D][r]
    float* mks = reinterpret_cast<float*>(bks + D * r);                // [D]
    const __nv_bfloat16* qsrc = q + (static_cast<int64_t>(s) * Hq + h * G) * D;
    const __nv_bfloat16* bk = basis + static_cast<int64_t>(h) * 2 * D * r;
    const float* mk = mu + static_cast<int64_t>(h) * 2 * D;
    for (int e = tid; e < G * D / 8; e += kProThreads) cp_async16(qs + e * 8, qsrc + e * 8);
    for (int e = tid; e < D * r / 8; e += kProThreads) cp_async16(bks + e * 8, bk + e * 8);
    for (int e = tid; e < D / 4; e += kProThreads) cp_async16(mks + e * 4, mk + e * 4);
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    for (int e = tid; e < G * r + G; e += kProThreads) {
      float acc = 0.f;
      if (e < G * r) {
        const int g = e / r, o = e % r;
#pragma unroll 8
        for (int k = 0; k < D; ++k)
          acc = fmaf(__bfloat162float(qs[g * D + k]), __bfloat162float(bks[k * r + o]), acc);
        qp[(static_cast<int64_t>(s) * Hq + h * G + g) * r + o] = acc * scale2;
      } else {
        const int g = e - G * r;
#pragma unroll 8
        for (int k = 0; k < D; ++k) acc = fmaf(__bfloat162float(qs[g * D + k]), mks[k], acc);
        qmu[static_cast<int64_t>(s) * Hq + h * G + g] = acc * scale2;
      }
    }
    return;
  }

  // ---- q . r~K_j over tasks of kProTaskTiles 16-reference tiles of one (sequence, kv head) ----
  // A task reads the context length, its block ids and q at once, then keeps two tiles' K rows in flight:
  // tile i + 2 is issued as soon as tile i is multiplied.
  const int gq = lane >> 2, tq = lane & 3;
  const int tasks_u = ceil_div_d(max_ref, 16 * kProTaskTiles);  // tasks per (sequence, kv head)
  const int64_t ntasks = static_cast<int64_t>(units) * tasks_u;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x - units) * (kProThreads / 32);
  for (int64_t task = static_cast<int64_t>(blockIdx.x - units) * (kProThreads / 32) + warp; task < ntasks;
       task += nwarps) {
    const int u = static_cast<int>(task / tasks_u);
    const int s = u / H, h = u % H;
    const int j0 = static_cast<int>(task % tasks_u) * (16 * kProTaskTiles);
    const int ctx = __ldg(context_lens + s);
    const int* bt = block_tables + static_cast<int64_t>(s) * max_blocks;
    // raw block ids of rows gq and gq + 8 of every tile, read while the context length is in flight
    // (j < max_ref <= max_blocks keeps them inside the table)
    int raw[kProTaskTiles][2];
#pragma unroll
    for (int i = 0; i < kProTaskTiles; ++i)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int j = j0 + 16 * i + gq + 8 * hr;
        raw[i][hr] = j < max_ref ? __ldg(bt + j) : 0;
      }
    const __nv_bfloat16* qsrc = q + (static_cast<int64_t>(s) * Hq + h * G + (gq < G ? gq : 0)) * D;
    uint4 qv[NCH];
#pragma unroll
    for (int m = 0; m < NCH; ++m)
      qv[m] = gq < G ? __ldg(reinterpret_cast<const uint4*>(qsrc) + tq + 4 * m) : make_uint4(0u, 0u, 0u, 0u);
    int nref = 0;
    if (ctx < 0 || ctx > max_ctx) {
      if (lane == 0) record_error(DKV_DEVERR_BOUNDS);
    } else {
      nref = ceil_div_d(ctx, R);
    }
    if (j0 >= nref) continue;  // warp-uniform: the task lies past the context
    float* dst = sref + static_cast<int64_t>(u) * max_ref * G;

    // K rows of tile i (rows gq, gq + 8), zero past the context
    auto issue = [&](int i, uint4 (&k)[2][NCH]) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int j = j0 + 16 * i + gq + 8 * hr;
        if (j < nref) {
          int pb = raw[i][hr];
          if (pb < 0 || pb >= num_blocks) {
            record_error(DKV_DEVERR_BLOCK_ID);
            pb = 0;  // read a valid block instead; the error word reports the bad table
          }
          const uint4* row = reinterpret_cast<const uint4*>(refs + (static_cast<int64_t>(pb) * H + h) * 2 * D);
#pragma unroll
          for (int m = 0; m < NCH; ++m) k[hr][m] = __ldg(row + tq + 4 * m);
        } else {
#pragma unroll
          for (int m = 0; m < NCH; ++m) k[hr][m] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    };
    auto word = [](const uint4& v, int w) { return w == 0 ? v.x : w == 1 ? v.y : w == 2 ? v.z : v.w; };
    auto multiply = [&](int i, const uint4 (&k)[2][NCH]) {
      const int ja = j0 + 16 * i + gq, jb = ja + 8;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < NKS; ++ks) {
        const int m = ks >> 1, e = ks & 1;
        mma_bf16_16816_a4(acc, word(k[0][m], 2 * e), word(k[1][m], 2 * e), word(k[0][m], 2 * e + 1),
                          word(k[1][m], 2 * e + 1), word(qv[m], 2 * e), word(qv[m], 2 * e + 1));
      }
      // C rows gq, gq + 8 are references ja, jb; columns 2tq, 2tq + 1 are query heads
      if (2 * tq < G) {
        if constexpr (G == 1) {
          if (ja < nref) dst[ja] = acc[0] * scale2;
          if (jb < nref) dst[jb] = acc[2] * scale2;
        } else {
          if (ja < nref)
            *reinterpret_cast<float2*>(dst + static_cast<int64_t>(ja) * G + 2 * tq) =
                make_float2(acc[0] * scale2, acc[1] * scale2);
          if (jb < nref)
            *reinterpret_cast<float2*>(dst + static_cast<int64_t>(jb) * G + 2 * tq) =
                make_float2(acc[2] * scale2, acc[3] * scale2);
        }
      }
    };
    static_assert(kProTaskTiles % 2 == 0, "tiles are taken in pairs of buffers");
    uint4 ka[2][NCH], kb[2][NCH];
    issue(0, ka);
    issue(1, kb);
#pragma unroll
    for (int i = 0; i < kProTaskTiles; i += 2) {
      if (j0 + 16 * i >= nref) break;  // warp-uniform
      multiply(i, ka);
      if (i + 2 < kProTaskTiles && j0 + 16 * (i + 2) < nref) issue(i + 2, ka);
      if (j0 + 16 * (i + 1) >= nref) break;
      multiply(i + 1, kb);
      if (i + 3 < kProTaskTiles && j0 + 16 * (i + 3) < nref) issue(i + 3, kb);
    }
  }
}

// ------------------------------------------------------------------------------------------------
// Split-K main kernel.
//   warps 0..7  consumers: 4 lanes per token, r/4 code dimensions per lane
//   warp 8      producer: whole paged blocks (codes + indices) by bulk copy into a 4-stage ring
//   warp 9      gatherer: for each landed stage, reads the reference indices and gathers q.r~K_idx (one
//               16-byte row per token from L2) into the stage, so consumers never wait on a dependent
//               global load
// ------------------------------------------------------------------------------------------------
constexpr int kDecNCW = 8;                // consumer warps
constexpr int kDecThreads = (kDecNCW + 2) * 32;
constexpr int kDecStages = 4;
// The running max is raised only when a stage exceeds it by more than 2^kRescaleLog2, so every softmax
// weight p = 2^(s - m) stays <= 16.  On the bf16 path the per-reference mass is accumulated with native
// 32-bit integer shared-memory atomics in fixed point (p * 2^14; float atomics on shared memory are
// compare-and-swap loops, several times slower): a split holds at most 8192 tokens, so a bin never
// exceeds 8192 * 16 * 2^14 = 2^31.  The fp32 path keeps exact float atomics.
constexpr float kRescaleLog2 = 4.0f;
constexpr float kMassScale = 16384.0f;        // 2^14
constexpr float kMassScaleInv = 1.0f / 16384.0f;

template <typename T>
struct MassBin {
  using type = float;
  static __device__ __forceinline__ void add(float* b, float p) { atomicAdd(b, p); }
  static __device__ __forceinline__ float value(float b) { return b; }
  static __device__ __forceinline__ void scale(float* b, float a) { *b *= a; }
};
template <>
struct MassBin<__nv_bfloat16> {
  using type = uint32_t;
  static __device__ __forceinline__ void add(uint32_t* b, float p) { atomicAdd(b, __float2uint_rn(p * kMassScale)); }
  static __device__ __forceinline__ float value(uint32_t b) { return static_cast<float>(b) * kMassScaleInv; }
  static __device__ __forceinline__ void scale(uint32_t* b, float a) { *b = __float2uint_rn(static_cast<float>(*b) * a); }
};

template <typename T, int RK, int G>
struct SplitCfg {
  static constexpr int ES = sizeof(T);
  static constexpr int STG = decode_stage_tokens(RK, ES);  // tokens per stage (the split plan uses the same)
  static constexpr int NGRP = STG / (kDecNCW * 8);  // 8-token groups per warp per stage
  static constexpr int DPL = RK / 4;                 // code dims per lane
  static constexpr int CODE_BYTES = STG * 2 * RK * ES;
  static constexpr int IDX_BYTES = STG * 4;
  static constexpr int SREF_BYTES = STG * G * 4;
  static constexpr int STAGE_BYTES = CODE_BYTES + IDX_BYTES + SREF_BYTES;
  static constexpr int HDR_BYTES = 128;  // barriers + abort flag
};

template <typename T, int RK, int G>
size_t split_smem_bytes(int jcap_max) {
  using C = SplitCfg<T, RK, G>;
  return C::HDR_BYTES + static_cast<size_t>(kDecStages) * C::STAGE_BYTES +
         static_cast<size_t>(jcap_max) * G * 4 + 2 * kDecNCW * G * 4 + kDecNCW * G * RK * 4 + kDecNCW * G * 4;
}

template <typename T, int RK, int G, bool SPARSE>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(
    const T* __restrict__ codes, const int* __restrict__ ref_idx, const int* __restrict__ context_lens,
    const int* __restrict__ block_tables, int max_blocks, int num_blocks, int Hq, int H, int R, int max_ctx,
    int max_ref, int tps, int nsplit, const float* __restrict__ qp, const float* __restrict__ qmu,
    const float* __restrict__ sref, float* __restrict__ part_ml, float* __restrict__ part_acc,
    float* __restrict__ part_bins, const int* __restrict__ sel, const int* __restrict__ cu_sel, int max_sel) {
  using C = SplitCfg<T, RK, G>;
  constexpr int STG = C::STG, NGRP = C::NGRP, DPL = C::DPL;
  extern __shared__ __align__(128) uint8_t sm_split[];
  uint64_t* full = reinterpret_cast<uint64_t*>(sm_split);
  uint64_t* gath = full + kDecStages;
  uint64_t* empty = gath + kDecStages;
  volatile int* sAbort = reinterpret_cast<volatile int*>(empty + kDecStages);
  uint8_t* stages = sm_split + C::HDR_BYTES;
  using Bin = MassBin<T>;
  using BinT = typename Bin::type;
  BinT* bins = reinterpret_cast<BinT*>(stages + kDecStages * C::STAGE_BYTES);

  const int split = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const SeqExtent ext = seq_extent<SPARSE>(context_lens, cu_sel, s, max_ctx, max_sel);
  const int t_begin = split * tps;
  const int t_end = min(ext.n, t_begin + tps);
  const int hq0 = h * G;
  const int64_t ml_base = (static_cast<int64_t>(s) * Hq + hq0) * nsplit + split;  // + g * nsplit

  if (t_begin >= t_end) {  // empty split: neutral partials
    if (tid < G) {
      part_ml[(ml_base + tid * nsplit) * 2] = -INFINITY;
      part_ml[(ml_base + tid * nsplit) * 2 + 1] = 0.f;
    }
    for (int e = tid; e < G * RK; e += blockDim.x) part_acc[(ml_base + (e / RK) * nsplit) * RK + e % RK] = 0.f;
    return;
  }
  const int jcap = split_jcap<SPARSE>(ext, t_end, R);
  float* wmax = reinterpret_cast<float*>(bins + static_cast<size_t>(jcap) * G);  // [2][NCW][G]
  float* red = wmax + 2 * kDecNCW * G;                 // [NCW][G][RK]
  float* lred = red + kDecNCW * G * RK;                // [NCW][G]

  if (tid == 0) {
    for (int i = 0; i < kDecStages; ++i) {
      mbar_init(smem_u32(full + i), SPARSE ? 32 : 1);  // sparse: one cp.async arrival per producer lane
      mbar_init(smem_u32(gath + i), 1);
      mbar_init(smem_u32(empty + i), kDecNCW);
    }
    *sAbort = 0;
    fence_barrier_init();
  }
  for (int e = tid; e < jcap * G; e += blockDim.x) bins[e] = BinT(0);
  __syncthreads();

  const int nst = ceil_div_d(t_end - t_begin, STG);
  const int blk0 = t_begin / R;
  const int nblk = ceil_div_d(t_end, R);
  const int BPS = STG / R;
  const uint32_t blk_code_bytes = static_cast<uint32_t>(R) * 2 * RK * sizeof(T);
  const uint32_t blk_idx_bytes = static_cast<uint32_t>(R) * 4;

  if (warp == kDecNCW && SPARSE) {
    // ---------------- producer, sparse: each listed token's code row and index by cp.async ----------------
    constexpr int ROWB = 2 * RK * static_cast<int>(sizeof(T));  // bytes of one token's codes
    const int* list = sel + ext.sel0;
    const int* btrow = block_tables + static_cast<int64_t>(s) * max_blocks;
    for (int st = 0; st < nst; ++st) {
      const int slot = st % kDecStages;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(smem_u32(empty + slot), ((st / kDecStages) & 1) ^ 1, sAbort);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      uint8_t* sc = stages + slot * C::STAGE_BYTES;
      for (int n = lane; n < STG; n += 32) {
        const int e = t_begin + st * STG + n;
        if (e >= t_end) break;
        const int p = checked_pos(list, e, ext.ctx);
        int pb = __ldg(btrow + p / R);
        if (pb < 0 || pb >= num_blocks) {
          record_error(DKV_DEVERR_BLOCK_ID);
          pb = 0;  // read a valid block instead; the error word reports the bad table
        }
        const int64_t row = (static_cast<int64_t>(pb) * H + h) * R + p % R;
        const uint8_t* src = reinterpret_cast<const uint8_t*>(codes + row * 2 * RK);
#pragma unroll
        for (int c = 0; c < ROWB / 16; ++c) cp_async_cg16(smem_u32(sc + n * ROWB + c * 16), src + c * 16);
        cp_async_n<4>(smem_u32(sc + C::CODE_BYTES + n * 4), ref_idx + row);
      }
      cp_async_mbar_arrive(smem_u32(full + slot));
    }
    cp_async_wait_all();  // no copy into this CTA's shared memory is left in flight when the warp returns
    return;
  }
  if (warp == kDecNCW) {
    // ---------------- producer: whole paged blocks by bulk copy ----------------
    for (int st = 0; st < nst; ++st) {
      const int slot = st % kDecStages;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(smem_u32(empty + slot), ((st / kDecStages) & 1) ^ 1, sAbort);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        // aborted: wait (bounded) for the copies of the last stages armed before the warp returns
        if (lane == 0)
          for (int i = st > kDecStages ? st - kDecStages : 0; i < st; ++i)
            mbar_drain(smem_u32(full + i % kDecStages), (i / kDecStages) & 1);
        break;
      }
      const int lb = blk0 + st * BPS + lane;
      const bool valid = lane < BPS && lb < nblk;
      const int pb = valid ? checked_block(block_tables, max_blocks, num_blocks, s, lb) : 0;
      const int nvalid = __popc(__ballot_sync(0xffffffffu, valid));
      if (lane == 0) mbar_arrive_expect_tx(smem_u32(full + slot), nvalid * (blk_code_bytes + blk_idx_bytes));
      __syncwarp();
      if (valid) {
        uint8_t* sc = stages + slot * C::STAGE_BYTES;
        const int64_t cell = static_cast<int64_t>(pb) * H + h;
        bulk_g2s(smem_u32(sc + lane * blk_code_bytes), codes + cell * R * 2 * RK, blk_code_bytes,
                 smem_u32(full + slot));
        bulk_g2s(smem_u32(sc + C::CODE_BYTES + lane * blk_idx_bytes), ref_idx + cell * R, blk_idx_bytes,
                 smem_u32(full + slot));
      }
    }
    return;
  }
  const float* sref_sh = sref + (static_cast<int64_t>(s) * H + h) * max_ref * G;
  if (warp == kDecNCW + 1) {
    // ---------------- gatherer: q.r~K_idx rows into the stage ----------------
    for (int st = 0; st < nst; ++st) {
      const int slot = st % kDecStages;
      if (!mbar_wait(smem_u32(full + slot), (st / kDecStages) & 1, sAbort)) break;
      uint8_t* sc = stages + slot * C::STAGE_BYTES;
      const int* si = reinterpret_cast<const int*>(sc + C::CODE_BYTES);
      float* sg = reinterpret_cast<float*>(sc + C::CODE_BYTES + C::IDX_BYTES);
      const int tok_base = t_begin + st * STG;
      float v[STG / 32][G];
#pragma unroll
      for (int k = 0; k < STG / 32; ++k) {
        const int tok = k * 32 + lane;
        const int t = tok_base + tok;
        int idx = t < t_end ? si[tok] : 0;
        if (t < t_end && (idx < 0 || idx >= jcap)) {
          record_error(DKV_DEVERR_REF_IDX);
          idx = 0;
        }
        const float* row = sref_sh + static_cast<int64_t>(idx) * G;
        if constexpr (G % 4 == 0) {
#pragma unroll
          for (int g4 = 0; g4 < G / 4; ++g4) {
            const float4 q = __ldg(reinterpret_cast<const float4*>(row) + g4);
            v[k][4 * g4] = q.x, v[k][4 * g4 + 1] = q.y, v[k][4 * g4 + 2] = q.z, v[k][4 * g4 + 3] = q.w;
          }
        } else {
#pragma unroll
          for (int g = 0; g < G; ++g) v[k][g] = __ldg(row + g);
        }
      }
#pragma unroll
      for (int k = 0; k < STG / 32; ++k)
#pragma unroll
        for (int g = 0; g < G; ++g) sg[(k * 32 + lane) * G + g] = v[k][g];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(gath + slot));  // release: the gathered rows are visible
    }
    return;
  }

  // ---------------- consumers ----------------
  const int cw = warp, tig = lane >> 2, sub = lane & 3;
  float qv[G][DPL], qm[G], m[G], l[G], acc[G][DPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float* qrow = qp + (static_cast<int64_t>(s) * Hq + hq0 + g) * RK + sub * DPL;
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      qv[g][i] = qrow[i];
      acc[g][i] = 0.f;
    }
    qm[g] = qmu[static_cast<int64_t>(s) * Hq + hq0 + g];
    m[g] = -INFINITY;
    l[g] = 0.f;
  }
  bool aborted = false;

  for (int st = 0; st < nst; ++st) {
    const int slot = st % kDecStages;
    // On a timeout the wait raises the shared abort flag; the stage is then processed from stale shared
    // memory (indices were range-checked by the gatherer or are stale in-range values) and every consumer
    // leaves together after the next CTA barrier.
    mbar_wait(smem_u32(gath + slot), (st / kDecStages) & 1, sAbort);
    const uint8_t* sc8 = stages + slot * C::STAGE_BYTES;
    const T* sc = reinterpret_cast<const T*>(sc8);
    const int* si = reinterpret_cast<const int*>(sc8 + C::CODE_BYTES);
    const float* sg = reinterpret_cast<const float*>(sc8 + C::CODE_BYTES + C::IDX_BYTES);
    const int tok_base = t_begin + st * STG;
    float s2[NGRP][G];
    int ix[NGRP];
    bool vl[NGRP];
#pragma unroll
    for (int grp = 0; grp < NGRP; ++grp) {
      const int tok = cw * (STG / kDecNCW) + grp * 8 + tig;
      const int t = tok_base + tok;
      vl[grp] = t < t_end;
      int idx = vl[grp] ? si[tok] : 0;
      if (idx < 0 || idx >= jcap) idx = 0;  // recorded by the gatherer
      ix[grp] = idx;
      float kk[DPL];
      load_elems<T, DPL>(sc + tok * 2 * RK + sub * DPL, kk);
      float gref[G];
      if constexpr (G % 4 == 0) {
#pragma unroll
        for (int g4 = 0; g4 < G / 4; ++g4) {
          const float4 q = reinterpret_cast<const float4*>(sg + tok * G)[g4];
          gref[4 * g4] = q.x, gref[4 * g4 + 1] = q.y, gref[4 * g4 + 2] = q.z, gref[4 * g4 + 3] = q.w;
        }
      } else {
#pragma unroll
        for (int g = 0; g < G; ++g) gref[g] = sg[tok * G + g];
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) a = fmaf(qv[g][i], kk[i], a);
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        s2[grp][g] = vl[grp] ? qm[g] + gref[g] + a : -INFINITY;
      }
    }
    // stage maximum per query head, CTA-wide
    float* wm = wmax + (st & 1) * kDecNCW * G;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mx = s2[0][g];
#pragma unroll
      for (int grp = 1; grp < NGRP; ++grp) mx = fmaxf(mx, s2[grp][g]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      if (lane == 0) wm[cw * G + g] = mx;
    }
    if (named_bar_or(1, kDecNCW * 32, *sAbort != 0)) {
      aborted = true;
      break;
    }
    bool need = false;
    float alpha[G];
    bool rescale_bins = false;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float M = wm[g];
#pragma unroll
      for (int w = 1; w < kDecNCW; ++w) M = fmaxf(M, wm[w * G + g]);
      alpha[g] = 1.f;
      if (M > m[g] + kRescaleLog2) {
        need = true;
        if (m[g] != -INFINITY) {
          alpha[g] = exp2f(m[g] - M);
          rescale_bins = true;
        } else {
          alpha[g] = 0.f;
        }
        m[g] = M;
      }
    }
    if (need) {  // uniform across the consumer threads (same shared data)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        l[g] *= alpha[g];
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[g][i] *= alpha[g];
      }
      if (rescale_bins) {
        for (int e = tid; e < jcap * G; e += kDecNCW * 32) {
          float a = 1.f;
#pragma unroll
          for (int g = 0; g < G; ++g)
            if (e % G == g) a = alpha[g];
          Bin::scale(bins + e, a);
        }
        named_bar_sync(1, kDecNCW * 32);
      }
    }
#pragma unroll
    for (int grp = 0; grp < NGRP; ++grp) {
      const int tok = cw * (STG / kDecNCW) + grp * 8 + tig;
      float vv[DPL];
      load_elems<T, DPL>(sc + tok * 2 * RK + RK + sub * DPL, vv);
      // a token past the end has p = 0, but its stage row may hold stale bits (0 * NaN = NaN)
#pragma unroll
      for (int i = 0; i < DPL; ++i) vv[i] = vl[grp] ? vv[i] : 0.f;
      float p[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        p[g] = vl[grp] ? exp2f(s2[grp][g] - m[g]) : 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[g][i] = fmaf(p[g], vv[i], acc[g][i]);
      }
#pragma unroll
      for (int g = 0; g < G; ++g)
        if ((g & 3) == sub) {
          l[g] += p[g];
          if (vl[grp]) Bin::add(bins + ix[grp] * G + g, p[g]);
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(empty + slot));
  }
  named_bar_sync(1, kDecNCW * 32);  // all mass adds done (every consumer reaches this once)
  if (aborted) return;

  float* gb = part_bins + ((static_cast<int64_t>(s) * H + h) * nsplit + split) * static_cast<int64_t>(max_ref) * G;
  for (int e = tid; e < jcap * G; e += kDecNCW * 32) gb[e] = Bin::value(bins[e]);
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      float a = acc[g][i];
      a += __shfl_xor_sync(0xffffffffu, a, 4);
      a += __shfl_xor_sync(0xffffffffu, a, 8);
      a += __shfl_xor_sync(0xffffffffu, a, 16);
      if (tig == 0) red[(cw * G + g) * RK + sub * DPL + i] = a;
    }
    float lv = (g & 3) == sub ? l[g] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lv += __shfl_xor_sync(0xffffffffu, lv, o);
    if (lane == 0) lred[cw * G + g] = lv;
  }
  named_bar_sync(1, kDecNCW * 32);
  for (int e = tid; e < G * RK; e += kDecNCW * 32) {
    const int g = e / RK, o = e % RK;
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kDecNCW; ++w) a += red[(w * G + g) * RK + o];
    part_acc[(ml_base + g * nsplit) * RK + o] = a;
  }
  if (tid < G) {
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kDecNCW; ++w) L += lred[w * G + tid];
    part_ml[(ml_base + tid * nsplit) * 2] = m[tid];
    part_ml[(ml_base + tid * nsplit) * 2 + 1] = L;
  }
}

// ------------------------------------------------------------------------------------------------
// Split-K main kernel, bf16 with r in {32, 64}: the two per-token contractions on the tensor cores.
//
// For a split of cached tokens t of one (sequence, kv head), in the log2 domain:
//   S[t][g]   = q'[g] . cK[t]                    score of query head g against the K code
//   s2        = q.mu_K + q.r~K_idx(t) + S         p = 2^(s2 - m) with a CTA-wide lazy running max m
//   acc[g][:] += sum_t p[t][g] cV[t][:]          latent V accumulator
//   bins[idx(t)][g] += p[t][g]                   per-reference mass (32-bit fixed-point shared atomics)
// Both products run as mma.sync m16n8k16 on 16-token groups.  G >= 4: the tokens are the MMA rows and the
// heads its 8 columns ([q'_hi | q'_lo] for G = 4), and the V product is transposed with movmatrix building
// its B operand from the p fragment.  G < 4: the heads are the A rows, the hi halves in rows 0..7 and the lo
// halves in rows 8..15.  q' and p are split into bf16 hi + lo parts, so both products carry about 16 mantissa
// bits.  Codes arrive by tensor-map loads with
// the 128-byte swizzle (one box of R rows x 64 columns per paged block), so the ldmatrix reads are
// bank-conflict free.
//
// The kernel is persistent: one CTA per SM takes work items (sequence, kv head, split) round-robin, and the
// stage ring runs on across items.
//   warps 0..7  consumers (32 tokens of each stage per warp, two 16-token groups)
//   warp 8      producer (tensor-map loads of codes + bulk copies of indices)
//   warps 9, 10 gatherers (q.r~K_idx rows into the stage, half of its tokens each)
// Neither the producer nor the gatherers wait on a global load inside the stage loop.  An item's block ids
// and context length are read one item ahead, and the gathered q.r~K_idx rows are asynchronous copies
// (cp.async) whose completion the stage's barrier counts.  Either wait would otherwise cost one memory
// latency per stage and cap the ring at about one stage in flight.
// ------------------------------------------------------------------------------------------------
constexpr int kMaxSplitBlocks = kMaxSplitTokens / 16;  // paged blocks of one split (R >= 16)
constexpr int kBtRegs = kMaxSplitBlocks / 32;          // block ids per producer lane
constexpr int kMmaNCW = 8;     // consumer warps of the tensor-core split kernel (STG / 128 16-token groups each per stage)
constexpr int kMmaGW = 2;      // gatherer warps (each takes half of a stage's tokens)
constexpr int kMmaThreads = (kMmaNCW + 1 + kMmaGW) * 32;  // + producer + gatherers

// STG = tokens per stage: 256 with one CTA per SM, 128 with two CTAs per SM (a smaller ring per CTA, twice the
// consumer warps per SM), chosen at launch by what the shared memory holds.
// Q4 (4-bit codes): the producer's bulk copies land in a staging area of packed rows (r bytes a token) and
// bf16 scale pairs; each consumer warp expands the nibbles of the rows it reads into its bf16 tiles, and
// reads the scale pairs where they landed.
// KT: reference slots per token (1; 2 or 4 with the k-nearest retrieval, whose token mixes the mean of its
// slots' references): KT indices and KT gathered q.r~K rows per token.
template <int RK, int G, int STG, bool Q4 = false, int KT = 1>
struct MmaSplitCfg {
  static constexpr int TILES = RK / 32;                         // swizzled 64-column tiles per token row
  static constexpr int TILE_BYTES = STG * 128;
  static constexpr int CODE_BYTES = TILES * TILE_BYTES;
  static constexpr int IDX_BYTES = STG * 4 * KT;
  static constexpr int SREF_BYTES = STG * G * 4 * KT;
  static constexpr int Q4ROW_OFF = CODE_BYTES + IDX_BYTES + SREF_BYTES;
  static constexpr int Q4ROW_BYTES = Q4 ? STG * RK : 0;         // packed nibble rows
  static constexpr int Q4SC_OFF = Q4ROW_OFF + Q4ROW_BYTES;
  static constexpr int Q4SC_BYTES = Q4 ? STG * 4 : 0;           // bf16 (K, V) scale pairs
  static constexpr int STAGE_BYTES = (Q4SC_OFF + Q4SC_BYTES + 1023) / 1024 * 1024;
  static constexpr int HDR_BYTES = 1024;                        // barriers; keeps the stages 1024-aligned
  static constexpr int MAX_STAGES = 4;
};

// Shared memory of the split kernel beside the stage ring: mass bins, stage maxima, reductions, block ids.
template <int RK, int G>
size_t split_mma_tail_bytes(int jcap_max) {
  return (static_cast<size_t>(jcap_max) * G * 4 + 15) / 16 * 16 + kMmaNCW * G * 4 + kMmaNCW * G * RK * 4 +
         kMmaNCW * G * 4 + kMaxSplitBlocks * 4;
}
// Stages of STG tokens that fit in `limit` bytes (min_stages..4), or 0 if not even min_stages do.
template <int RK, int G, int STG, bool Q4 = false, int KT = 1>
int split_mma_stages(int jcap_max, size_t limit, int min_stages) {
  using C = MmaSplitCfg<RK, G, STG, Q4, KT>;
  const size_t fixed = 1024 /* alignment slack */ + C::HDR_BYTES + split_mma_tail_bytes<RK, G>(jcap_max);
  if (fixed + static_cast<size_t>(min_stages) * C::STAGE_BYTES > limit) return 0;
  const int ns = static_cast<int>((limit - fixed) / C::STAGE_BYTES);
  return ns > C::MAX_STAGES ? C::MAX_STAGES : ns;
}
template <int RK, int G, int STG, bool Q4 = false, int KT = 1>
size_t split_mma_smem_bytes(int jcap_max, int stages) {
  using C = MmaSplitCfg<RK, G, STG, Q4, KT>;
  return 1024 + C::HDR_BYTES + static_cast<size_t>(stages) * C::STAGE_BYTES + split_mma_tail_bytes<RK, G>(jcap_max);
}
// Shared memory per CTA when two CTAs share an SM (228 KB per SM, 1 KB of it reserved per CTA).
constexpr size_t kHalfSmLimit = 112 * 1024;
// Launch shape of the tensor-core split kernel for a context bound: two CTAs per SM with 128-token stages when
// the per-reference mass and three stages fit in half an SM's shared memory, else one CTA per SM with
// 256-token stages (at least two of them), else none (stages == 0).
struct MmaSplitShape {
  int stg = 256, stages = 0, ctas_per_sm = 1;
  size_t smem = 0;
  bool gbins = false;  // per-reference masses in global memory (the GB kernel)
};
// Two CTAs per SM are built for r = 32 with G <= 4 only: those consumers fit in 88 registers (two 11-warp CTAs
// in the 64K-register file, checked by the launch bounds); the other shapes need more.
template <int RK, int G>
constexpr bool kTwoCtaSplit = RK == 32 && G <= 4;

template <int RK, int G, bool Q4 = false, int KT = 1>
MmaSplitShape split_mma_shape(int jcap_max) {
  MmaSplitShape m;
  if constexpr (kTwoCtaSplit<RK, G> && KT == 1) {
    const int s128 = split_mma_stages<RK, G, 128, Q4, KT>(jcap_max, kHalfSmLimit, 3);
    if (s128 > 0) {
      m.stg = 128;
      m.stages = s128;
      m.ctas_per_sm = 2;
      m.smem = split_mma_smem_bytes<RK, G, 128, Q4, KT>(jcap_max, s128);
      return m;
    }
  }
  m.stages = split_mma_stages<RK, G, 256, Q4, KT>(jcap_max, 226 * 1024, 2);
  if (m.stages > 0) m.smem = split_mma_smem_bytes<RK, G, 256, Q4, KT>(jcap_max, m.stages);
  return m;
}

// Launch shape of the global-mass (GB) split kernel: one CTA per SM, 256-token stages, no masses in shared
// memory.  It replaces the shared-memory masses when those leave fewer than kGbinsBelowStages stages.
constexpr int kGbinsBelowStages = 3;
template <int RK, int G>
MmaSplitShape split_mma_shape_gb() {
  MmaSplitShape m;
  m.stages = split_mma_stages<RK, G, 256>(0, 226 * 1024, 2);
  if (m.stages > 0) m.smem = split_mma_smem_bytes<RK, G, 256>(0, m.stages);
  m.gbins = true;
  return m;
}

// Eight 4-bit codes (one nibble word: nibble k holds code 2k, nibble k + 4 code 2k + 1, two's complement) as
// eight bf16 values in order.  Offset binary (x ^ 8) in a bf16 mantissa gives 128 + (code + 8) exactly;
// subtracting 136 leaves the code, also exactly.
__device__ __forceinline__ uint4 q4_word_to_bf16x8(uint32_t w) {
  const uint32_t x = w ^ 0x88888888u;
  const __nv_bfloat162 off = __floats2bfloat162_rn(136.f, 136.f);
  uint32_t o[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t b = ((x >> (4 * k)) & 0x000F000Fu) | 0x43004300u;
    const __nv_bfloat162 v = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&b), off);
    o[k] = *reinterpret_cast<const uint32_t*>(&v);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Two floats to a bf16x2 word (x0 in the low half), round to nearest even.
__device__ __forceinline__ uint32_t cvt_bf16x2(float x0, float x1) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(x1), "f"(x0));
  return d;
}
// bf16 hi/lo split of a pair: x = hi + lo with hi = RNE_bf16(x), lo = RNE_bf16(x - hi).
__device__ __forceinline__ void split_pack(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = cvt_bf16x2(x0, x1);
  lo = cvt_bf16x2(x0 - __uint_as_float(hi << 16), x1 - __uint_as_float(hi & 0xffff0000u));
}
// 2^x with the hardware approximation (ex2.approx: relative error about 2^-22; 2^-inf = 0).
// round(p * kMassScale) as an unsigned integer, for 0 <= p * kMassScale < 2^22: adding 2^23 in one fused
// multiply-add leaves the round-to-nearest-even integer in the low mantissa bits (same value as
// __float2uint_rn(p * kMassScale), without the conversion unit).
__device__ __forceinline__ uint32_t mass_fixed(float p) {
  return __float_as_uint(fmaf(p, kMassScale, 8388608.0f)) - 0x4B000000u;
}
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Shared-memory address of 16-byte chunk c of row n in a swizzled [rows][128 B] tile (128-byte swizzle).
__device__ __forceinline__ uint32_t swz(uint32_t tile, int n, int c) {
  return tile + static_cast<uint32_t>(n) * 128u + (static_cast<uint32_t>(c ^ (n & 7)) << 4);
}

// Maximum of one head's per-warp stage maxima ([kMmaNCW] floats, 16-byte aligned).
__device__ __forceinline__ float stage_max_row(const float* row) {
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMmaNCW / 4; ++i) {
    const float4 w = reinterpret_cast<const float4*>(row)[i];
    m = fmaxf(m, fmaxf(fmaxf(w.x, w.y), fmaxf(w.z, w.w)));
  }
  return m;
}

// GB (global bins): the per-reference masses live in the item's slice of the workspace's per-split masses,
// accumulated with global atomics in the same fixed point, and are converted to fp32 in place when the item
// ends.  It serves contexts whose masses do not fit in shared memory beside two stages.
template <int RK, int G, bool SPARSE, int STG, bool Q4, int KT, bool GB = false>
__global__ void __launch_bounds__(kMmaThreads, STG == 128 ? 2 : 1) decode_split_mma_kernel(
    const __grid_constant__ CUtensorMap codes_map, const int* __restrict__ ref_idx,
    const int* __restrict__ context_lens, const int* __restrict__ block_tables, int max_blocks, int num_blocks,
    int num_seqs, int Hq, int H, int R, int max_ctx, int max_ref, int tps, int nsplit, int nstages,
    const float* __restrict__ qp,
    const float* __restrict__ qmu, const float* __restrict__ sref, float* __restrict__ part_ml,
    float* __restrict__ part_acc, float* __restrict__ part_bins, const __nv_bfloat16* __restrict__ codes,
    const int* __restrict__ sel, const int* __restrict__ cu_sel, int max_sel) {
  using C = MmaSplitCfg<RK, G, STG, Q4, KT>;
  static_assert(KT == 1 || (!SPARSE && !Q4 && G >= 4), "k-nearest slots: dense bf16 decode, tokens as MMA rows");
  static_assert(!GB || (!SPARSE && !Q4 && KT == 1 && STG == 256), "global masses: dense bf16, one CTA per SM");
  static_assert(!(Q4 && SPARSE), "4-bit codes are decoded densely");
  static_assert(!Q4 || G >= 4, "4-bit codes: tokens are the MMA rows");
  static_assert(G <= 8, "heads of a group are padded to 8 rows of the 16-row fragment");
  constexpr int NDT = RK / 8;  // 8-wide dimension tiles of the V accumulator
  constexpr int NGRP = STG / (kMmaNCW * 16);  // 16-token groups per warp per stage
  extern __shared__ uint8_t sm_mma_raw[];
  uint8_t* smb = align_shared<1024>(sm_mma_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smb);
  uint64_t* gath = full + C::MAX_STAGES;
  uint64_t* empty = gath + C::MAX_STAGES;
  volatile int* sAbort = reinterpret_cast<volatile int*>(empty + C::MAX_STAGES);
  uint8_t* stages = smb + C::HDR_BYTES;
  // per-reference masses of the current item [jcap][G] (shared memory; GB: none here, see above)
  uint32_t* sbins = reinterpret_cast<uint32_t*>(stages + nstages * C::STAGE_BYTES);

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  // per-warp stage maxima [G][NCW] of an exchange, on a 16-byte boundary (they are read as float4)
  float* wmax = reinterpret_cast<float*>(
      sbins + (GB ? 0 : ((static_cast<size_t>(max_ref) * G + 3) & ~static_cast<size_t>(3))));
  float* red = wmax + kMmaNCW * G;                                                 // [NCW][G][RK]
  float* lred = red + kMmaNCW * G * RK;                                            // [NCW][G]
  int* sbt = reinterpret_cast<int*>(lred + kMmaNCW * G);                           // [kMaxSplitBlocks]

  if (tid == 0) {
    for (int i = 0; i < nstages; ++i) {
      // dense: one arrive with the transaction bytes of the tensor-map loads; sparse: one cp.async arrival per
      // producer lane (each lane gathers its own token rows)
      mbar_init(smem_u32(full + i), SPARSE ? 32 : 1);
      mbar_init(smem_u32(gath + i), kMmaGW * (1 + 32));  // per gatherer: lane 0 + one cp.async arrival per lane
      mbar_init(smem_u32(empty + i), kMmaNCW);
    }
    *sAbort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // Launched programmatically after the prologue: the producer streams codes, indices and block ids (written
  // before this decode call) at once; the gatherers and consumers wait for the prologue's q.r~K_j, q' and q.mu_K.
  // The combine may be scheduled as SMs free up; it waits for this grid before reading its partials.
  griddep_launch_dependents();

  // Work items (sequence, kv head, split), split fastest, taken round-robin by the persistent CTAs.  Every
  // role walks the same item sequence and counts stages globally (g), so the stage ring, its barriers and
  // their phases run on across items without draining.  Splits that start past the context are skipped:
  // the combine reads no partials of them.
  const int n_items = num_seqs * H * nsplit;
  const int BPS = STG / R;  // 4..16 blocks per stage
  const uint32_t blk_code_bytes = static_cast<uint32_t>(R) * 2 * RK * 2;
  const uint32_t blk_idx_bytes = static_cast<uint32_t>(R) * 4 * KT;

  if (warp == kMmaNCW && SPARSE) {
    // ---------------- producer, sparse ----------------
    // Each listed token's code row (TILES x 128 bytes) and reference index are gathered by cp.async into the
    // layout the tensor-map loads produce (chunk c of stage row n at swz(tile, n, c)); lane L takes the list
    // entries L, L + 32, ... of a stage, and its copies' completion is one arrival on the stage barrier.  The
    // positions of stage st + 1 are read while stage st is issued, and the block ids of stage st before the
    // wait for its slot, so both loads overlap that wait.
    constexpr int EPL = STG / 32;  // list entries per lane and stage
    int it = blockIdx.x;
    SeqExtent ext_n = it < n_items ? seq_extent<SPARSE>(context_lens, cu_sel, it / (H * nsplit), max_ctx, max_sel)
                                  : SeqExtent{0, 0, 0};
    int slot = 0;
    uint32_t ph = 0;  // ring slot and the parity of its current phase, carried across items
    bool ok = true;
    for (; it < n_items && ok; it += gridDim.x) {
      const SeqExtent ext = ext_n;
      if (it + static_cast<int>(gridDim.x) < n_items)
        ext_n = seq_extent<SPARSE>(context_lens, cu_sel, (it + gridDim.x) / (H * nsplit), max_ctx, max_sel);
      const int split = it % nsplit, h = (it / nsplit) % H, s = it / (H * nsplit);
      const int t_begin = split * tps, t_end = min(ext.n, t_begin + tps);
      if (t_begin >= t_end) continue;
      const int nst = ceil_div_d(t_end - t_begin, STG);
      const int* list = sel + ext.sel0;
      const int* btrow = block_tables + static_cast<int64_t>(s) * max_blocks;
      int pos[EPL];
      auto load_pos = [&](int st) {
#pragma unroll
        for (int k = 0; k < EPL; ++k) {
          const int e = t_begin + st * STG + k * 32 + lane;
          pos[k] = e < t_end ? checked_pos(list, e, ext.ctx) : -1;
        }
      };
      load_pos(0);
      for (int st = 0; st < nst; ++st) {
        int rowid[EPL];  // (physical block * H_kv + h) * R + row within the block (< 2^31); -1 past the list
#pragma unroll
        for (int k = 0; k < EPL; ++k) {
          rowid[k] = -1;
          if (pos[k] >= 0) {
            int pb = __ldg(btrow + pos[k] / R);
            if (pb < 0 || pb >= num_blocks) {
              record_error(DKV_DEVERR_BLOCK_ID);
              pb = 0;  // read a valid block instead; the error word reports the bad table
            }
            rowid[k] = (pb * H + h) * R + pos[k] % R;
          }
        }
        if (st + 1 < nst) load_pos(st + 1);
        int w = 1;
        if (lane == 0) w = mbar_wait(smem_u32(empty + slot), ph ^ 1, sAbort);
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) {
          ok = false;
          break;
        }
        uint8_t* sc = stages + slot * C::STAGE_BYTES;
        const uint32_t sc32 = smem_u32(sc);
#pragma unroll
        for (int k = 0; k < EPL; ++k) {
          if (rowid[k] < 0) continue;
          const int n = k * 32 + lane;
          const __nv_bfloat16* src = codes + static_cast<int64_t>(rowid[k]) * 2 * RK;
#pragma unroll
          for (int kt = 0; kt < C::TILES; ++kt)
#pragma unroll
            for (int c = 0; c < 8; ++c) cp_async_cg16(swz(sc32 + kt * C::TILE_BYTES, n, c), src + kt * 64 + c * 8);
          cp_async_n<4>(smem_u32(sc + C::CODE_BYTES + n * 4), ref_idx + rowid[k]);
        }
        cp_async_mbar_arrive(smem_u32(full + slot));
        if (++slot == nstages) {
          slot = 0;
          ph ^= 1u;
        }
      }
    }
    cp_async_wait_all();  // no copy into this CTA's shared memory is left in flight when the warp returns
    return;
  }
  if (warp == kMmaNCW) {
    // ---------------- producer ----------------
    if (!Q4 && lane == 0) prefetch_tensormap(&codes_map);
    // Raw block ids of an item are read one item ahead (while the previous item streams) and range-checked
    // into shared memory when the item starts, so the stage loop never waits on a global load.
    int bt_raw[kBtRegs];
    auto load_ids = [&](int it) {
      const int s = it / (H * nsplit), blk0 = (it % nsplit) * tps / R;
      const int nreq = min(tps / R, max_blocks - blk0);
      const int* row = block_tables + static_cast<int64_t>(s) * max_blocks + blk0;
#pragma unroll
      for (int k = 0; k < kBtRegs; ++k) bt_raw[k] = k * 32 + lane < nreq ? __ldg(row + k * 32 + lane) : 0;
    };
    int it = blockIdx.x;
    SeqExtent ext_n = it < n_items ? seq_extent<SPARSE>(context_lens, cu_sel, it / (H * nsplit), max_ctx, max_sel)
                                  : SeqExtent{0, 0, 0};
    if (it < n_items) load_ids(it);
    uint32_t g = 0;   // stages armed so far
    int slot = 0;
    uint32_t ph = 0;  // ring slot and the parity of its current phase
    bool ok = true;
    for (; it < n_items && ok; it += gridDim.x) {
      const SeqExtent ext = ext_n;
      const int split = it % nsplit, h = (it / nsplit) % H;
      const int t_begin = split * tps, t_end = min(ext.n, t_begin + tps);
      const int blk0 = t_begin / R, nblk = ceil_div_d(t_end, R);
#pragma unroll
      for (int k = 0; k < kBtRegs; ++k) {
        const int i = k * 32 + lane;
        if (blk0 + i < nblk) {
          int pb = bt_raw[k];
          if (pb < 0 || pb >= num_blocks) {
            record_error(DKV_DEVERR_BLOCK_ID);
            pb = 0;  // read a valid block instead; the error word reports the bad table
          }
          sbt[i] = pb;
        }
      }
      __syncwarp();
      if (it + static_cast<int>(gridDim.x) < n_items) {
        ext_n = seq_extent<SPARSE>(context_lens, cu_sel, (it + gridDim.x) / (H * nsplit), max_ctx, max_sel);
        load_ids(it + gridDim.x);
      }
      if (t_begin >= t_end) continue;
      const int nst = ceil_div_d(t_end - t_begin, STG);
      for (int st = 0; st < nst; ++st, ++g) {
        int w = 1;
        if (lane == 0) w = mbar_wait(smem_u32(empty + slot), ph ^ 1, sAbort);
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) {
          ok = false;
          break;
        }
        const int lbi = st * BPS + lane;
        const bool valid = lane < BPS && blk0 + lbi < nblk;
        const int pb = valid ? sbt[lbi] : 0;
        const int nvalid = __popc(__ballot_sync(0xffffffffu, valid));
        const uint32_t blk_bytes = Q4 ? static_cast<uint32_t>(R) * (RK + 4) : blk_code_bytes;
        if (lane == 0) mbar_arrive_expect_tx(smem_u32(full + slot), nvalid * (blk_bytes + blk_idx_bytes));
        __syncwarp();
        if (valid) {
          uint8_t* sc = stages + slot * C::STAGE_BYTES;
          const int64_t cell = static_cast<int64_t>(pb) * H + h;
          if constexpr (Q4) {  // packed rows, then the scale pairs, of this block (one cell is R*(r+4) bytes)
            const uint8_t* cp = reinterpret_cast<const uint8_t*>(codes) + cell * R * (RK + 4);
            bulk_g2s(smem_u32(sc + C::Q4ROW_OFF + lane * R * RK), cp, R * RK, smem_u32(full + slot));
            bulk_g2s(smem_u32(sc + C::Q4SC_OFF + lane * R * 4), cp + R * RK, R * 4, smem_u32(full + slot));
          } else {
#pragma unroll
            for (int kt = 0; kt < C::TILES; ++kt)
              tma_load_2d(smem_u32(sc + kt * C::TILE_BYTES + lane * R * 128), &codes_map, kt * 64,
                          static_cast<int>(cell * R), smem_u32(full + slot));
          }
          bulk_g2s(smem_u32(sc + C::CODE_BYTES + lane * blk_idx_bytes), ref_idx + cell * R * KT, blk_idx_bytes,
                   smem_u32(full + slot));
        }
        if (++slot == nstages) {
          slot = 0;
          ph ^= 1u;
        }
      }
      __syncwarp();  // the next item's block ids overwrite sbt
    }
    // Aborted: the loads of the last stages armed may still be landing in this CTA's shared memory; wait
    // (bounded) for the full barrier of each before the warp returns.  Stage i completes phase i / nstages.
    if (!ok && lane == 0)
      for (uint32_t i = g > static_cast<uint32_t>(nstages) ? g - nstages : 0; i < g; ++i)
        mbar_drain(smem_u32(full + i % nstages), (i / nstages) & 1);
    return;
  }
  if (warp > kMmaNCW) {
    // ---------------- gatherers ----------------
    griddep_wait();  // q.r~K_j rows come from the prologue
    constexpr int TPG = STG / kMmaGW;  // tokens of a stage per gatherer warp
    const int tg0 = (warp - kMmaNCW - 1) * TPG;
    int it = blockIdx.x;
    SeqExtent ext_n = it < n_items ? seq_extent<SPARSE>(context_lens, cu_sel, it / (H * nsplit), max_ctx, max_sel)
                                  : SeqExtent{0, 0, 0};
    int slot = 0;
    uint32_t ph = 0;  // ring slot and the parity of its current phase
    bool ok = true;
    for (; it < n_items && ok; it += gridDim.x) {
      const SeqExtent ext = ext_n;
      if (it + static_cast<int>(gridDim.x) < n_items)
        ext_n = seq_extent<SPARSE>(context_lens, cu_sel, (it + gridDim.x) / (H * nsplit), max_ctx, max_sel);
      const int split = it % nsplit, h = (it / nsplit) % H, s = it / (H * nsplit);
      const int t_begin = split * tps, t_end = min(ext.n, t_begin + tps);
      if (t_begin >= t_end) continue;
      const int nst = ceil_div_d(t_end - t_begin, STG);
      const int jcap = split_jcap<SPARSE>(ext, t_end, R);
      const float* sref_sh = sref + (static_cast<int64_t>(s) * H + h) * max_ref * G;
      for (int st = 0; st < nst; ++st) {
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(full + slot), ph, sAbort))) {
          ok = false;  // decided once per warp, so the lanes leave together
          break;
        }
        uint8_t* sc = stages + slot * C::STAGE_BYTES;
        int* si = reinterpret_cast<int*>(sc + C::CODE_BYTES);
        float* sg = reinterpret_cast<float*>(sc + C::CODE_BYTES + C::IDX_BYTES);
        const int tok_base = t_begin + st * STG;
        int vi[TPG / 32][KT];
#pragma unroll
        for (int k = 0; k < TPG / 32; ++k) {
          const int tok = tg0 + k * 32 + lane;
          const int t = tok_base + tok;
#pragma unroll
          for (int q = 0; q < KT; ++q) {
            int idx = t < t_end ? si[tok * KT + q] : 0;
            // -1 marks an unfilled slot of the k-nearest retrieval (fewer than k visible references)
            if (t < t_end && !(KT > 1 && idx == -1) && (idx < 0 || idx >= jcap)) {
              record_error(DKV_DEVERR_REF_IDX);
              idx = 0;
            }
            vi[k][q] = idx;
          }
        }
        // the consumers read the range-checked indices (tokens past the end read 0) and q.r~K_idx rows
#pragma unroll
        for (int k = 0; k < TPG / 32; ++k) {
          const int tok = tg0 + k * 32 + lane;
#pragma unroll
          for (int q = 0; q < KT; ++q) {
            si[tok * KT + q] = vi[k][q];
            const float* row = sref_sh + static_cast<int64_t>(vi[k][q] < 0 ? 0 : vi[k][q]) * G;
            const uint32_t dst = smem_u32(sg + (tok * KT + q) * G);
            if constexpr (G * 4 <= 16) {
              cp_async_n<G * 4>(dst, row);
            } else {
#pragma unroll
              for (int c = 0; c < G / 4; ++c) cp_async_n<16>(dst + 16 * c, row + 4 * c);
            }
          }
        }
        // Code rows of tokens past the end (last stage of a context only) hold stale shared memory or the
        // unused tail of a paged block.  Their softmax weight is 0, but 0 * (inf or NaN) would still reach
        // the V product, so they are zeroed (whole 128-byte rows: the swizzle only permutes within a row).
        // (4-bit codes: the consumer warps expand their rows and write zero rows past the end.)
        const int nval = Q4 ? tg0 + TPG : max(tg0, min(tg0 + TPG, t_end - tok_base));
        if (nval < tg0 + TPG) {
          const int nz = (tg0 + TPG - nval) * C::TILES * 8;  // 16-byte stores
          for (int e = lane; e < nz; e += 32) {
            const int row = nval + e / (C::TILES * 8), rem = e % (C::TILES * 8);
            *reinterpret_cast<uint4*>(sc + (rem / 8) * C::TILE_BYTES + row * 128 + (rem % 8) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_shared();  // these generic writes precede the slot's next tensor-map / bulk fill
        cp_async_mbar_arrive(smem_u32(gath + slot));  // counts once this lane's row copies have landed
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(gath + slot));  // release: indices and zeroed rows are visible
        if (++slot == nstages) {
          slot = 0;
          ph ^= 1u;
        }
      }
    }
    cp_async_wait_all();  // no gathered row is left in flight when the warp returns (an abort included)
    return;
  }

  // ---------------- consumers ----------------
  griddep_wait();  // q' and q.mu_K come from the prologue
  if constexpr (G >= 4) {
    // Tokens are the 16 rows of every MMA and the query heads sit in its 8 columns.  For G = 4 the columns
    // are [q'_hi of heads 0..3 | q'_lo of heads 0..3]: one MMA per 16-wide k-step, and the hi and lo halves
    // of a score meet across the lane pair (tq, tq ^ 2).  For G = 8 the columns are the 8 heads and hi / lo
    // are two MMAs into one accumulator.  The V product runs transposed,
    //   acc^T[dim][col] += sum_t cV[t][dim] p[t][col]     (A = cV^T by ldmatrix.trans, B = p),
    // with the p fragment of the score layout turned into the B operand by movmatrix.  Every lane carries
    // two heads (hb, hb + 1) of two token rows (gq, gq + 8) per 16-token group, so all 32 lanes do useful
    // softmax work.
    constexpr bool kDup = G == 4;
    constexpr int NKS = RK / 16;  // k-steps of the score product = 16-dim tiles of the V product
    constexpr int NGR = STG / (kMmaNCW * 16);  // 16-token groups per warp and stage
    const int gq = lane >> 2, tq = lane & 3;
    const int w32 = warp * (STG / kMmaNCW);  // this warp's first token in the stage
    const int hb = kDup ? 2 * (tq & 1) : 2 * tq;  // this lane's heads: hb, hb + 1
    const int rh = kDup ? (tq >> 1) : 0;          // G = 4: the token row (gq or gq + 8) whose mass this lane adds
    const int mat = lane >> 3;                    // ldmatrix: the 8x8 matrix this lane addresses
    // Byte offsets of this lane's ldmatrix rows in a stage, for the warp's first 16-token group (the next
    // group is 16 rows = 2048 bytes further on).  Rows sit at multiples of 8 plus lane & 7, so the 128-byte
    // swizzle term is fixed per lane and the stage loop only adds the slot's base address.
    uint32_t offK[NKS], offV[NKS];
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks) {
      const int krow = w32 + (mat & 1) * 8 + (lane & 7), kcol = 16 * ks + (mat >> 1) * 8;  // K codes
      const int vrow = w32 + (mat >> 1) * 8 + (lane & 7), vcol = RK + 16 * ks + (mat & 1) * 8;  // V codes
      offK[ks] = swz((kcol / 64) * C::TILE_BYTES, krow, (kcol % 64) / 8);
      offV[ks] = swz((vcol / 64) * C::TILE_BYTES, vrow, (vcol % 64) / 8);
    }
    // This lane's q' values and q.mu_K for an item, read one item ahead so that their latency hides under
    // the previous item's stages.
    float qn[NKS][2][2], qmn[2];
    int q_it = -1;
    auto fetch_q = [&](int itq) {
      const int sq = itq / (H * nsplit), hq = (itq / nsplit) % H;
      const float* qrow = qp + (static_cast<int64_t>(sq) * Hq + hq * G + (kDup ? (gq & 3) : gq)) * RK;
#pragma unroll
      for (int ks = 0; ks < NKS; ++ks)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int k0 = 16 * ks + 8 * half + 2 * tq;
          qn[ks][half][0] = qrow[k0];
          qn[ks][half][1] = qrow[k0 + 1];
        }
      qmn[0] = qmu[static_cast<int64_t>(sq) * Hq + hq * G + hb];
      qmn[1] = qmu[static_cast<int64_t>(sq) * Hq + hq * G + hb + 1];
      q_it = itq;
    };
    int it = blockIdx.x;
    SeqExtent ext_n = it < n_items ? seq_extent<SPARSE>(context_lens, cu_sel, it / (H * nsplit), max_ctx, max_sel)
                                  : SeqExtent{0, 0, 0};
    if (it < n_items) fetch_q(it);
    int slot = 0;
    uint32_t ph = 0;  // ring slot and the parity of its current phase, carried across items
    bool aborted = false;
    for (; it < n_items; it += gridDim.x) {
      const SeqExtent ext = ext_n;
      if (it + static_cast<int>(gridDim.x) < n_items)
        ext_n = seq_extent<SPARSE>(context_lens, cu_sel, (it + gridDim.x) / (H * nsplit), max_ctx, max_sel);
      const int split = it % nsplit, h = (it / nsplit) % H, s = it / (H * nsplit);
      const int t_begin = split * tps, t_end = min(ext.n, t_begin + tps);
      if (t_begin >= t_end) continue;
      const int nst = ceil_div_d(t_end - t_begin, STG);
      const int jcap = split_jcap<SPARSE>(ext, t_end, R);
      const int hq0 = h * G;
      const int64_t ml_base = (static_cast<int64_t>(s) * Hq + hq0) * nsplit + split;  // + g * nsplit
      float* gb = part_bins + ((static_cast<int64_t>(s) * H + h) * nsplit + split) * static_cast<int64_t>(max_ref) * G;
      uint32_t* bins = GB ? reinterpret_cast<uint32_t*>(gb) : sbins;
      if (q_it != it) fetch_q(it);  // only when the item before it was skipped
      uint32_t qb[NKS][2][kDup ? 1 : 2];  // B fragments of q': [k-step][k half][hi / lo]
#pragma unroll
      for (int ks = 0; ks < NKS; ++ks)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t hi, lo;
          split_pack(qn[ks][half][0], qn[ks][half][1], hi, lo);
          if constexpr (kDup) {
            qb[ks][half][0] = gq < 4 ? hi : lo;
          } else {
            qb[ks][half][0] = hi;
            qb[ks][half][1] = lo;
          }
        }
      const float qm0 = qmn[0], qm1 = qmn[1];
      if (it + static_cast<int>(gridDim.x) < n_items) fetch_q(it + gridDim.x);  // in flight during this item
      float m_all[G];
#pragma unroll
      for (int g = 0; g < G; ++g) m_all[g] = -INFINITY;
      float m2[2] = {-INFINITY, -INFINITY}, l2[2] = {0.f, 0.f};
      float acc[NKS][4];
#pragma unroll
      for (int dt = 0; dt < NKS; ++dt)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[dt][c] = 0.f;
      // Mass bins start at zero; the first stage's barrier below orders these stores before any atomic add.
      // 16-byte stores: jcap * G is a multiple of 4 (G >= 4) and the bins start 1024-byte aligned
      for (int e = tid; e < jcap * G / 4; e += kMmaNCW * 32)
        reinterpret_cast<uint4*>(bins)[e] = make_uint4(0u, 0u, 0u, 0u);

      for (int st = 0; st < nst; ++st) {
        mbar_wait(smem_u32(gath + slot), ph, sAbort);  // a timeout raises the abort flag
        const uint8_t* sc8 = stages + slot * C::STAGE_BYTES;
        const uint32_t kbase = smem_u32(sc8);  // column c of a token row: tile c / 64, 16-byte chunk (c % 64) / 8
        const int* si = reinterpret_cast<const int*>(sc8 + C::CODE_BYTES);
        const float* sg = reinterpret_cast<const float*>(sc8 + C::CODE_BYTES + C::IDX_BYTES);
        const int tok_base = t_begin + st * STG;
        const int lim = t_end - tok_base;  // tokens of this stage that lie inside the context
        if constexpr (Q4) {
          // 4-bit codes: this warp expands the packed rows it reads into its bf16 tiles (exact: offset binary
          // in a bf16 mantissa minus 136), zero rows past the end; each lane takes words lane, lane + 32, ...
          // of the group's 16 rows.
          constexpr int W = RK / 4;  // nibble words (8 codes) per token row
          uint8_t* scw = stages + slot * C::STAGE_BYTES;
#pragma unroll
          for (int gr = 0; gr < NGR; ++gr)
#pragma unroll
            for (int v = 0; v < 16 * W / 32; ++v) {
              const int e = lane + 32 * v, row = e / W, wi = e % W;
              const int tok = w32 + gr * 16 + row;
              const uint32_t wd = *reinterpret_cast<const uint32_t*>(scw + C::Q4ROW_OFF + tok * RK + wi * 4);
              const uint4 o = tok < lim ? q4_word_to_bf16x8(wd) : make_uint4(0u, 0u, 0u, 0u);
              *reinterpret_cast<uint4*>(scw + (swz(kbase + (wi / 8) * C::TILE_BYTES, tok, wi % 8) - kbase)) = o;
            }
          __syncwarp();  // the warp's ldmatrix reads of these rows follow
        }

        // scores S[t][col] = cK[t][:] . Bq[:][col] of both groups
        float sc[NGR][4];
#pragma unroll
        for (int gr = 0; gr < NGR; ++gr) {
#pragma unroll
          for (int c = 0; c < 4; ++c) sc[gr][c] = 0.f;
#pragma unroll
          for (int ks = 0; ks < NKS; ++ks) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(kbase + offK[ks] + gr * 2048, a0, a1, a2, a3);
            mma_bf16_16816_a4(sc[gr], a0, a1, a2, a3, qb[ks][0][0], qb[ks][1][0]);
            if constexpr (!kDup) mma_bf16_16816_a4(sc[gr], a0, a1, a2, a3, qb[ks][0][1], qb[ks][1][1]);
          }
        }
        if constexpr (kDup) {
#pragma unroll
          for (int gr = 0; gr < NGR; ++gr)
#pragma unroll
            for (int c = 0; c < 4; ++c) sc[gr][c] += __shfl_xor_sync(0xffffffffu, sc[gr][c], 2);
        }
        // s2 for rows gq (c = 0, 1) and gq + 8 (c = 2, 3), heads hb (even c) and hb + 1 (odd c)
        float s2[NGR][4];
        int ix[NGR][2];
        int ixk[NGR][2][KT];   // k-nearest retrieval: the rows' slot ordinals (-1 unfilled)
        float kinv[NGR][2];     // and 1 / (filled slots)
        float svr[NGR][2];  // 4-bit codes: V scales of rows gq, gq + 8
#pragma unroll
        for (int gr = 0; gr < NGR; ++gr) svr[gr][0] = svr[gr][1] = 1.f;
        bool up = false;  // a score of this lane above its head's running maximum by more than 2^kRescaleLog2
#pragma unroll
        for (int gr = 0; gr < NGR; ++gr)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            const int tok = w32 + gr * 16 + gq + 8 * hr;
            const bool vt = tok < lim;
            float2 g2;
            if constexpr (KT == 1) {
              ix[gr][hr] = si[tok];  // range-checked by the gatherer
              g2 = *reinterpret_cast<const float2*>(sg + tok * G + hb);
            } else {  // the mean of the filled slots' q.r~K rows
              g2 = make_float2(0.f, 0.f);
              int cnt = 0;
#pragma unroll
              for (int q = 0; q < KT; ++q) {
                const int j = si[tok * KT + q];
                ixk[gr][hr][q] = j;
                if (j >= 0) {
                  const float2 gg = *reinterpret_cast<const float2*>(sg + (tok * KT + q) * G + hb);
                  g2.x += gg.x;
                  g2.y += gg.y;
                  ++cnt;
                }
              }
              kinv[gr][hr] = cnt > 0 ? 1.f / static_cast<float>(cnt) : 0.f;
              g2.x *= kinv[gr][hr];
              g2.y *= kinv[gr][hr];
            }
            float skc = 1.f;  // 4-bit codes: the MMA ran on the integer levels; the K scale restores the score
            if constexpr (Q4) {  // the token's (K, V) scales, bf16 in the staged block
              const uint32_t sp = *reinterpret_cast<const uint32_t*>(sc8 + C::Q4SC_OFF + tok * 4);
              skc = vt ? __uint_as_float(sp << 16) : 0.f;
              svr[gr][hr] = vt ? __uint_as_float(sp & 0xffff0000u) : 0.f;
            }
            s2[gr][2 * hr] = vt ? qm0 + g2.x + skc * sc[gr][2 * hr] : -INFINITY;
            s2[gr][2 * hr + 1] = vt ? qm1 + g2.y + skc * sc[gr][2 * hr + 1] : -INFINITY;
            up = up || s2[gr][2 * hr] > m2[0] + kRescaleLog2 || s2[gr][2 * hr + 1] > m2[1] + kRescaleLog2;
          }
        // One CTA-wide vote per stage: does any score lie above its head's running maximum by more than
        // 2^kRescaleLog2, or has a wait timed out?  Both are rare, and only then are the stage maxima
        // exchanged (a second vote tells an abort apart, on the flag value this thread voted with).
        const bool ab = *sAbort != 0;
        if (named_bar_or(1, kMmaNCW * 32, up || ab)) {
          if (named_bar_or(1, kMmaNCW * 32, ab)) {
            aborted = true;
            break;
          }
          float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
          for (int gr = 0; gr < NGR; ++gr)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
              mx0 = fmaxf(mx0, s2[gr][2 * hr]);
              mx1 = fmaxf(mx1, s2[gr][2 * hr + 1]);
            }
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
          }
          // [G][NCW]; written only after a vote that every consumer thread reaches once it has read the
          // maxima of an earlier exchange, so one buffer serves every stage
          if (gq == 0 && (!kDup || tq < 2)) {
            wmax[hb * kMmaNCW + warp] = mx0;
            wmax[(hb + 1) * kMmaNCW + warp] = mx1;
          }
          named_bar_sync(1, kMmaNCW * 32);
          // per-head factors for every head (the mass bins hold all heads); every consumer thread reads the
          // same shared maxima, so every decision below is uniform
          bool rescale_bins = false;
          float alpha[G];
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float M = stage_max_row(wmax + g * kMmaNCW);
            alpha[g] = 1.f;
            if (M > m_all[g] + kRescaleLog2) {
              if (m_all[g] != -INFINITY) {
                alpha[g] = fast_exp2(m_all[g] - M);
                rescale_bins = true;
              } else {
                alpha[g] = 0.f;
              }
              m_all[g] = M;
            }
          }
          float a0 = 1.f, a1 = 1.f;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            if (g == hb) {
              a0 = alpha[g];
              m2[0] = m_all[g];
            }
            if (g == hb + 1) {
              a1 = alpha[g];
              m2[1] = m_all[g];
            }
          }
          l2[0] *= a0;
          l2[1] *= a1;
#pragma unroll
          for (int dt = 0; dt < NKS; ++dt) {
            acc[dt][0] *= a0;
            acc[dt][1] *= a1;
            acc[dt][2] *= a0;
            acc[dt][3] *= a1;
          }
          if (rescale_bins) {
            for (int e = tid; e < jcap * G; e += kMmaNCW * 32) {
              float a = 1.f;
#pragma unroll
              for (int g = 0; g < G; ++g)
                if (e % G == g) a = alpha[g];
              bins[e] = __float2uint_rn(static_cast<float>(bins[e]) * a);
            }
            named_bar_sync(1, kMmaNCW * 32);
          }
        }
        // softmax weights, mass per reference, and the V product per group
#pragma unroll
        for (int gr = 0; gr < NGR; ++gr) {
          float p[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) p[c] = fast_exp2(s2[gr][c] - m2[c & 1]);  // s2 = -inf gives 0
          l2[0] += p[0] + p[2];
          l2[1] += p[1] + p[3];
          // Mass of heads hb and hb + 1 (two 32-bit shared atomics: measured cheaper than one 64-bit add).
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            if (kDup && hr != rh) continue;
            if (s2[gr][2 * hr] != -INFINITY) {
              if constexpr (KT == 1) {
                uint32_t* bj = bins + ix[gr][hr] * G + hb;
                atomicAdd(bj, mass_fixed(p[2 * hr]));
                atomicAdd(bj + 1, mass_fixed(p[2 * hr + 1]));
              } else {  // the token's weight spreads evenly over its filled slots
                const uint32_t m0 = mass_fixed(p[2 * hr] * kinv[gr][hr]);
                const uint32_t m1 = mass_fixed(p[2 * hr + 1] * kinv[gr][hr]);
#pragma unroll
                for (int q = 0; q < KT; ++q) {
                  if (ixk[gr][hr][q] < 0) continue;
                  uint32_t* bj = bins + ixk[gr][hr][q] * G + hb;
                  atomicAdd(bj, m0);
                  atomicAdd(bj + 1, m1);
                }
              }
            }
          }
          // B operand of the V product (k = the group's 16 tokens, n = the 8 columns): the p fragment holds
          // rows gq / gq + 8 and columns 2tq, 2tq + 1 of two 8x8 blocks, movmatrix transposes each block.
          uint32_t w0h, w0l, w1h, w1l;
          // (4-bit codes: the V product runs on the integer levels, so each row's weight carries its V scale)
          split_pack(p[0] * svr[gr][0], p[1] * svr[gr][0], w0h, w0l);  // token row gq
          split_pack(p[2] * svr[gr][1], p[3] * svr[gr][1], w1h, w1l);  // token row gq + 8
          uint32_t b0, b1, b0l = 0u, b1l = 0u;
          if constexpr (kDup) {
            b0 = movmatrix_t(tq < 2 ? w0h : w0l);  // columns 0..3 carry p_hi, columns 4..7 p_lo
            b1 = movmatrix_t(tq < 2 ? w1h : w1l);
          } else {
            b0 = movmatrix_t(w0h);
            b1 = movmatrix_t(w1h);
            b0l = movmatrix_t(w0l);
            b1l = movmatrix_t(w1l);
          }
#pragma unroll
          for (int dt = 0; dt < NKS; ++dt) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(kbase + offV[dt] + gr * 2048, a0, a1, a2, a3);
            mma_bf16_16816_a4(acc[dt], a0, a1, a2, a3, b0, b1);
            if constexpr (!kDup) mma_bf16_16816_a4(acc[dt], a0, a1, a2, a3, b0l, b1l);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(empty + slot));
        if (++slot == nstages) {
          slot = 0;
          ph ^= 1u;
        }
      }
      named_bar_sync(1, kMmaNCW * 32);  // all mass adds done (every consumer reaches this once)
      if (aborted) return;

      // 16-byte loads and stores (gb is 16-byte aligned: max_ref * G is a multiple of 4 for G >= 4); GB: the
      // conversion is in place, each thread reading its own words before writing them
      for (int e = tid; e < jcap * G / 4; e += kMmaNCW * 32) {
        const uint4 b = reinterpret_cast<const uint4*>(bins)[e];
        reinterpret_cast<float4*>(gb)[e] =
            make_float4(static_cast<float>(b.x) * kMassScaleInv, static_cast<float>(b.y) * kMassScaleInv,
                        static_cast<float>(b.z) * kMassScaleInv, static_cast<float>(b.w) * kMassScaleInv);
      }
      if constexpr (kDup) {
#pragma unroll
        for (int dt = 0; dt < NKS; ++dt)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[dt][c] += __shfl_xor_sync(0xffffffffu, acc[dt][c], 2);  // hi + lo
      }
      if (!kDup || tq < 2) {
#pragma unroll
        for (int dt = 0; dt < NKS; ++dt) {
          const int d0 = 16 * dt + gq;
          red[(warp * G + hb) * RK + d0] = acc[dt][0];
          red[(warp * G + hb + 1) * RK + d0] = acc[dt][1];
          red[(warp * G + hb) * RK + d0 + 8] = acc[dt][2];
          red[(warp * G + hb + 1) * RK + d0 + 8] = acc[dt][3];
        }
      }
      float la = l2[0], lb = l2[1];
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        la += __shfl_xor_sync(0xffffffffu, la, o);
        lb += __shfl_xor_sync(0xffffffffu, lb, o);
      }
      if (gq == 0 && (!kDup || tq < 2)) {
        lred[warp * G + hb] = la;
        lred[warp * G + hb + 1] = lb;
      }
      named_bar_sync(1, kMmaNCW * 32);
      for (int e = tid; e < G * RK; e += kMmaNCW * 32) {
        const int g = e / RK, o = e % RK;
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < kMmaNCW; ++w) a += red[(w * G + g) * RK + o];
        part_acc[(ml_base + g * nsplit) * RK + o] = a;
      }
      if (tid < G) {
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kMmaNCW; ++w) L += lred[w * G + tid];
        float mt = -INFINITY;
#pragma unroll
        for (int g = 0; g < G; ++g)
          if (g == tid) mt = m_all[g];
        part_ml[(ml_base + tid * nsplit) * 2] = mt;
        part_ml[(ml_base + tid * nsplit) * 2 + 1] = L;
      }
    }
  } else {
    // Query heads are the MMA rows: row gq carries the bf16 hi half of head gq's q' (or p) and row gq + 8 its
    // lo half, so one MMA takes both halves and the two accumulator rows are added per item.
    const int gq = lane >> 2, tq = lane & 3;  // fragment row (query head) and column pair
    const bool head_ok = gq < G;
    const int w32 = warp * (STG / kMmaNCW);  // this warp's first token in the stage
    int it = blockIdx.x;
    SeqExtent ext_n = it < n_items ? seq_extent<SPARSE>(context_lens, cu_sel, it / (H * nsplit), max_ctx, max_sel)
                                  : SeqExtent{0, 0, 0};
    int slot = 0;
    uint32_t ph = 0;  // ring slot and the parity of its current phase, carried across items
    bool aborted = false;
    for (; it < n_items; it += gridDim.x) {
      const SeqExtent ext = ext_n;
      if (it + static_cast<int>(gridDim.x) < n_items)
        ext_n = seq_extent<SPARSE>(context_lens, cu_sel, (it + gridDim.x) / (H * nsplit), max_ctx, max_sel);
      const int split = it % nsplit, h = (it / nsplit) % H, s = it / (H * nsplit);
      const int t_begin = split * tps, t_end = min(ext.n, t_begin + tps);
      if (t_begin >= t_end) continue;
      const int nst = ceil_div_d(t_end - t_begin, STG);
      const int jcap = split_jcap<SPARSE>(ext, t_end, R);
      const int hq0 = h * G;
      const int64_t ml_base = (static_cast<int64_t>(s) * Hq + hq0) * nsplit + split;  // + g * nsplit
      float* gb = part_bins + ((static_cast<int64_t>(s) * H + h) * nsplit + split) * static_cast<int64_t>(max_ref) * G;
      uint32_t* bins = GB ? reinterpret_cast<uint32_t*>(gb) : sbins;
      uint32_t qa_hi[RK / 16][2], qa_lo[RK / 16][2];
      {
        const float* qrow = qp + (static_cast<int64_t>(s) * Hq + hq0 + (head_ok ? gq : 0)) * RK;
#pragma unroll
        for (int ks = 0; ks < RK / 16; ++ks)
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int k0 = 16 * ks + 8 * half + 2 * tq;
            const float x0 = head_ok ? qrow[k0] : 0.f, x1 = head_ok ? qrow[k0 + 1] : 0.f;
            split_pack(x0, x1, qa_hi[ks][half], qa_lo[ks][half]);
          }
      }
      const float qm = head_ok ? qmu[static_cast<int64_t>(s) * Hq + hq0 + gq] : 0.f;
      float m_all[G];
#pragma unroll
      for (int g = 0; g < G; ++g) m_all[g] = -INFINITY;
      float m_own = -INFINITY, l_own = 0.f;
      float acc[NDT][4];
#pragma unroll
      for (int dt = 0; dt < NDT; ++dt)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[dt][c] = 0.f;
      // Mass bins start at zero; the first stage's barrier below orders these stores before any atomic add.
      for (int e = tid; e < jcap * G; e += kMmaNCW * 32) bins[e] = 0u;

      for (int st = 0; st < nst; ++st) {
        mbar_wait(smem_u32(gath + slot), ph, sAbort);  // a timeout raises the abort flag
        const uint8_t* sc8 = stages + slot * C::STAGE_BYTES;
        const uint32_t kbase = smem_u32(sc8);  // column c of a token row: tile c / 64, 16-byte chunk (c % 64) / 8
        const int* si = reinterpret_cast<const int*>(sc8 + C::CODE_BYTES);
        const float* sg = reinterpret_cast<const float*>(sc8 + C::CODE_BYTES + C::IDX_BYTES);
        const int tok_base = t_begin + st * STG;

        // scores of both groups (two 8-token column tiles each)
        float scf[NGRP][2][4];
#pragma unroll
        for (int gr = 0; gr < NGRP; ++gr)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int c = 0; c < 4; ++c) scf[gr][nt][c] = 0.f;
            const int row = w32 + gr * 16 + nt * 8 + (lane & 7);
#pragma unroll
            for (int kq = 0; kq < RK / 32; ++kq) {  // 32 K-code columns per ldmatrix.x4 (K codes lie in tile 0)
              uint32_t b[4];
              ldsm_x4(swz(kbase, row, 4 * kq + (lane >> 3)), b[0], b[1], b[2], b[3]);
#pragma unroll
              for (int kk = 0; kk < 2; ++kk) {
                const int ks = kq * 2 + kk;
                // rows gq: q'_hi of head gq; rows gq + 8: its q'_lo (one MMA for both halves)
                mma_bf16_16816_a4(scf[gr][nt], qa_hi[ks][0], qa_lo[ks][0], qa_hi[ks][1], qa_lo[ks][1], b[2 * kk],
                                  b[2 * kk + 1]);
              }
            }
          }
        // s2 for head gq and tokens w32 + gr*16 + nt*8 + 2tq (+1)
        float s2[NGRP][2][2];
        int ix[NGRP][2][2];
        bool up = false;  // a score of this lane above its head's running maximum by more than 2^kRescaleLog2
#pragma unroll
        for (int gr = 0; gr < NGRP; ++gr)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int tok = w32 + gr * 16 + nt * 8 + 2 * tq + e;
              const bool vt = head_ok && tok_base + tok < t_end;
              ix[gr][nt][e] = si[tok];  // range-checked by the gatherer
              s2[gr][nt][e] = vt ? qm + sg[tok * G + gq] + (scf[gr][nt][e] + scf[gr][nt][e + 2]) : -INFINITY;
              up = up || s2[gr][nt][e] > m_own + kRescaleLog2;
            }
        // One CTA-wide vote per stage on a raised maximum or a timed-out wait; only then are the stage maxima
        // exchanged (the second vote tells an abort apart, on the flag value this thread voted with).
        const bool ab = *sAbort != 0;
        if (named_bar_or(1, kMmaNCW * 32, up || ab)) {
          if (named_bar_or(1, kMmaNCW * 32, ab)) {
            aborted = true;
            break;
          }
          float mx = -INFINITY;
#pragma unroll
          for (int gr = 0; gr < NGRP; ++gr)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int e = 0; e < 2; ++e) mx = fmaxf(mx, s2[gr][nt][e]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          // [G][NCW]; written only after a vote that every consumer thread reaches once it has read the
          // maxima of an earlier exchange, so one buffer serves every stage
          if (tq == 0 && head_ok) wmax[gq * kMmaNCW + warp] = mx;
          named_bar_sync(1, kMmaNCW * 32);
          // per-head factors for every head (the mass bins hold all heads); uniform over the consumer threads
          bool rescale_bins = false;
          float alpha[G];
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float M = stage_max_row(wmax + g * kMmaNCW);
            alpha[g] = 1.f;
            if (M > m_all[g] + kRescaleLog2) {
              if (m_all[g] != -INFINITY) {
                alpha[g] = fast_exp2(m_all[g] - M);
                rescale_bins = true;
              } else {
                alpha[g] = 0.f;
              }
              m_all[g] = M;
            }
          }
          float a_own = 1.f;
#pragma unroll
          for (int g = 0; g < G; ++g)
            if (g == gq) {
              a_own = alpha[g];
              m_own = m_all[g];
            }
          l_own *= a_own;
#pragma unroll
          for (int dt = 0; dt < NDT; ++dt)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[dt][c] *= a_own;
          if (rescale_bins) {
            for (int e = tid; e < jcap * G; e += kMmaNCW * 32) {
              float a = 1.f;
#pragma unroll
              for (int g = 0; g < G; ++g)
                if (e % G == g) a = alpha[g];
              bins[e] = __float2uint_rn(static_cast<float>(bins[e]) * a);
            }
            named_bar_sync(1, kMmaNCW * 32);
          }
        }
        // softmax weights, mass per reference, and V products per group
#pragma unroll
        for (int gr = 0; gr < NGRP; ++gr) {
          float p[2][2];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              p[nt][e] = fast_exp2(s2[gr][nt][e] - m_own);  // s2 = -inf gives 0
              l_own += p[nt][e];
              if (s2[gr][nt][e] != -INFINITY)
                atomicAdd(bins + ix[gr][nt][e] * G + gq, __float2uint_rn(p[nt][e] * kMassScale));
            }
          uint32_t pa_hi[2], pa_lo[2];
          split_pack(p[0][0], p[0][1], pa_hi[0], pa_lo[0]);  // a0: tokens 2tq, 2tq+1 of column tile 0
          split_pack(p[1][0], p[1][1], pa_hi[1], pa_lo[1]);  // a2: tokens 8 + 2tq, +1
#pragma unroll
          for (int dp = 0; dp < RK / 16; ++dp) {  // pairs of 8-wide V dimension tiles
            const int mat = lane >> 3;             // matrix: (token half = mat & 1, dimension tile 2dp + (mat >> 1))
            const int row = w32 + gr * 16 + (mat & 1) * 8 + (lane & 7);
            const int col = RK + 8 * (2 * dp + (mat >> 1));  // V codes start at column r
            uint32_t b[4];
            ldsm_x4_t(swz(kbase + (col / 64) * C::TILE_BYTES, row, (col % 64) / 8), b[0], b[1], b[2], b[3]);
            // rows gq: p_hi of head gq; rows gq + 8: its p_lo (summed once, when the item is written out)
            mma_bf16_16816_a4(acc[2 * dp], pa_hi[0], pa_lo[0], pa_hi[1], pa_lo[1], b[0], b[1]);
            mma_bf16_16816_a4(acc[2 * dp + 1], pa_hi[0], pa_lo[0], pa_hi[1], pa_lo[1], b[2], b[3]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(empty + slot));
        if (++slot == nstages) {
          slot = 0;
          ph ^= 1u;
        }
      }
      named_bar_sync(1, kMmaNCW * 32);  // all mass adds done (every consumer reaches this once)
      if (aborted) return;

      // (GB: in place, each thread reading its own word before writing it)
      for (int e = tid; e < jcap * G; e += kMmaNCW * 32) gb[e] = static_cast<float>(bins[e]) * kMassScaleInv;
      if (head_ok) {
#pragma unroll
        for (int dt = 0; dt < NDT; ++dt) {
          red[(warp * G + gq) * RK + dt * 8 + 2 * tq] = acc[dt][0] + acc[dt][2];  // hi rows + lo rows
          red[(warp * G + gq) * RK + dt * 8 + 2 * tq + 1] = acc[dt][1] + acc[dt][3];
        }
      }
      float lv = l_own;
      lv += __shfl_xor_sync(0xffffffffu, lv, 1);
      lv += __shfl_xor_sync(0xffffffffu, lv, 2);
      if (tq == 0 && head_ok) lred[warp * G + gq] = lv;
      named_bar_sync(1, kMmaNCW * 32);
      for (int e = tid; e < G * RK; e += kMmaNCW * 32) {
        const int g = e / RK, o = e % RK;
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < kMmaNCW; ++w) a += red[(w * G + g) * RK + o];
        part_acc[(ml_base + g * nsplit) * RK + o] = a;
      }
      if (tid < G) {
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kMmaNCW; ++w) L += lred[w * G + tid];
        part_ml[(ml_base + tid * nsplit) * 2] = m_all[tid];
        part_ml[(ml_base + tid * nsplit) * 2 + 1] = L;
      }
    }
  }
}

// ------------------------------------------------------------------------------------------------
// Combine.  CTA = (chunk of kCombineRefs references, kv head, sequence), 256 threads.
//   1. asynchronous copies of the chunk's V reference rows into shared memory (they do not depend on the
//      split kernel's results), and the first batch of mass bins into registers
//   2. split weights alpha_k = 2^(m_k - M) and the mass L per query head
//   3. reference mass w_j = sum_k alpha_k bins_k[j], two threads per reference (even / odd splits)
//   4. partial[g][:] = sum_j w_j r~V_j over the chunk, written to the workspace
//   5. the last chunk CTA of a (seq, kv head) adds the partials, acc B_V^T and mu_V, divides by L
// ------------------------------------------------------------------------------------------------
// V-row stride in the combine's shared memory: bf16 rows are padded by 16 bytes so that ldmatrix reads of
// 8 consecutive rows fall in distinct banks
template <typename T, int D>
__host__ __device__ constexpr int combine_vstride() { return sizeof(T) == 2 ? D + 8 : D; }

template <typename T, int D, int G>
__host__ __device__ constexpr int combine_vrow_bytes(int r) {
  return ((kCombineRefs * combine_vstride<T, D>() * static_cast<int>(sizeof(T)) > (G * r + D * (r + 1)) * 4
               ? kCombineRefs * combine_vstride<T, D>() * static_cast<int>(sizeof(T))
               : (G * r + D * (r + 1)) * 4) + 15) / 16 * 16;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(256) decode_combine_kernel(
    const T* __restrict__ refs, const T* __restrict__ basis, const float* __restrict__ mu,
    const int* __restrict__ context_lens, const int* __restrict__ block_tables, int max_blocks, int num_blocks,
    int Hq, int H, int r, int R, int max_ctx, int max_ref, int tps, int nsplit, int nchunk,
    const float* __restrict__ part_ml, const float* __restrict__ part_acc, const float* __restrict__ part_bins,
    float* __restrict__ cpart, int* __restrict__ counters, T* __restrict__ out, float* __restrict__ lse,
    const int* __restrict__ cu_sel, int max_sel) {
  constexpr int V = 16 / sizeof(T);
  constexpr int VPR = D / V;                                 // 16-byte vectors per V reference row
  constexpr int NBV = (D * 64 * static_cast<int>(sizeof(T)) / 16 + 255) / 256;  // B_V vectors per thread (r <= 64)
  extern __shared__ __align__(16) unsigned char smc_raw[];
  // V rows (storage type); the finishing CTA reuses this area for acc [G][r] and B_V [D][r+1] (fp32)
  const int vrow_bytes = combine_vrow_bytes<T, D, G>(r);
  constexpr int VS = combine_vstride<T, D>();
  T* vrows = reinterpret_cast<T*>(smc_raw);                  // [kCombineRefs][VS]
  float* alpha = reinterpret_cast<float*>(smc_raw + vrow_bytes);  // [G][nsplit]
  float* Ls = alpha + G * nsplit;                            // [G]
  float* Ms = Ls + G;                                        // [G]
  float* w = Ms + G;                                         // [2][kCombineRefs][G]
  // bf16: the masses as hi + lo A fragments [k-step][lane] (16-byte aligned), built once for every warp
  uint4* wfrag = reinterpret_cast<uint4*>(
      smc_raw + ((static_cast<size_t>(vrow_bytes) + (G * nsplit + 2 * G + 2 * kCombineRefs * G) * 4 + 15) & ~size_t(15)));
  __shared__ int s_last;

  const int c = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const int jbase = c * kCombineRefs;
  // The block ids of this thread's V-row pieces are read while the context length is in flight (all loads
  // at once, j < max_ref <= max_blocks keeps them inside the table) and range-checked once it is known.
  constexpr int NCV = kCombineRefs * VPR / 256;  // 16-byte V-row pieces per thread
  int pbv[NCV];
#pragma unroll
  for (int u = 0; u < NCV; ++u) {
    const int jj = (tid + u * 256) / VPR;
    pbv[u] = jbase + jj < max_ref ? __ldg(block_tables + static_cast<int64_t>(s) * max_blocks + jbase + jj) : 0;
  }
  const int ctx = checked_ctx(context_lens, s, max_ctx);
  const int n_ref = ceil_div_d(ctx, R);
  const int nneed = n_ref > 0 ? ceil_div_d(n_ref, kCombineRefs) : 1;
  if (c >= nneed) return;
  const int hq0 = h * G;
  // splits that ran: over the context (dense) or over the selected list (sparse, cu_sel != nullptr)
  int nspan = ctx;
  if (cu_sel != nullptr) {
    const int a0 = __ldg(cu_sel + s);
    nspan = __ldg(cu_sel + s + 1) - a0;
    if (a0 < 0 || nspan < 0 || nspan > max_sel) nspan = 0;  // recorded by the split kernel
  }
  const int nsp_used = nspan > 0 ? ceil_div_d(nspan, tps) : 0;
  const int nj = max(0, min(kCombineRefs, n_ref - jbase));

  // 1. V reference rows of this chunk -> shared memory (the copies depend on no further global read)
#pragma unroll
  for (int u = 0; u < NCV; ++u) {
    const int e = tid + u * 256, jj = e / VPR, cv = e % VPR;
    if (jj < nj) {
      int pb = pbv[u];
      if (pb < 0 || pb >= num_blocks) {
        record_error(DKV_DEVERR_BLOCK_ID);
        pb = 0;  // read a valid block instead; the error word reports the bad table
      }
      cp_async16(vrows + jj * VS + cv * V, refs + (static_cast<int64_t>(pb) * H + h) * 2 * D + D + cv * V);
    }
  }
  cp_async_commit();
  if constexpr (sizeof(T) == 2) {
    // rows past the chunk's references are read by the tensor-core product (with zero weight): zero them,
    // since 0 * (stale NaN bits) would not be zero
    for (int e = tid; e < (kCombineRefs - nj) * VPR; e += 256)
      *reinterpret_cast<uint4*>(vrows + (nj + e / VPR) * VS + (e % VPR) * V) = make_uint4(0u, 0u, 0u, 0u);
  }
  // Everything above reads inputs of the decode call only; the split kernel's partials are read below, once
  // that grid has completed (this kernel may have been launched before it finished).
  griddep_wait();
  // 2a. the first batch of this thread's mass bins (3. below) is loaded now, so that its latency overlaps the
  //     split weights: reference j is at jj = tid % kCombineRefs, splits k = k0 + par, k0 + par + 2, ...
  const int jj = tid % kCombineRefs, par = tid / kCombineRefs;
  const int j = jbase + jj;
  // dense: splits ending at or before token jR never saw reference j; sparse: any split may have
  const int k0 = cu_sel != nullptr ? 0 : (j * R) / tps;
  constexpr int KB = 8;  // splits per batch in flight
  const float* b0 = part_bins + (static_cast<int64_t>(s) * H + h) * nsplit * static_cast<int64_t>(max_ref) * G +
                    static_cast<int64_t>(j) * G;
  const int64_t kstride = static_cast<int64_t>(max_ref) * G;
  float bb[KB][G];
  auto load_batch = [&](int kb) {
#pragma unroll
    for (int i = 0; i < KB; ++i) {
      const int k = kb + 2 * i;
      const float* b = b0 + k * kstride;
      if (jj < nj && k < nsp_used) {
        if constexpr (G % 4 == 0) {
#pragma unroll
          for (int g4 = 0; g4 < G / 4; ++g4) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(b) + g4);
            bb[i][4 * g4] = v.x, bb[i][4 * g4 + 1] = v.y, bb[i][4 * g4 + 2] = v.z, bb[i][4 * g4 + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int g = 0; g < G; ++g) bb[i][g] = __ldcg(b + g);
        }
      } else {
#pragma unroll
        for (int g = 0; g < G; ++g) bb[i][g] = 0.f;
      }
    }
  };
  load_batch(k0 + par);

  // 2. split weights per query head: warp g reduces over the splits
  for (int g = warp; g < G; g += 8) {
    const float2* ml = reinterpret_cast<const float2*>(part_ml) + (static_cast<int64_t>(s) * Hq + hq0 + g) * nsplit;
    float M = -INFINITY;
    for (int k = lane; k < nsp_used; k += 32) M = fmaxf(M, __ldcg(&ml[k].x));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int k = lane; k < nsplit; k += 32) {
      float a = 0.f;
      if (k < nsp_used) {
        const float2 v = __ldcg(&ml[k]);
        if (M != -INFINITY && v.x != -INFINITY) a = exp2f(v.x - M);
        L += a * v.y;
      }
      alpha[g * nsplit + k] = a;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) {
      Ls[g] = L;
      Ms[g] = M;
    }
  }
  __syncthreads();

  // 3. w_j = sum_k alpha_k bins_k[j]; splits whose tokens end before reference j never touched it.  Eight
  //    splits' loads in flight per batch, then the multiply-adds in split order.
  {
    float wv[G];
#pragma unroll
    for (int g = 0; g < G; ++g) wv[g] = 0.f;
    if (jj < nj) {
      for (int kb = k0 + par; kb < nsp_used; kb += 2 * KB) {
        if (kb != k0 + par) load_batch(kb);
#pragma unroll
        for (int i = 0; i < KB; ++i) {
          const int k = kb + 2 * i;
          if (k < nsp_used) {
#pragma unroll
            for (int g = 0; g < G; ++g) wv[g] = fmaf(alpha[g * nsplit + k], bb[i][g], wv[g]);
          }
        }
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) w[(par * kCombineRefs + jj) * G + g] = wv[g];
  }
  cp_async_wait_all();
  __syncthreads();

  // 4. partial[g][dd] = sum_j w_j r~V_j[dd] over this chunk of references
  float* cp = cpart + ((static_cast<int64_t>(s) * H + h) * nchunk + c) * G * D;
  if constexpr (sizeof(T) == 2) {
    // the masses as A fragments (heads as rows, references as k; bf16 hi + lo), one (k-step, lane) slot per
    // thread, so that the warps below only load them
    static_assert(kCombineRefs / 16 * 32 == 256, "one fragment slot per thread");
    {
      const int ks = tid >> 5, gq = (tid & 31) >> 2, tq = tid & 3;
      float wa[4] = {0.f, 0.f, 0.f, 0.f};
      if (gq < G) {
        const int j0 = ks * 16 + 2 * tq;
        const int jx[4] = {j0, j0 + 1, j0 + 8, j0 + 9};
#pragma unroll
        for (int q = 0; q < 4; ++q) wa[q] = w[jx[q] * G + gq] + w[(kCombineRefs + jx[q]) * G + gq];
      }
      uint4 f;
      split_pack(wa[0], wa[1], f.x, f.z);
      split_pack(wa[2], wa[3], f.y, f.w);
      wfrag[tid] = f;
    }
    __syncthreads();
    // on the tensor cores: [heads x references] x [references x d] with mma.sync m16n8k16; the masses are
    // split into bf16 hi + lo (about 16 mantissa bits; hi in rows 0..7, lo in rows 8..15 of one MMA), the V
    // rows are exact bf16.  Warp w takes dimensions
    // 16w .. 16w + 15 (D / 16 warps are active).
    if (warp < D / 16) {
      const int gq = lane >> 2, tq = lane & 3;
      float acc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[nt][q] = 0.f;
      const uint32_t vb = smem_u32(vrows + ((lane & 7) + 8 * ((lane >> 3) & 1)) * VS + warp * 16 + 8 * (lane >> 4));
#pragma unroll
      for (int ks = 0; ks < kCombineRefs / 16; ++ks) {
        const uint4 f = wfrag[ks * 32 + lane];
        const uint32_t a0h = f.x, a2h = f.y, a0l = f.z, a2l = f.w;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + ks * 16 * VS * 2, b0, b1, b2, b3);
        // rows gq: the masses' hi halves; rows gq + 8: their lo halves (added below)
        mma_bf16_16816_a4(acc[0], a0h, a0l, a2h, a2l, b0, b1);
        mma_bf16_16816_a4(acc[1], a0h, a0l, a2h, a2l, b2, b3);
      }
      if (gq < G) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
          *reinterpret_cast<float2*>(cp + gq * D + warp * 16 + nt * 8 + 2 * tq) =
              make_float2(acc[nt][0] + acc[nt][2], acc[nt][1] + acc[nt][3]);
      }
    }
  } else {
    constexpr int NGS = 256 / D;  // thread groups over query heads
    const int dd = tid % D, gs = tid / D;
    float pa[G];
#pragma unroll
    for (int g = 0; g < G; ++g) pa[g] = 0.f;
#pragma unroll 4
    for (int jj = 0; jj < nj; ++jj) {
      const float vv = Elem<T>::to_f(vrows[jj * VS + dd]);
#pragma unroll
      for (int g = 0; g < G; ++g)
        if (g % NGS == gs) pa[g] = fmaf(w[jj * G + g] + w[(kCombineRefs + jj) * G + g], vv, pa[g]);
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
      if (g % NGS == gs) cp[g * D + dd] = pa[g];
  }

  // 5. the last chunk CTA of this (seq, kv head) finishes
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(counters + static_cast<int64_t>(s) * H + h, 1);
    s_last = prev == nneed - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // acc_g = sum_k alpha_k acc_k (as [G][r]) and B_V as [D][r+1] floats, both over the V-row area
  float* accs = reinterpret_cast<float*>(smc_raw);
  float* bvs = accs + G * r;
  for (int e = tid; e < G * r; e += 256) {
    const int g = e / r, o = e % r;
    const float* pa_k = part_acc + ((static_cast<int64_t>(s) * Hq + hq0 + g) * nsplit) * r + o;
    float a = 0.f;
    for (int k0 = 0; k0 < nsp_used; k0 += 16) {  // sixteen loads in flight, then the sums in split order
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) x[i] = k0 + i < nsp_used ? __ldcg(pa_k + static_cast<int64_t>(k0 + i) * r) : 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (k0 + i < nsp_used) a = fmaf(alpha[g * nsplit + k0 + i], x[i], a);
    }
    accs[e] = a;
  }
  {
    const uint4* bv4 = reinterpret_cast<const uint4*>(basis + (static_cast<int64_t>(h) * 2 + 1) * D * r);  // B_V [D][r]
    const int nbv = D * r / V;
    uint4 bvr[NBV];
#pragma unroll
    for (int u = 0; u < NBV; ++u)
      if (tid + u * 256 < nbv) bvr[u] = __ldg(bv4 + tid + u * 256);
#pragma unroll
    for (int u = 0; u < NBV; ++u) {
      const int e = tid + u * 256;
      if (e < nbv) {
        float x[V];
        unpack16(bvr[u], x, static_cast<T*>(nullptr));
        const int k = (e * V) / r, o0 = (e * V) % r;
#pragma unroll
        for (int qq = 0; qq < V; ++qq) bvs[k * (r + 1) + o0 + qq] = x[qq];
      }
    }
  }
  __syncthreads();
  const float* mv = mu + (static_cast<int64_t>(h) * 2 + 1) * D;
  const float* cps = cpart + (static_cast<int64_t>(s) * H + h) * nchunk * G * D;
  for (int e = tid; e < G * D; e += 256) {
    const int g = e / D, k = e % D;
    float a = 0.f;
    for (int c0 = 0; c0 < nneed; c0 += 16) {  // sixteen loads in flight, then the sums in chunk order
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) x[i] = c0 + i < nneed ? __ldcg(cps + static_cast<int64_t>(c0 + i) * G * D + g * D + k) : 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) a += x[i];
    }
    for (int o = 0; o < r; ++o) a = fmaf(accs[g * r + o], bvs[k * (r + 1) + o], a);
    const float L = Ls[g];
    const float o_val = L > 0.f ? __ldg(mv + k) + a / L : 0.f;
    out[(static_cast<int64_t>(s) * Hq + hq0 + g) * D + k] = Elem<T>::from_f(o_val);
  }
  if (lse != nullptr && tid < G) {
    const float L = Ls[tid];
    lse[static_cast<int64_t>(s) * Hq + hq0 + tid] = L > 0.f ? (Ms[tid] + log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
}

// ------------------------------------------------------------------------------------------------
// Host side.
// ------------------------------------------------------------------------------------------------
template <typename T, int RK, int G>
static dkv_status launch_split(const DecodeArgs& a, const DecodeWs& L, uint8_t* ws, cudaStream_t st) {
  const dkv_shape& sh = *a.shape;
  const size_t smem = split_smem_bytes<T, RK, G>(L.max_ref);
  if (smem > 226 * 1024) return DKV_ERR_UNSUPPORTED;  // 227 KB opt-in minus static shared memory
  constexpr auto kDense = decode_split_kernel<T, RK, G, false>;
  constexpr auto kSparse = decode_split_kernel<T, RK, G, true>;
  const bool sparse = a.cu_sel != nullptr;
  if (!(sparse ? ensure_max_dynamic_smem<kSparse>() : ensure_max_dynamic_smem<kDense>())) return DKV_ERR_CUDA;
  dim3 grid(L.nsplit, sh.num_kv_heads, a.num_seqs);
  prof_begin(DKV_KERNEL_DECODE_SPLIT, st);
  (sparse ? kSparse : kDense)<<<grid, kDecThreads, smem, st>>>(
      static_cast<const T*>(a.cache->codes), a.cache->ref_idx, a.context_lens, a.block_tables, a.max_blocks,
      a.cache->num_blocks, sh.num_q_heads, sh.num_kv_heads, sh.ref_stride, a.max_ctx, L.max_ref, L.tps, L.nsplit,
      reinterpret_cast<const float*>(ws + L.qp), reinterpret_cast<const float*>(ws + L.qmu),
      reinterpret_cast<const float*>(ws + L.sref), reinterpret_cast<float*>(ws + L.ml),
      reinterpret_cast<float*>(ws + L.acc), reinterpret_cast<float*>(ws + L.bins), a.sel, a.cu_sel, a.max_sel);
  prof_end(DKV_KERNEL_DECODE_SPLIT, st);
  return DKV_OK;
}

template <typename T, int D, int G>
static dkv_status launch_combine(const DecodeArgs& a, const DecodeWs& L, uint8_t* ws, cudaStream_t st) {
  const dkv_shape& sh = *a.shape;
  const size_t smem = static_cast<size_t>(combine_vrow_bytes<T, D, G>(sh.rank)) +
                      (static_cast<size_t>(G) * L.nsplit + 2 * G + 2 * kCombineRefs * G) * 4 + 16 +
                      (sizeof(T) == 2 ? kCombineRefs / 16 * 32 * 16 : 0);
  if (smem > 226 * 1024) return DKV_ERR_UNSUPPORTED;  // 227 KB opt-in minus static shared memory
  if (!ensure_max_dynamic_smem<decode_combine_kernel<T, D, G>>()) return DKV_ERR_CUDA;
  dim3 grid(L.nchunk, sh.num_kv_heads, a.num_seqs);
  prof_begin(DKV_KERNEL_DECODE_COMBINE, st);
  // programmatic: its V-row copies overlap the split kernel's last items (it waits before reading partials)
  const cudaError_t e = launch_programmatic(
      decode_combine_kernel<T, D, G>, grid, dim3(256), smem, st, static_cast<const T*>(a.cache->refs),
      static_cast<const T*>(a.params->basis), a.params->mu, a.context_lens, a.block_tables, a.max_blocks,
      a.cache->num_blocks, sh.num_q_heads, sh.num_kv_heads, sh.rank, sh.ref_stride, a.max_ctx, L.max_ref, L.tps,
      L.nsplit, L.nchunk, reinterpret_cast<const float*>(ws + L.ml), reinterpret_cast<const float*>(ws + L.acc),
      reinterpret_cast<const float*>(ws + L.bins), reinterpret_cast<float*>(ws + L.cpart),
      reinterpret_cast<int*>(ws + L.cnt), static_cast<T*>(a.out), a.lse, a.cu_sel, a.max_sel);
  prof_end(DKV_KERNEL_DECODE_COMBINE, st);
  return e == cudaSuccess ? DKV_OK : DKV_ERR_CUDA;
}

template <int RK, int G, int STG, bool Q4, int KT, bool GB = false>
static dkv_status launch_split_mma_stg(const DecodeArgs& a, const DecodeWs& L, uint8_t* ws, cudaStream_t st,
                                       const MmaSplitShape& ms) {
  const dkv_shape& sh = *a.shape;
  // 4-bit codes, k-nearest slots and global masses are decoded densely; the sparse instantiation of those
  // configurations is never launched
  constexpr bool kCanSparse = !Q4 && KT == 1 && !GB;
  constexpr auto kDense = decode_split_mma_kernel<RK, G, false, STG, Q4, KT, GB>;
  constexpr auto kSparse = decode_split_mma_kernel<RK, G, kCanSparse, STG, Q4, KT, GB>;
  const bool sparse = kCanSparse && a.cu_sel != nullptr;
  if (!(sparse ? ensure_max_dynamic_smem<kSparse, true>() : ensure_max_dynamic_smem<kDense, true>()))
    return DKV_ERR_CUDA;
  CUtensorMap codes_map = {};  // codes as [num_blocks * H_kv * R rows][2r columns], boxes of R rows x 64 columns
  if (!Q4 && !make_map_bf16(&codes_map, a.cache->codes, 2 * RK,
                            static_cast<uint64_t>(a.cache->num_blocks) * sh.num_kv_heads * sh.ref_stride,
                            sh.ref_stride))
    return DKV_ERR_CUDA;
  // persistent: one or two CTAs per SM (the stage ring and the mass bins fill the shared memory), items
  // round-robin
  const int64_t n_items = static_cast<int64_t>(L.nsplit) * sh.num_kv_heads * a.num_seqs;
  if (n_items > INT32_MAX) return DKV_ERR_UNSUPPORTED;
  const int slots = num_sms() * ms.ctas_per_sm;
  const int grid = static_cast<int>(n_items < slots ? n_items : slots);
  prof_begin(DKV_KERNEL_DECODE_SPLIT, st);
  const cudaError_t e = launch_programmatic(
      sparse ? kSparse : kDense, dim3(grid), dim3(kMmaThreads), ms.smem, st, codes_map,
      static_cast<const int*>(a.cache->ref_idx), a.context_lens, a.block_tables, a.max_blocks, a.cache->num_blocks,
      a.num_seqs, sh.num_q_heads, sh.num_kv_heads, sh.ref_stride, a.max_ctx, L.max_ref, L.tps, L.nsplit, ms.stages,
      reinterpret_cast<const float*>(ws + L.qp), reinterpret_cast<const float*>(ws + L.qmu),
      reinterpret_cast<const float*>(ws + L.sref), reinterpret_cast<float*>(ws + L.ml),
      reinterpret_cast<float*>(ws + L.acc), reinterpret_cast<float*>(ws + L.bins),
      static_cast<const __nv_bfloat16*>(a.cache->codes), a.sel, a.cu_sel, a.max_sel);
  prof_end(DKV_KERNEL_DECODE_SPLIT, st);
  return e == cudaSuccess ? DKV_OK : DKV_ERR_CUDA;
}

template <int RK, int G, bool Q4 = false, int KT = 1>
static dkv_status launch_split_mma(const DecodeArgs& a, const DecodeWs& L, uint8_t* ws, cudaStream_t st) {
  const MmaSplitShape ms = split_mma_shape<RK, G, Q4, KT>(L.max_ref);
  // Dense bf16 keeps the per-reference masses in global memory when shared memory holds them beside fewer
  // than kGbinsBelowStages stages (or none): the freed shared memory deepens the ring to four stages.  On the
  // 64-sequence serving mix (7664 references, two stages otherwise) the split kernel takes 1.09 instead of
  // 1.21 ms.
  if constexpr (!Q4 && KT == 1) {
    if (a.cu_sel == nullptr && ms.ctas_per_sm == 1 && ms.stages < kGbinsBelowStages) {
      const MmaSplitShape mg = split_mma_shape_gb<RK, G>();
      if (mg.stages > ms.stages) return launch_split_mma_stg<RK, G, 256, false, 1, true>(a, L, ws, st, mg);
    }
  }
  if (ms.stages < 2) return DKV_ERR_UNSUPPORTED;  // per-reference mass does not fit beside two stages
  if constexpr (kTwoCtaSplit<RK, G> && KT == 1)
    if (ms.stg == 128) return launch_split_mma_stg<RK, G, 128, Q4, KT>(a, L, ws, st, ms);
  return launch_split_mma_stg<RK, G, 256, Q4, KT>(a, L, ws, st, ms);
}

template <typename T, int G>
static dkv_status dispatch_rank(const DecodeArgs& a, const DecodeWs& L, uint8_t* ws, cudaStream_t st) {
  constexpr bool kMma = sizeof(T) == 2;  // bf16: tensor-core split kernel for r in {32, 64}
  if (a.topk > 1) {  // k-nearest slots: tensor-core split kernel, tokens as the MMA rows (G >= 4), bf16
    if constexpr (kMma && G >= 4) {
      if (!is_q4(*a.shape)) {
        const bool r32 = a.shape->rank == 32, r64 = a.shape->rank == 64 && G == 4;
        if (a.topk == 2 && r32) return launch_split_mma<32, G, false, 2>(a, L, ws, st);
        if (a.topk == 4 && r32) return launch_split_mma<32, G, false, 4>(a, L, ws, st);
        if (a.topk == 2 && r64) return launch_split_mma<64, G, false, 2>(a, L, ws, st);
        if (a.topk == 4 && r64) return launch_split_mma<64, G, false, 4>(a, L, ws, st);
      }
    }
    return DKV_ERR_UNSUPPORTED;
  }
  if (is_q4(*a.shape)) {  // 4-bit codes: tensor-core split kernel, tokens as the MMA rows (G >= 4)
    if constexpr (kMma && G >= 4) {
      if (a.shape->rank == 32) return launch_split_mma<32, G, true>(a, L, ws, st);
      if (a.shape->rank == 64 && G == 4) return launch_split_mma<64, G, true>(a, L, ws, st);
    }
    return DKV_ERR_UNSUPPORTED;
  }
  switch (a.shape->rank) {
    case 16: return launch_split<T, 16, G>(a, L, ws, st);
    case 32:
      if constexpr (kMma) return launch_split_mma<32, G>(a, L, ws, st);
      return launch_split<T, 32, G>(a, L, ws, st);
    case 64:
      if constexpr (kMma) return launch_split_mma<64, G>(a, L, ws, st);
      if constexpr (G <= 4) return launch_split<T, 64, G>(a, L, ws, st);
      break;
    case 128:
      if constexpr (G <= 2 && sizeof(T) == 2) return launch_split<T, 128, G>(a, L, ws, st);
      break;
  }
  return DKV_ERR_UNSUPPORTED;
}

// Split CTAs that share an SM for this shape and context bound (the split plan counts slots of the device).
static int split_ctas_per_sm(const dkv_shape& sh, int max_ref, int topk) {
  if (topk > 1) return 1;  // k-nearest slots: one CTA per SM (wider stages)
  if ((sh.dtype != DKV_BF16 && sh.dtype != DKV_BF16_Q4) || (sh.rank != 32 && sh.rank != 64)) return 1;
  const int G = sh.num_q_heads / sh.num_kv_heads;
  const bool r32 = sh.rank == 32;
  if (is_q4(sh)) return r32 && G == 4 ? split_mma_shape<32, 4, true>(max_ref).ctas_per_sm : 1;
  switch (G) {
    case 1: return (r32 ? split_mma_shape<32, 1>(max_ref) : split_mma_shape<64, 1>(max_ref)).ctas_per_sm;
    case 2: return (r32 ? split_mma_shape<32, 2>(max_ref) : split_mma_shape<64, 2>(max_ref)).ctas_per_sm;
    case 4: return (r32 ? split_mma_shape<32, 4>(max_ref) : split_mma_shape<64, 4>(max_ref)).ctas_per_sm;
    case 8: return r32 ? split_mma_shape<32, 8>(max_ref).ctas_per_sm : 1;
  }
  return 1;
}

DecodeWs decode_layout(const dkv_shape& sh, int num_seqs, int max_ctx, int max_sel, int topk) {
  const int max_ref = std::max(1, max_refs(max_ctx, sh.ref_stride));
  return decode_ws_layout(sh, num_seqs, max_ctx, max_sel, split_ctas_per_sm(sh, max_ref, topk));
}

// Whether the split and combine kernels' shared memory holds this shape and context bound, with the same
// sizes their launches use: the split keeps a mass per visible reference and query head beside its stage
// ring, the combine a weight per split.  Decided before anything is launched.
template <typename T, int D, int G>
static dkv_status decode_fits_g(const dkv_shape& sh, int num_seqs, int max_ctx, int max_sel, int topk) {
  const DecodeWs L = decode_layout(sh, num_seqs, max_ctx, max_sel, topk);
  constexpr size_t kLimit = 226 * 1024;  // 227 KB opt-in minus static shared memory
  constexpr bool kMma = sizeof(T) == 2;
  bool split_ok = false;
  if (topk > 1) {
    if constexpr (kMma && G >= 4) {
      if (!is_q4(sh) && sh.rank == 32)
        split_ok = (topk == 2 ? split_mma_shape<32, G, false, 2>(L.max_ref).stages
                              : split_mma_shape<32, G, false, 4>(L.max_ref).stages) >= 2;
      if (!is_q4(sh) && sh.rank == 64 && G == 4)
        split_ok = (topk == 2 ? split_mma_shape<64, G, false, 2>(L.max_ref).stages
                              : split_mma_shape<64, G, false, 4>(L.max_ref).stages) >= 2;
    }
  } else if (is_q4(sh)) {
    if constexpr (kMma && G >= 4) {
      if (sh.rank == 32) split_ok = split_mma_shape<32, G, true>(L.max_ref).stages >= 2;
      if (sh.rank == 64 && G == 4) split_ok = split_mma_shape<64, G, true>(L.max_ref).stages >= 2;
    }
  } else switch (sh.rank) {
    case 16: split_ok = split_smem_bytes<T, 16, G>(L.max_ref) <= kLimit; break;
    case 32:
      if constexpr (kMma)
        split_ok = split_mma_shape<32, G>(L.max_ref).stages >= 2 ||
                   (max_sel < 0 && split_mma_shape_gb<32, G>().stages >= 2);
      else split_ok = split_smem_bytes<T, 32, G>(L.max_ref) <= kLimit;
      break;
    case 64:
      if constexpr (kMma)
        split_ok = split_mma_shape<64, G>(L.max_ref).stages >= 2 ||
                   (max_sel < 0 && split_mma_shape_gb<64, G>().stages >= 2);
      else if constexpr (G <= 4) split_ok = split_smem_bytes<T, 64, G>(L.max_ref) <= kLimit;
      break;
  }
  if (!split_ok) return DKV_ERR_UNSUPPORTED;
  const size_t combine = static_cast<size_t>(combine_vrow_bytes<T, D, G>(sh.rank)) +
                         (static_cast<size_t>(G) * L.nsplit + 2 * G + 2 * kCombineRefs * G) * 4 + 16 +
                         (sizeof(T) == 2 ? kCombineRefs / 16 * 32 * 16 : 0);
  return combine <= kLimit ? DKV_OK : DKV_ERR_UNSUPPORTED;
}

template <typename T, int D>
static dkv_status decode_fits_d(const dkv_shape& sh, int num_seqs, int max_ctx, int max_sel, int topk) {
  switch (sh.num_q_heads / sh.num_kv_heads) {
    case 1: return decode_fits_g<T, D, 1>(sh, num_seqs, max_ctx, max_sel, topk);
    case 2: return decode_fits_g<T, D, 2>(sh, num_seqs, max_ctx, max_sel, topk);
    case 4: return decode_fits_g<T, D, 4>(sh, num_seqs, max_ctx, max_sel, topk);
    case 8: return decode_fits_g<T, D, 8>(sh, num_seqs, max_ctx, max_sel, topk);
  }
  return DKV_ERR_UNSUPPORTED;
}

dkv_status decode_supported(const dkv_shape& sh, int num_seqs, int max_ctx, int max_sel, int topk) {
  if (sh.dtype == DKV_F32)
    return sh.head_dim == 64 ? decode_fits_d<float, 64>(sh, num_seqs, max_ctx, max_sel, topk)
                             : decode_fits_d<float, 128>(sh, num_seqs, max_ctx, max_sel, topk);
  return sh.head_dim == 64 ? decode_fits_d<__nv_bfloat16, 64>(sh, num_seqs, max_ctx, max_sel, topk)
                           : decode_fits_d<__nv_bfloat16, 128>(sh, num_seqs, max_ctx, max_sel, topk);
}

template <typename T, int D, int G>
static dkv_status launch_decode_g(const DecodeArgs& a, uint8_t* ws, cudaStream_t st) {
  const dkv_shape& sh = *a.shape;
  const DecodeWs L = decode_layout(sh, a.num_seqs, a.max_ctx, a.cu_sel != nullptr ? a.max_sel : -1, a.topk);
  const float scale = a.softmax_scale > 0.f ? a.softmax_scale : 1.0f / sqrtf(static_cast<float>(D));
  const float scale2 = scale * 1.4426950408889634f;
  if (cudaMemsetAsync(ws + L.cnt, 0, static_cast<size_t>(a.num_seqs) * sh.num_kv_heads * 4, st) != cudaSuccess)
    return DKV_ERR_CUDA;
  if constexpr (sizeof(T) == 2) {
    // S * H_kv CTAs for q B_K and q . mu_K (short: they leave within microseconds), then as many tile CTAs
    // as the SMs hold at once, looping over the tile tasks
    constexpr auto kPro = decode_prologue_tc_kernel<D, G>;
    const size_t smem = static_cast<size_t>(G * D + D * sh.rank) * 2 + D * 4;
    const int64_t units = static_cast<int64_t>(a.num_seqs) * sh.num_kv_heads;
    const int64_t tasks = units * ceil_div64(L.max_ref, 16 * kProTaskTiles);
    int64_t tile_ctas = static_cast<int64_t>(num_sms()) * resident_ctas<kPro>(kProThreads, smem);
    const int64_t need = ceil_div64(tasks, kProThreads / 32);
    if (tile_ctas > need) tile_ctas = need;
    if (units + tile_ctas > INT32_MAX) return DKV_ERR_UNSUPPORTED;
    prof_begin(DKV_KERNEL_DECODE_PROLOGUE, st);
    kPro<<<static_cast<unsigned>(units + tile_ctas), kProThreads, smem, st>>>(
        static_cast<const __nv_bfloat16*>(a.q), a.params->mu, static_cast<const __nv_bfloat16*>(a.params->basis),
        static_cast<const __nv_bfloat16*>(a.cache->refs), a.context_lens, a.block_tables, a.max_blocks,
        a.cache->num_blocks, a.num_seqs, sh.num_q_heads, sh.num_kv_heads, sh.rank, sh.ref_stride, a.max_ctx,
        L.max_ref, scale2, reinterpret_cast<float*>(ws + L.qp),
        reinterpret_cast<float*>(ws + L.qmu), reinterpret_cast<float*>(ws + L.sref));
    prof_end(DKV_KERNEL_DECODE_PROLOGUE, st);
  } else {
    dim3 grid(static_cast<unsigned>(ceil_div64(L.max_ref, kProRefs)), sh.num_kv_heads, a.num_seqs);
    // queries, B_K and mu_K (fp32)
    const size_t smem = static_cast<size_t>(G * D + D * sh.rank + D) * 4;
    if (!ensure_max_dynamic_smem<decode_prologue_kernel<T, D, G>>()) return DKV_ERR_CUDA;
    prof_begin(DKV_KERNEL_DECODE_PROLOGUE, st);
    decode_prologue_kernel<T, D, G><<<grid, kProRefs, smem, st>>>(
        static_cast<const T*>(a.q), a.params->mu, static_cast<const T*>(a.params->basis),
        static_cast<const T*>(a.cache->refs), a.context_lens, a.block_tables, a.max_blocks, a.cache->num_blocks,
        sh.num_q_heads, sh.num_kv_heads, sh.rank, sh.ref_stride, a.max_ctx, L.max_ref, scale2,
        reinterpret_cast<float*>(ws + L.qp), reinterpret_cast<float*>(ws + L.qmu),
        reinterpret_cast<float*>(ws + L.sref));
    prof_end(DKV_KERNEL_DECODE_PROLOGUE, st);
  }
  dkv_status s = dispatch_rank<T, G>(a, L, ws, st);
  if (s != DKV_OK) return s;
  return launch_combine<T, D, G>(a, L, ws, st);
}

template <typename T, int D>
static dkv_status launch_decode_d(const DecodeArgs& a, uint8_t* ws, cudaStream_t st) {
  switch (a.shape->num_q_heads / a.shape->num_kv_heads) {
    case 1: return launch_decode_g<T, D, 1>(a, ws, st);
    case 2: return launch_decode_g<T, D, 2>(a, ws, st);
    case 4: return launch_decode_g<T, D, 4>(a, ws, st);
    case 8: return launch_decode_g<T, D, 8>(a, ws, st);
  }
  return DKV_ERR_UNSUPPORTED;
}

template <typename T>
static dkv_status launch_decode_t(const DecodeArgs& a, uint8_t* ws, cudaStream_t st) {
  return a.shape->head_dim == 64 ? launch_decode_d<T, 64>(a, ws, st) : launch_decode_d<T, 128>(a, ws, st);
}

dkv_status launch_decode(const DecodeArgs& a, void* workspace, cudaStream_t st) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const dkv_status s = a.shape->dtype == DKV_F32 ? launch_decode_t<float>(a, ws, st)
                                                 : launch_decode_t<__nv_bfloat16>(a, ws, st);
  if (s != DKV_OK) return s;
  return cudaGetLastError() == cudaSuccess ? DKV_OK : DKV_ERR_CUDA;
}

}  // namespace dkv
