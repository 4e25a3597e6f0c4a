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
//                           exceeds it by more than 2^8 (then acc, l and the mass bins are rescaled), and
//                           p, l, acc = sum p cV and bins[j] += p are accumulated.
//   decode_combine_kernel   merges the splits (max / sum-exp), forms sum_j w_j r~V_j per chunk of
//                           references; the last chunk CTA of a (seq, kv head) adds acc B_V^T and mu,
//                           divides by the softmax mass and writes out and lse.
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
// Prologue.  CTA = (64 references, kv head, sequence), 256 threads.
// ------------------------------------------------------------------------------------------------
constexpr int kProRefs = 64;

template <typename T>
__global__ void __launch_bounds__(256) decode_prologue_kernel(
    const T* __restrict__ q, const float* __restrict__ mu, const T* __restrict__ basis, const T* __restrict__ refs,
    const int* __restrict__ context_lens, const int* __restrict__ block_tables, int max_blocks, int num_blocks,
    int Hq, int H, int d, int r, int R, int max_ctx, int max_ref, float scale2, float* __restrict__ qp,
    float* __restrict__ qmu, float* __restrict__ sref) {
  extern __shared__ float qs[];  // [G][d]
  const int s = blockIdx.z, h = blockIdx.y, j0 = blockIdx.x * kProRefs;
  const int G = Hq / H, tid = threadIdx.x;
  const int ctx = checked_ctx(context_lens, s, max_ctx);
  const int n_ref = ceil_div_d(ctx, R);
  if (blockIdx.x != 0 && j0 >= n_ref) return;
  for (int e = tid; e < G * d; e += blockDim.x)
    qs[e] = Elem<T>::to_f(q[(static_cast<int64_t>(s) * Hq + h * G) * d + e]);
  __syncthreads();
  if (blockIdx.x == 0) {
    const T* bk = basis + static_cast<int64_t>(h) * 2 * d * r;  // B_K [d][r]
    for (int e = tid; e < G * r; e += blockDim.x) {
      const int g = e / r, o = e % r;
      float a = 0.f;
      for (int k = 0; k < d; ++k) a = fmaf(qs[g * d + k], Elem<T>::to_f(bk[k * r + o]), a);
      qp[(static_cast<int64_t>(s) * Hq + h * G + g) * r + o] = a * scale2;
    }
    const float* mk = mu + static_cast<int64_t>(h) * 2 * d;
    if (tid < G) {
      float a = 0.f;
      for (int k = 0; k < d; ++k) a = fmaf(qs[tid * d + k], mk[k], a);
      qmu[static_cast<int64_t>(s) * Hq + h * G + tid] = a * scale2;
    }
  }
  // q . r~K_j: 4 threads per reference, each a quarter of d
  const int jj = tid >> 2, sub = tid & 3;
  const int j = j0 + jj;
  const bool ok = j < n_ref;
  float part[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) part[g] = 0.f;
  if (ok) {
    const int pb = checked_block(block_tables, max_blocks, num_blocks, s, j);
    const T* row = refs + (static_cast<int64_t>(pb) * H + h) * 2 * d + sub * (d / 4);
    for (int k0 = 0; k0 < d / 4; k0 += 16 / static_cast<int>(sizeof(T))) {
      constexpr int NV = 16 / sizeof(T);
      float x[NV];
      load_elems<T, NV>(row + k0, x);
#pragma unroll
      for (int g = 0; g < 8; ++g)
        if (g < G) {
#pragma unroll
          for (int e = 0; e < NV; ++e) part[g] = fmaf(x[e], qs[g * d + sub * (d / 4) + k0 + e], part[g]);
        }
    }
  }
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    part[g] += __shfl_xor_sync(0xffffffffu, part[g], 1);
    part[g] += __shfl_xor_sync(0xffffffffu, part[g], 2);
  }
  if (ok && sub == 0) {
    float* dst = sref + ((static_cast<int64_t>(s) * H + h) * max_ref + j) * G;
    for (int g = 0; g < G; ++g) dst[g] = part[g] * scale2;
  }
}

// ------------------------------------------------------------------------------------------------
// Split-K main kernel.
// ------------------------------------------------------------------------------------------------
constexpr int kDecNCW = 8;                // consumer warps
constexpr int kDecThreads = (kDecNCW + 1) * 32;
constexpr int kDecStages = 4;
constexpr float kRescaleLog2 = 8.0f;      // raise the running max only when a stage exceeds it by 2^8

template <typename T, int RK>
struct SplitCfg {
  static constexpr int ES = sizeof(T);
  static constexpr int STG_RAW = 16384 / (2 * RK * ES);
  static constexpr int STG = STG_RAW < 64 ? 64 : (STG_RAW > 256 ? 256 : STG_RAW);  // tokens per stage
  static constexpr int NGRP = STG / (kDecNCW * 8);  // 8-token groups per warp per stage
  static constexpr int DPL = RK / 4;                 // code dims per lane
  static constexpr int CODE_BYTES = STG * 2 * RK * ES;
  static constexpr int IDX_BYTES = STG * 4;
  static constexpr int STAGE_BYTES = CODE_BYTES + IDX_BYTES;
  static constexpr int HDR_BYTES = 128;  // barriers + abort flag
};

template <typename T, int RK, int G>
size_t split_smem_bytes(int jcap_max) {
  using C = SplitCfg<T, RK>;
  return C::HDR_BYTES + static_cast<size_t>(kDecStages) * C::STAGE_BYTES +
         static_cast<size_t>(jcap_max) * G * 4 + 2 * kDecNCW * G * 4 + kDecNCW * G * RK * 4 + kDecNCW * G * 4;
}

template <typename T, int RK, int G>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(
    const T* __restrict__ codes, const int* __restrict__ ref_idx, const int* __restrict__ context_lens,
    const int* __restrict__ block_tables, int max_blocks, int num_blocks, int Hq, int H, int R, int max_ctx,
    int max_ref, int tps, int nsplit, const float* __restrict__ qp, const float* __restrict__ qmu,
    const float* __restrict__ sref, float* __restrict__ part_ml, float* __restrict__ part_acc,
    float* __restrict__ part_bins) {
  using C = SplitCfg<T, RK>;
  constexpr int STG = C::STG, NGRP = C::NGRP, DPL = C::DPL;
  extern __shared__ __align__(128) uint8_t sm_split[];
  uint64_t* full = reinterpret_cast<uint64_t*>(sm_split);
  uint64_t* empty = full + kDecStages;
  volatile int* sAbort = reinterpret_cast<volatile int*>(empty + kDecStages);
  uint8_t* stages = sm_split + C::HDR_BYTES;
  float* bins = reinterpret_cast<float*>(stages + kDecStages * C::STAGE_BYTES);

  const int split = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const int ctx = checked_ctx(context_lens, s, max_ctx);
  const int t_begin = split * tps;
  const int t_end = min(ctx, t_begin + tps);
  const int hq0 = h * G;
  const int64_t ml_base = (static_cast<int64_t>(s) * Hq + hq0) * nsplit + split;  // + g * nsplit

  if (t_begin >= t_end) {  // empty split: neutral partials
    if (tid < G) {
      part_ml[(ml_base + tid * nsplit) * 2] = -INFINITY;
      part_ml[(ml_base + tid * nsplit) * 2 + 1] = 0.f;
    }
    for (int e = tid; e < G * RK; e += blockDim.x)
      part_acc[(ml_base + (e / RK) * nsplit) * RK + e % RK] = 0.f;
    return;
  }
  const int n_ref = ceil_div_d(ctx, R);
  const int jcap = ceil_div_d(t_end, R);
  float* wmax = bins + static_cast<size_t>(jcap) * G;  // [2][NCW][G]
  float* red = wmax + 2 * kDecNCW * G;                 // [NCW][G][RK]
  float* lred = red + kDecNCW * G * RK;                // [NCW][G]

  if (tid == 0) {
    for (int i = 0; i < kDecStages; ++i) {
      mbar_init(smem_u32(full + i), 1);
      mbar_init(smem_u32(empty + i), kDecNCW);
    }
    *sAbort = 0;
    fence_barrier_init();
  }
  for (int e = tid; e < jcap * G; e += blockDim.x) bins[e] = 0.f;
  __syncthreads();

  const int nst = ceil_div_d(t_end - t_begin, STG);
  const int blk0 = t_begin / R;
  const int nblk = ceil_div_d(t_end, R);
  constexpr int BPS_MAX = 256 / 16;
  const int BPS = STG / R;
  const uint32_t blk_code_bytes = static_cast<uint32_t>(R) * 2 * RK * sizeof(T);
  const uint32_t blk_idx_bytes = static_cast<uint32_t>(R) * 4;

  if (warp == kDecNCW) {
    // ---------------- producer: whole paged blocks by bulk copy ----------------
    for (int st = 0; st < nst; ++st) {
      const int slot = st % kDecStages;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(smem_u32(empty + slot), ((st / kDecStages) & 1) ^ 1, sAbort);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const int lb = blk0 + st * BPS + lane;
      const bool valid = lane < BPS && lane < BPS_MAX && lb < nblk;
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
  const float* sref_sh = sref + (static_cast<int64_t>(s) * H + h) * max_ref * G;
  bool aborted = false;

  for (int st = 0; st < nst; ++st) {
    const int slot = st % kDecStages;
    // On a timeout the wait raises the shared abort flag; the stage is then processed from stale shared
    // memory (indices are range-checked) and every consumer leaves together after the next CTA barrier.
    mbar_wait(smem_u32(full + slot), (st / kDecStages) & 1, sAbort);
    const T* sc = reinterpret_cast<const T*>(stages + slot * C::STAGE_BYTES);
    const int* si = reinterpret_cast<const int*>(stages + slot * C::STAGE_BYTES + C::CODE_BYTES);
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
      if (vl[grp] && (idx < 0 || idx >= jcap)) {
        record_error(DKV_DEVERR_REF_IDX);
        idx = 0;
      }
      ix[grp] = idx;
      float kk[DPL];
      load_elems<T, DPL>(sc + tok * 2 * RK + sub * DPL, kk);
      float part[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) a = fmaf(qv[g][i], kk[i], a);
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        part[g] = a;
      }
      const float* sr = sref_sh + static_cast<int64_t>(idx) * G;
#pragma unroll
      for (int g = 0; g < G; ++g) s2[grp][g] = vl[grp] ? qm[g] + __ldg(sr + g) + part[g] : -INFINITY;
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
    named_bar_sync(1, kDecNCW * 32);
    if (*sAbort) {
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
        for (int e = tid; e < jcap * G; e += kDecNCW * 32) bins[e] *= alpha[e % G];
        named_bar_sync(1, kDecNCW * 32);
      }
    }
#pragma unroll
    for (int grp = 0; grp < NGRP; ++grp) {
      const int tok = cw * (STG / kDecNCW) + grp * 8 + tig;
      float vv[DPL];
      load_elems<T, DPL>(sc + tok * 2 * RK + RK + sub * DPL, vv);
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
          if (vl[grp]) atomicAdd(bins + ix[grp] * G + g, p[g]);
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(empty + slot));
  }
  named_bar_sync(1, kDecNCW * 32);  // all mass adds done
  if (aborted) return;

  float* gb = part_bins + ((static_cast<int64_t>(s) * H + h) * nsplit + split) * static_cast<int64_t>(max_ref) * G;
  for (int e = tid; e < jcap * G; e += kDecNCW * 32) gb[e] = bins[e];
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
  (void)n_ref;
}

// ------------------------------------------------------------------------------------------------
// Combine.  CTA = (chunk of 256 references, kv head, sequence), 256 threads.
// ------------------------------------------------------------------------------------------------
constexpr int kCombSub = 64;  // reference rows staged at a time

template <typename T, int G>
__global__ void __launch_bounds__(256) decode_combine_kernel(
    const T* __restrict__ refs, const T* __restrict__ basis, const float* __restrict__ mu,
    const int* __restrict__ context_lens, const int* __restrict__ block_tables, int max_blocks, int num_blocks,
    int Hq, int H, int d, int r, int R, int max_ctx, int max_ref, int tps, int nsplit, int nchunk,
    const float* __restrict__ part_ml, const float* __restrict__ part_acc, const float* __restrict__ part_bins,
    float* __restrict__ cpart, int* __restrict__ counters, T* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ float smc[];
  float* alpha = smc;                         // [G][nsplit]
  float* Ls = alpha + G * nsplit;             // [G]
  float* Ms = Ls + G;                         // [G]
  float* w = Ms + G;                          // [256][G]
  float* vs = w + kCombineRefs * G;           // [kCombSub][d]
  __shared__ int s_last;

  const int c = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const int ctx = checked_ctx(context_lens, s, max_ctx);
  const int n_ref = ceil_div_d(ctx, R);
  const int nneed = n_ref > 0 ? ceil_div_d(n_ref, kCombineRefs) : 1;
  if (c >= nneed) return;
  const int hq0 = h * G;
  const int nsp_used = ctx > 0 ? ceil_div_d(ctx, tps) : 0;

  // split weights per query head: warp g reduces over splits
  for (int g = warp; g < G; g += 8) {
    const float* ml = part_ml + ((static_cast<int64_t>(s) * Hq + hq0 + g) * nsplit) * 2;
    float M = -INFINITY;
    for (int k = lane; k < nsp_used; k += 32) M = fmaxf(M, ml[2 * k]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int k = lane; k < nsplit; k += 32) {
      float a = 0.f;
      if (k < nsp_used && M != -INFINITY && ml[2 * k] != -INFINITY) a = exp2f(ml[2 * k] - M);
      alpha[g * nsplit + k] = a;
      if (k < nsp_used) L += a * ml[2 * k + 1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) {
      Ls[g] = L;
      Ms[g] = M;
    }
  }
  __syncthreads();

  // reference mass w_j = sum_k alpha_k bins_k[j] over the splits whose tokens can reach j
  const int jbase = c * kCombineRefs;
  {
    const int j = jbase + tid;
    float wv[G];
#pragma unroll
    for (int g = 0; g < G; ++g) wv[g] = 0.f;
    if (j < n_ref) {
      for (int k = 0; k < nsp_used; ++k) {
        const int jcap_k = ceil_div_d(min(ctx, (k + 1) * tps), R);
        if (j >= jcap_k) continue;
        const float* b = part_bins + ((static_cast<int64_t>(s) * H + h) * nsplit + k) * static_cast<int64_t>(max_ref) * G +
                         static_cast<int64_t>(j) * G;
#pragma unroll
        for (int g = 0; g < G; ++g) wv[g] = fmaf(alpha[g * nsplit + k], b[g], wv[g]);
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) w[tid * G + g] = wv[g];
  }

  // partial[g][dd] = sum_j w_j r~V_j[dd] over this chunk
  const int ngs = 256 / d;  // thread groups over heads
  const int dd = tid % d, gs = tid / d;
  float pa[G];
#pragma unroll
  for (int g = 0; g < G; ++g) pa[g] = 0.f;
  const int nj = min(kCombineRefs, n_ref - jbase);
  for (int j0 = 0; j0 < nj; j0 += kCombSub) {
    __syncthreads();
    const int rows = min(kCombSub, nj - j0);
    for (int e = tid; e < kCombSub * d; e += 256) {
      const int jj = e / d, k = e % d;
      float v = 0.f;
      if (jj < rows) {
        const int pb = checked_block(block_tables, max_blocks, num_blocks, s, jbase + j0 + jj);
        v = Elem<T>::to_f(refs[(static_cast<int64_t>(pb) * H + h) * 2 * d + d + k]);
      }
      vs[e] = v;
    }
    __syncthreads();
    for (int jj = 0; jj < rows; ++jj) {
      const float vv = vs[jj * d + dd];
#pragma unroll
      for (int g = 0; g < G; ++g)
        if (g % ngs == gs) pa[g] = fmaf(w[(j0 + jj) * G + g], vv, pa[g]);
    }
  }
  float* cp = cpart + ((static_cast<int64_t>(s) * H + h) * nchunk + c) * G * d;
#pragma unroll
  for (int g = 0; g < G; ++g)
    if (g % ngs == gs) cp[g * d + dd] = pa[g];

  // the last chunk CTA of this (seq, kv head) finishes
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(counters + static_cast<int64_t>(s) * H + h, 1);
    s_last = prev == nneed - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // acc_g = sum_k alpha_k acc_k (reuse w as [G][r])
  float* accs = w;
  for (int e = tid; e < G * r; e += 256) {
    const int g = e / r, o = e % r;
    const float* pa_k = part_acc + ((static_cast<int64_t>(s) * Hq + hq0 + g) * nsplit) * r + o;
    float a = 0.f;
    for (int k = 0; k < nsp_used; ++k) a = fmaf(alpha[g * nsplit + k], __ldcg(pa_k + static_cast<int64_t>(k) * r), a);
    accs[e] = a;
  }
  __syncthreads();
  const T* bv = basis + (static_cast<int64_t>(h) * 2 + 1) * d * r;  // B_V [d][r]
  const float* mv = mu + (static_cast<int64_t>(h) * 2 + 1) * d;
  const float* cps = cpart + (static_cast<int64_t>(s) * H + h) * nchunk * G * d;
  for (int e = tid; e < G * d; e += 256) {
    const int g = e / d, k = e % d;
    float a = 0.f;
    for (int cc = 0; cc < nneed; ++cc) a += __ldcg(cps + static_cast<int64_t>(cc) * G * d + g * d + k);
    for (int o = 0; o < r; ++o) a = fmaf(accs[g * r + o], Elem<T>::to_f(bv[k * r + o]), a);
    const float L = Ls[g];
    const float o_val = L > 0.f ? mv[k] + a / L : 0.f;
    out[(static_cast<int64_t>(s) * Hq + hq0 + g) * d + k] = Elem<T>::from_f(o_val);
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
  if (smem > 227 * 1024) return DKV_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(decode_split_kernel<T, RK, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return DKV_ERR_CUDA;
  dim3 grid(L.nsplit, sh.num_kv_heads, a.num_seqs);
  prof_begin(DKV_KERNEL_DECODE_SPLIT, st);
    decode_split_kernel<T, RK, G><<<grid, kDecThreads, smem, st>>>(
      static_cast<const T*>(a.cache->codes), a.cache->ref_idx, a.context_lens, a.block_tables, a.max_blocks,
      a.cache->num_blocks, sh.num_q_heads, sh.num_kv_heads, sh.ref_stride, a.max_ctx, L.max_ref, L.tps, L.nsplit,
      reinterpret_cast<const float*>(ws + L.qp), reinterpret_cast<const float*>(ws + L.qmu),
      reinterpret_cast<const float*>(ws + L.sref), reinterpret_cast<float*>(ws + L.ml),
      reinterpret_cast<float*>(ws + L.acc), reinterpret_cast<float*>(ws + L.bins));
    prof_end(DKV_KERNEL_DECODE_SPLIT, st);
  return DKV_OK;
}

template <typename T, int G>
static dkv_status launch_combine(const DecodeArgs& a, const DecodeWs& L, uint8_t* ws, cudaStream_t st) {
  const dkv_shape& sh = *a.shape;
  const int d = sh.head_dim;
  const size_t smem = (static_cast<size_t>(G) * L.nsplit + 2 * G + kCombineRefs * G + kCombSub * d) * 4;
  if (smem > 227 * 1024) return DKV_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(decode_combine_kernel<T, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return DKV_ERR_CUDA;
  dim3 grid(L.nchunk, sh.num_kv_heads, a.num_seqs);
  prof_begin(DKV_KERNEL_DECODE_COMBINE, st);
    decode_combine_kernel<T, G><<<grid, 256, smem, st>>>(
      static_cast<const T*>(a.cache->refs), static_cast<const T*>(a.params->basis), a.params->mu, a.context_lens,
      a.block_tables, a.max_blocks, a.cache->num_blocks, sh.num_q_heads, sh.num_kv_heads, d, sh.rank,
      sh.ref_stride, a.max_ctx, L.max_ref, L.tps, L.nsplit, L.nchunk, reinterpret_cast<const float*>(ws + L.ml),
      reinterpret_cast<const float*>(ws + L.acc), reinterpret_cast<const float*>(ws + L.bins),
      reinterpret_cast<float*>(ws + L.cpart), reinterpret_cast<int*>(ws + L.cnt), static_cast<T*>(a.out), a.lse);
    prof_end(DKV_KERNEL_DECODE_COMBINE, st);
  return DKV_OK;
}

template <typename T, int G>
static dkv_status dispatch_rank(const DecodeArgs& a, const DecodeWs& L, uint8_t* ws, cudaStream_t st) {
  switch (a.shape->rank) {
    case 16: return launch_split<T, 16, G>(a, L, ws, st);
    case 32: return launch_split<T, 32, G>(a, L, ws, st);
    case 64:
      if constexpr (G <= 4) return launch_split<T, 64, G>(a, L, ws, st);
      break;
    case 128:
      if constexpr (G <= 2 && sizeof(T) == 2) return launch_split<T, 128, G>(a, L, ws, st);
      break;
  }
  return DKV_ERR_UNSUPPORTED;
}

template <typename T, int G>
static dkv_status launch_decode_g(const DecodeArgs& a, uint8_t* ws, cudaStream_t st) {
  const dkv_shape& sh = *a.shape;
  const DecodeWs L = decode_ws_layout(sh, a.num_seqs, a.max_ctx);
  const float scale = a.softmax_scale > 0.f ? a.softmax_scale : 1.0f / sqrtf(static_cast<float>(sh.head_dim));
  const float scale2 = scale * 1.4426950408889634f;
  if (cudaMemsetAsync(ws + L.cnt, 0, static_cast<size_t>(a.num_seqs) * sh.num_kv_heads * 4, st) != cudaSuccess)
    return DKV_ERR_CUDA;
  {
    dim3 grid(static_cast<unsigned>(ceil_div64(L.max_ref, kProRefs)), sh.num_kv_heads, a.num_seqs);
    const size_t smem = static_cast<size_t>(G) * sh.head_dim * 4;
    prof_begin(DKV_KERNEL_DECODE_PROLOGUE, st);
    decode_prologue_kernel<T><<<grid, 256, smem, st>>>(
        static_cast<const T*>(a.q), a.params->mu, static_cast<const T*>(a.params->basis),
        static_cast<const T*>(a.cache->refs), a.context_lens, a.block_tables, a.max_blocks, a.cache->num_blocks,
        sh.num_q_heads, sh.num_kv_heads, sh.head_dim, sh.rank, sh.ref_stride, a.max_ctx, L.max_ref, scale2,
        reinterpret_cast<float*>(ws + L.qp), reinterpret_cast<float*>(ws + L.qmu),
        reinterpret_cast<float*>(ws + L.sref));
    prof_end(DKV_KERNEL_DECODE_PROLOGUE, st);
  }
  dkv_status s = dispatch_rank<T, G>(a, L, ws, st);
  if (s != DKV_OK) return s;
  return launch_combine<T, G>(a, L, ws, st);
}

template <typename T>
static dkv_status launch_decode_t(const DecodeArgs& a, uint8_t* ws, cudaStream_t st) {
  switch (a.shape->num_q_heads / a.shape->num_kv_heads) {
    case 1: return launch_decode_g<T, 1>(a, ws, st);
    case 2: return launch_decode_g<T, 2>(a, ws, st);
    case 4: return launch_decode_g<T, 4>(a, ws, st);
    case 8: return launch_decode_g<T, 8>(a, ws, st);
  }
  return DKV_ERR_UNSUPPORTED;
}

dkv_status launch_decode(const DecodeArgs& a, void* workspace, cudaStream_t st) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const dkv_status s = a.shape->dtype == DKV_F32 ? launch_decode_t<float>(a, ws, st)
                                                 : launch_decode_t<__nv_bfloat16>(a, ws, st);
  if (s != DKV_OK) return s;
  return cudaGetLastError() == cudaSuccess ? DKV_OK : DKV_ERR_CUDA;
}

}  // namespace dkv
