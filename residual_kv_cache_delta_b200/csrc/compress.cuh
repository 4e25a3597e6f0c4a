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
// 1. Centre the new tokens.  One thread per 16-byte vector of one (token, kv head, K|V) row.
// ------------------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) center_kernel(const T* __restrict__ k_new, const T* __restrict__ v_new,
                                                     const float* __restrict__ mu, const int* __restrict__ cu_new,
                                                     const int* __restrict__ start_pos,
                                                     const int* __restrict__ block_tables, int max_blocks,
                                                     int num_blocks, int H, int d, int R, int64_t total_new,
                                                     int max_new, int max_ctx, T* __restrict__ xt,
                                                     T* __restrict__ refs) {
  constexpr int V = V16<T>::N;
  const int s = blockIdx.y;
  const int cpr = d / V;
  const int per_tok = H * 2 * cpr;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int n_local = static_cast<int>(i / per_tok);
  if (n_local >= max_new) return;
  SeqRange sr;
  if (!load_seq(cu_new, start_pos, s, total_new, max_new, max_ctx, sr)) {
    if (i == 0) record_error(DKV_DEVERR_BOUNDS);
    return;
  }
  if (n_local >= sr.n_new) return;
  int rem = static_cast<int>(i % per_tok);
  const int h = rem / (2 * cpr);
  rem %= 2 * cpr;
  const int kv = rem / cpr, c = rem % cpr;
  const int64_t row = sr.base + n_local;
  const int pos = sr.start + n_local;
  float x[V], m[V];
  V16<T>::load((kv ? v_new : k_new) + (row * H + h) * d + c * V, x);
  const float* mp = mu + (h * 2 + kv) * d + c * V;
#pragma unroll
  for (int e = 0; e < V; ++e) m[e] = __ldg(mp + e);
#pragma unroll
  for (int e = 0; e < V; ++e) x[e] = __fsub_rn(x[e], m[e]);  // IEEE fp32 subtract; rounding to S in store
  V16<T>::store(xt + (static_cast<int64_t>(h) * total_new + row) * (2 * d) + kv * d + c * V, x);
  if (pos % R == 0) {
    const int pb = lookup_block(block_tables, max_blocks, num_blocks, s, pos / R);
    if (pb >= 0) V16<T>::store(refs + ((static_cast<int64_t>(pb) * H + h) * 2 + kv) * d + c * V, x);
  }
}

// ------------------------------------------------------------------------------------------------
// 2. Reference prep: contiguous copy, inverse norm and projection of every visible reference.
//    CTA = (32 references, kv head, sequence), 256 threads.
// ------------------------------------------------------------------------------------------------
constexpr int kPrepRefs = 32;

template <typename T>
__global__ void __launch_bounds__(256) refprep_kernel(const T* __restrict__ refs, const T* __restrict__ basis,
                                                      const int* __restrict__ cu_new,
                                                      const int* __restrict__ start_pos,
                                                      const int* __restrict__ block_tables, int max_blocks,
                                                      int num_blocks, int H, int d, int r, int R,
                                                      int64_t total_new, int max_new, int max_ctx,
                                                      int64_t max_ref_pad, T* __restrict__ refc,
                                                      float* __restrict__ invn, float* __restrict__ pr) {
  constexpr int V = V16<T>::N;
  extern __shared__ float sm_prep[];
  const int d2 = 2 * d, r2 = 2 * r;
  const int rs_stride = d2 + 1;
  float* rs = sm_prep;                               // [32][2d+1]
  float* bs = rs + kPrepRefs * rs_stride;       // [2][d][r]
  const int s = blockIdx.z, h = blockIdx.y, j0 = blockIdx.x * kPrepRefs;
  SeqRange sr;
  if (!load_seq(cu_new, start_pos, s, total_new, max_new, max_ctx, sr)) return;  // recorded by center_kernel
  const int n_ref = ceil_div_i(sr.start + sr.n_new, R);
  if (j0 >= n_ref) return;
  const int tid = threadIdx.x;
  const int64_t rowbase = (static_cast<int64_t>(s) * H + h) * max_ref_pad;

  // basis of this kv head as fp32: bs[kv][k][o]
  const T* bsrc = basis + static_cast<int64_t>(h) * 2 * d * r;
  for (int e = tid; e < 2 * d * r; e += blockDim.x) bs[e] = Elem<T>::to_f(bsrc[e]);

  // reference rows: copy to the contiguous buffer and stage as fp32
  const int vec_per_row = d2 / V;
  for (int e = tid; e < kPrepRefs * vec_per_row; e += blockDim.x) {
    const int jj = e / vec_per_row, c = e % vec_per_row;
    const int j = j0 + jj;
    float x[V];
    bool ok = j < n_ref;
    int pb = 0;
    if (ok) {
      pb = lookup_block(block_tables, max_blocks, num_blocks, s, j);
      ok = pb >= 0;
    }
    if (ok) {
      const T* src = refs + (static_cast<int64_t>(pb) * H + h) * d2 + c * V;
      V16<T>::load(src, x);
      V16<T>::store(refc + (rowbase + j) * d2 + c * V, x);
    } else {
#pragma unroll
      for (int q = 0; q < V; ++q) x[q] = 0.f;
    }
#pragma unroll
    for (int q = 0; q < V; ++q) rs[jj * rs_stride + c * V + q] = x[q];
  }
  __syncthreads();

  // inverse norms: warp w handles references w, w+8, w+16, w+24
  const int w = tid >> 5, lane = tid & 31;
  for (int jj = w; jj < kPrepRefs; jj += 8) {
    float ss = 0.f;
    for (int k = lane; k < d2; k += 32) ss = fmaf(rs[jj * rs_stride + k], rs[jj * rs_stride + k], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0 && j0 + jj < n_ref) invn[rowbase + j0 + jj] = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
  }

  // projections: 8 threads per reference, each a contiguous run of 2r/8 outputs (K half: threads 0-3)
  const int jj = tid >> 3, part = tid & 7;
  const int no = r2 / 8;
  const int o0 = part * no;
  const int kv = o0 >= r ? 1 : 0;
  float acc[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) acc[m] = 0.f;
  const float* xr = rs + jj * rs_stride + kv * d;
  const float* bk = bs + kv * d * r + (o0 - kv * r);
  for (int k = 0; k < d; ++k) {
    const float xv = xr[k];
#pragma unroll
    for (int m = 0; m < 16; ++m)
      if (m < no) acc[m] = fmaf(xv, bk[k * r + m], acc[m]);
  }
  if (j0 + jj < n_ref) {
    float* dst = pr + (rowbase + j0 + jj) * r2 + o0;
#pragma unroll
    for (int m = 0; m < 16; ++m)
      if (m < no) dst[m] = acc[m];
  }
}

// blockdiag(B_K, B_V)^T as bf16 [2r][2d] per kv head: the B operand of the projection MMA.
__global__ void __launch_bounds__(256) blockdiag_kernel(const __nv_bfloat16* __restrict__ basis, int d, int r,
                                                        __nv_bfloat16* __restrict__ bd) {
  const int h = blockIdx.x;
  const int d2 = 2 * d, r2 = 2 * r;
  const __nv_bfloat16* b = basis + static_cast<int64_t>(h) * 2 * d * r;
  const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
  for (int e = threadIdx.x; e < r2 * d2; e += blockDim.x) {
    const int o = e / d2, k = e % d2;
    __nv_bfloat16 v = zero;
    if (o < r && k < d) v = b[k * r + o];
    if (o >= r && k >= d) v = b[d * r + (k - d) * r + (o - r)];
    bd[static_cast<int64_t>(h) * r2 * d2 + e] = v;
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
// 3b. tcgen05 search + codes (bf16 storage).
//
// Persistent CTAs, one per SM.  A work unit is 256 new tokens (two 128-row token tiles) of one
// (seq, kv head).  Its centred tokens stay resident in shared memory (operand A, K-major, 128-byte
// swizzle) while the visible references stream through a ring of 64-column K-chunks (operand B):
//   warp 0      TMA producer (one lane): A tiles, reference chunks, 1/|r| slices, the projection basis
//   warp 1      MMA issuer (one lane) + tensor-memory owner: per reference tile, D[tok][ref] over K = 2d
//               into one of two 256-column accumulators (both token tiles side by side); the last
//               item of a unit is the projection P = x~ . blockdiag(B_K, B_V) (N = 2r)
//   warps 2..9  epilogue: tcgen05.ld rows, scale by 1/|r_j|, causal mask j*R < t, running argmax (ties to
//               the smallest j); on the projection item, code = RNE(P - PR_j*), scattered to the cache.
// Accumulator double-buffering lets the epilogue of tile i overlap the MMAs of tile i+1.
// ------------------------------------------------------------------------------------------------
constexpr int kTcThreads = 320;
constexpr int kTcTileM = 128;
constexpr int kTcTiles = 2;                      // token tiles per unit
constexpr int kTcUnit = kTcTileM * kTcTiles;     // tokens per unit
constexpr int kTcStageBytes = 16384;             // 128 rows x 64 bf16
constexpr int kTcEpiWarps = 8;

template <int CH>
struct TcConfig {
  static constexpr int kABytes = kTcTiles * CH * kTcStageBytes;
  static constexpr int kStages = CH == 4 ? 5 : 8;
  static constexpr int kBarOffset = kABytes + kStages * kTcStageBytes + 2 * kRefTile * 4;
  static constexpr int kNumBars = 2 + 2 * kStages + 6;
  static constexpr int kSmemBytes = kBarOffset + kNumBars * 8 + 16 + 1024;  // + alignment slack
};

template <int CH>
__global__ void __launch_bounds__(kTcThreads, 1) search_tc_kernel(
    const __grid_constant__ CUtensorMap xt_map, const __grid_constant__ CUtensorMap refc_map,
    const __grid_constant__ CUtensorMap bd_map, const float* __restrict__ invn, const float* __restrict__ pr,
    const int* __restrict__ cu_new, const int* __restrict__ start_pos, const int* __restrict__ block_tables,
    int max_blocks, int num_blocks, int num_seqs, int H, int R, int r, int64_t total_new, int64_t max_ref_pad,
    int max_new, int max_ctx, int num_pairs, __nv_bfloat16* __restrict__ codes, int* __restrict__ ref_idx) {
  using C = TcConfig<CH>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kABytes;
  float* sInv = reinterpret_cast<float*>(sB + NS * kTcStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* a_full = bars + 0;
  uint64_t* a_empty = bars + 1;
  uint64_t* b_full = bars + 2;
  uint64_t* b_empty = bars + 2 + NS;
  uint64_t* acc_full = bars + 2 + 2 * NS;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* inv_full = acc_full + 4;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* sAbort = reinterpret_cast<volatile int*>(sTmem + 1);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(a_full), 1);
    mbar_init(smem_u32(a_empty), 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(smem_u32(b_full + i), 1);
      mbar_init(smem_u32(b_empty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(acc_full + i), 1);
      mbar_init(smem_u32(acc_empty + i), kTcEpiWarps);
      mbar_init(smem_u32(inv_full + i), 1);
    }
    *sAbort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&xt_map);
    prefetch_tensormap(&refc_map);
    prefetch_tensormap(&bd_map);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(sTmem), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *sTmem;

  const int r2 = 2 * r;
  const int64_t total_units = static_cast<int64_t>(num_pairs) * num_seqs * H;
  // per-role pipeline state
  uint32_t a_phase = 0, stage = 0, item = 0;
  uint32_t inv_cnt0 = 0, inv_cnt1 = 0;
  bool failed = false;

  for (int64_t u = blockIdx.x; u < total_units && !failed; u += gridDim.x) {
    // longest-first order: the last token pairs of every (seq, head) come first
    const int p = num_pairs - 1 - static_cast<int>(u / (static_cast<int64_t>(num_seqs) * H));
    const int rem = static_cast<int>(u % (static_cast<int64_t>(num_seqs) * H));
    const int s = rem / H, h = rem % H;
    SeqRange sr;
    if (!load_seq(cu_new, start_pos, s, total_new, max_new, max_ctx, sr)) continue;  // recorded by center
    if (p * kTcUnit >= sr.n_new) continue;
    const int t0 = sr.start + p * kTcUnit;
    const int n_here = min(kTcUnit, sr.n_new - p * kTcUnit);
    const int t_last = t0 + n_here - 1;
    const int nvis = ceil_div_i(t_last, R);
    const int nrt = ceil_div_i(nvis, kRefTile);
    const int row0 = static_cast<int>(static_cast<int64_t>(h) * total_new + sr.base + p * kTcUnit);
    const int64_t refrow0 = (static_cast<int64_t>(s) * H + h) * max_ref_pad;

    if (warp == 0) {
      if (lane == 0) {
        // ---------------- producer ----------------
        if (!mbar_wait(smem_u32(a_empty), a_phase ^ 1, sAbort)) { failed = true; break; }
        mbar_arrive_expect_tx(smem_u32(a_full), kTcTiles * CH * kTcStageBytes);
        for (int tt = 0; tt < kTcTiles; ++tt)
          for (int c = 0; c < CH; ++c)
            tma_load_2d(smem_u32(sA + (tt * CH + c) * kTcStageBytes), &xt_map, c * 64, row0 + tt * kTcTileM,
                        smem_u32(a_full));
        a_phase ^= 1;
        for (int rt = 0; rt <= nrt; ++rt, ++item) {
          const uint32_t buf = item & 1;
          if (rt < nrt) {
            if (!mbar_wait(smem_u32(acc_empty + buf), ((item >> 1) & 1) ^ 1, sAbort)) { failed = true; break; }
            mbar_arrive_expect_tx(smem_u32(inv_full + buf), kRefTile * 4);
            bulk_g2s(smem_u32(sInv + buf * kRefTile), invn + refrow0 + rt * kRefTile, kRefTile * 4,
                     smem_u32(inv_full + buf));
          }
          for (int c = 0; c < CH; ++c, ++stage) {
            const uint32_t slot = stage % NS;
            if (!mbar_wait(smem_u32(b_empty + slot), ((stage / NS) & 1) ^ 1, sAbort)) { failed = true; break; }
            if (rt < nrt) {
              mbar_arrive_expect_tx(smem_u32(b_full + slot), kTcStageBytes);
              tma_load_2d(smem_u32(sB + slot * kTcStageBytes), &refc_map, c * 64,
                          static_cast<int>(refrow0 + rt * kRefTile), smem_u32(b_full + slot));
            } else {
              mbar_arrive_expect_tx(smem_u32(b_full + slot), r2 * 128);
              tma_load_2d(smem_u32(sB + slot * kTcStageBytes), &bd_map, c * 64, h * r2, smem_u32(b_full + slot));
            }
          }
          if (failed) break;
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // ---------------- MMA issuer ----------------
        if (!mbar_wait(smem_u32(a_full), a_phase, sAbort)) { failed = true; break; }
        a_phase ^= 1;
        tc_fence_after();
        for (int rt = 0; rt <= nrt; ++rt, ++item) {
          const uint32_t buf = item & 1;
          if (!mbar_wait(smem_u32(acc_empty + buf), ((item >> 1) & 1) ^ 1, sAbort)) { failed = true; break; }
          tc_fence_after();
          const uint32_t idesc = idesc_bf16_f32(kTcTileM, rt < nrt ? kRefTile : r2);
          for (int c = 0; c < CH; ++c, ++stage) {
            const uint32_t slot = stage % NS;
            if (!mbar_wait(smem_u32(b_full + slot), (stage / NS) & 1, sAbort)) { failed = true; break; }
            tc_fence_after();
            const uint32_t b_addr = smem_u32(sB + slot * kTcStageBytes);
#pragma unroll
            for (int tt = 0; tt < kTcTiles; ++tt) {
              const uint32_t a_addr = smem_u32(sA + (tt * CH + c) * kTcStageBytes);
              const uint32_t d_tmem = tmem_base + buf * 256 + tt * kTcTileM;
#pragma unroll
              for (int k = 0; k < 4; ++k)
                umma_bf16(d_tmem, sw128_kmajor_desc(a_addr + k * 32), sw128_kmajor_desc(b_addr + k * 32), idesc,
                          (c | k) != 0 ? 1u : 0u);
            }
            umma_commit(smem_u32(b_empty + slot));
          }
          if (failed) break;
          umma_commit(smem_u32(acc_full + buf));
        }
        if (failed) break;
        umma_commit(smem_u32(a_empty));
      }
    } else {
      // ---------------- epilogue ----------------
      const int ew = warp - 2;
      const int tt = ew >> 2;
      const int q = warp & 3;  // tensor-memory lane quarter this warp may access
      const int row = q * 32 + lane;
      const int i = tt * kTcTileM + row;
      const bool valid = i < n_here;
      const int t = t0 + i;
      const int jlim = valid ? ceil_div_i(t, R) : 0;
      const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + tt * kTcTileM;
      float best[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      int bj[4] = {0, 0, 0, 0};
      for (int rt = 0; rt < nrt; ++rt, ++item) {
        const uint32_t buf = item & 1;
        uint32_t& ic = buf ? inv_cnt1 : inv_cnt0;
        if (!mbar_wait(smem_u32(acc_full + buf), (item >> 1) & 1, sAbort)) { failed = true; break; }
        if (!mbar_wait(smem_u32(inv_full + buf), ic & 1, sAbort)) { failed = true; break; }
        ++ic;
        tc_fence_after();
        const float* inv = sInv + buf * kRefTile;
        const int jb = rt * kRefTile;
        const bool full = jb + kRefTile <= jlim;
#pragma unroll 1
        for (int cc = 0; cc < kRefTile / 32; ++cc) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(lane_base + buf * 256 + cc * 32, v);
          tmem_ld_wait();
          const float4* inv4 = reinterpret_cast<const float4*>(inv + cc * 32);
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 iv = inv4[e4];
            const float ivs[4] = {iv.x, iv.y, iv.z, iv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = jb + cc * 32 + e4 * 4 + e;
              const float sc = __uint_as_float(v[e4 * 4 + e]) * ivs[e];
              if ((full || j < jlim) && sc > best[e]) {
                best[e] = sc;
                bj[e] = j;
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(acc_empty + buf));
      }
      if (failed) break;
      // projection item: codes
      const uint32_t buf = item & 1;
      if (!mbar_wait(smem_u32(acc_full + buf), (item >> 1) & 1, sAbort)) { failed = true; break; }
      tc_fence_after();
      int js = bj[0];
      float bs = best[0];
#pragma unroll
      for (int e = 1; e < 4; ++e)
        if (best[e] > bs || (best[e] == bs && bj[e] < js)) {
          bs = best[e];
          js = bj[e];
        }
      const bool isref = valid && (t % R) == 0;
      if (isref) js = t / R;
      int pb = -1;
      if (valid) pb = lookup_block(block_tables, max_blocks, num_blocks, s, t / R);
      const float* prow = pr + (refrow0 + js) * r2;
      __nv_bfloat16* cdst =
          pb >= 0 ? codes + ((static_cast<int64_t>(pb) * H + h) * R + t % R) * r2 : nullptr;
      for (int cc = 0; cc < r2 / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(lane_base + buf * 256 + cc * 32, v);
        tmem_ld_wait();
        if (pb >= 0) {
          uint32_t packed[16];
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 p4 = __ldg(reinterpret_cast<const float4*>(prow + cc * 32) + e4);
            const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
            float cv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) cv[e] = isref ? 0.f : __fsub_rn(__uint_as_float(v[e4 * 4 + e]), pv[e]);
            packed[e4 * 2] = pack_bf16x2(cv[0], cv[1]);
            packed[e4 * 2 + 1] = pack_bf16x2(cv[2], cv[3]);
          }
          uint4* dst4 = reinterpret_cast<uint4*>(cdst + cc * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst4[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(acc_empty + buf));
      ++item;
      if (pb >= 0) ref_idx[(static_cast<int64_t>(pb) * H + h) * R + t % R] = js;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ------------------------------------------------------------------------------------------------
// Host side.
// ------------------------------------------------------------------------------------------------
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

template <int CH>
static dkv_status launch_tc(const CompressArgs& a, const CompressWs& L, uint8_t* ws, cudaStream_t st) {
  const dkv_shape& sh = *a.shape;
  const int H = sh.num_kv_heads, d2 = 2 * sh.head_dim, r2 = 2 * sh.rank;
  CUtensorMap xt_map, refc_map, bd_map;
  if (!make_map_bf16(&xt_map, ws + L.xt, d2, static_cast<uint64_t>(H) * a.total_new, kTcTileM) ||
      !make_map_bf16(&refc_map, ws + L.refc, d2, static_cast<uint64_t>(a.num_seqs) * H * L.max_ref_pad,
                     kRefTile) ||
      !make_map_bf16(&bd_map, ws + L.bd, d2, static_cast<uint64_t>(H) * r2, r2))
    return DKV_ERR_CUDA;
  const int smem = TcConfig<CH>::kSmemBytes;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(search_tc_kernel<CH>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return DKV_ERR_CUDA;
    attr_set = true;
  }
  const int num_pairs = static_cast<int>(ceil_div64(a.max_new, kTcUnit));
  const int64_t units = static_cast<int64_t>(num_pairs) * a.num_seqs * H;
  const int grid = static_cast<int>(units < kNumSMs ? units : kNumSMs);
  prof_begin(DKV_KERNEL_SEARCH, st);
    search_tc_kernel<CH><<<grid, kTcThreads, smem, st>>>(
      xt_map, refc_map, bd_map, reinterpret_cast<const float*>(ws + L.invn),
      reinterpret_cast<const float*>(ws + L.pr), a.cu_new, a.start_pos, a.block_tables, a.max_blocks,
      a.cache->num_blocks, a.num_seqs, H, sh.ref_stride, sh.rank, a.total_new, L.max_ref_pad, a.max_new,
      a.max_ctx, num_pairs, static_cast<__nv_bfloat16*>(a.cache->codes), a.cache->ref_idx);
    prof_end(DKV_KERNEL_SEARCH, st);
  return DKV_OK;
}

template <typename T>
static dkv_status launch_compress_t(const CompressArgs& a, uint8_t* ws, cudaStream_t st) {
  const dkv_shape& sh = *a.shape;
  const int H = sh.num_kv_heads, d = sh.head_dim, r = sh.rank, R = sh.ref_stride;
  const CompressWs L = compress_ws_layout(sh, a.num_seqs, a.total_new, a.max_ctx);
  T* xt = reinterpret_cast<T*>(ws + L.xt);
  T* refc = reinterpret_cast<T*>(ws + L.refc);
  float* invn = reinterpret_cast<float*>(ws + L.invn);
  float* pr = reinterpret_cast<float*>(ws + L.pr);
  // 1. centre
  {
    const int64_t per_tok = static_cast<int64_t>(H) * 2 * (d / V16<T>::N);
    const int64_t n = per_tok * a.max_new;
    dim3 grid(static_cast<unsigned>(ceil_div64(n, 256)), a.num_seqs);
    prof_begin(DKV_KERNEL_CENTER, st);
    center_kernel<T><<<grid, 256, 0, st>>>(static_cast<const T*>(a.k_new), static_cast<const T*>(a.v_new),
                                           a.params->mu, a.cu_new, a.start_pos, a.block_tables, a.max_blocks,
                                           a.cache->num_blocks, H, d, R, a.total_new, a.max_new, a.max_ctx, xt,
                                           static_cast<T*>(a.cache->refs));
    prof_end(DKV_KERNEL_CENTER, st);
  }
  // 2. reference prep
  {
    const int nref = max_refs(a.max_ctx, R);
    dim3 grid(static_cast<unsigned>(ceil_div64(nref, kPrepRefs)), H, a.num_seqs);
    const size_t smem = (static_cast<size_t>(kPrepRefs) * (2 * d + 1) + 2 * d * r) * sizeof(float);
    static bool attr = false;
    if (!attr) {
      cudaFuncSetAttribute(refprep_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
      attr = true;
    }
    prof_begin(DKV_KERNEL_REFPREP, st);
    refprep_kernel<T><<<grid, 256, smem, st>>>(static_cast<const T*>(a.cache->refs),
                                               static_cast<const T*>(a.params->basis), a.cu_new, a.start_pos,
                                               a.block_tables, a.max_blocks, a.cache->num_blocks, H, d, r, R,
                                               a.total_new, a.max_new, a.max_ctx, L.max_ref_pad, refc, invn, pr);
    prof_end(DKV_KERNEL_REFPREP, st);
  }
  // 3. search + codes
  if constexpr (sizeof(T) == 2) {
#ifndef DKV_SEARCH_SIMT
    blockdiag_kernel<<<H, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(a.params->basis), d, r,
                                         reinterpret_cast<__nv_bfloat16*>(ws + L.bd));
    const dkv_status stt = d == 64 ? launch_tc<2>(a, L, ws, st) : launch_tc<4>(a, L, ws, st);
    if (stt != DKV_OK) return stt;
    return DKV_OK;
#endif
  }
  {
    dim3 grid(static_cast<unsigned>(ceil_div64(a.max_new, kSimtTok)), H, a.num_seqs);
    const size_t smem = (static_cast<size_t>(2 * d) * kSimtTok + kSimtRefs * 2 * d + kSimtRefs) * sizeof(float);
    static bool attr = false;
    if (!attr) {
      cudaFuncSetAttribute(search_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
      attr = true;
    }
    prof_begin(DKV_KERNEL_SEARCH, st);
    search_simt_kernel<T><<<grid, kSimtTok, smem, st>>>(
        xt, refc, invn, static_cast<const T*>(a.params->basis), a.cu_new, a.start_pos, a.block_tables,
        a.max_blocks, a.cache->num_blocks, H, d, r, R, a.total_new, a.max_new, a.max_ctx, L.max_ref_pad,
        static_cast<T*>(a.cache->codes), a.cache->ref_idx);
    prof_end(DKV_KERNEL_SEARCH, st);
  }
  return DKV_OK;
}

dkv_status launch_compress(const CompressArgs& a, void* workspace, cudaStream_t st) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const dkv_status s = a.shape->dtype == DKV_F32 ? launch_compress_t<float>(a, ws, st)
                                                 : launch_compress_t<__nv_bfloat16>(a, ws, st);
  if (s != DKV_OK) return s;
  return cudaGetLastError() == cudaSuccess ? DKV_OK : DKV_ERR_CUDA;
}

}  // namespace dkv
