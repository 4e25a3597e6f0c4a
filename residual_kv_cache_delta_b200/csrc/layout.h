// Host-side workspace layouts and launch-shape choices.  The *_workspace queries and the entry points
// both derive every offset from these functions, so a size returned by a query always fits the call.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "../../include/deltakv.h"

namespace dkv {

constexpr int kDefaultSMs = 148;       // B200; used only when no device can be queried
constexpr size_t kWsAlign = 1024;      // every workspace sub-buffer starts 1024-byte aligned
constexpr int kRefTile = 256;          // references per tensor-core tile (N of the pair score MMA)
constexpr int kCombineRefs = 128;      // references per combine CTA

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Streaming multiprocessors of the current device, queried once per device ordinal.  A size query on a host
// without a usable device falls back to the B200's 148, so that query still answers.
inline int num_sms() {
  static std::mutex mu;
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();  // leave no error behind for a later launch check
    return kDefaultSMs;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      return kDefaultSMs;
    }
    cached[dev] = n;
  }
  return cached[dev];
}

inline int elem_bytes(const dkv_shape& s) { return s.dtype == DKV_F32 ? 4 : 2; }
inline bool is_q4(const dkv_shape& s) { return s.dtype == DKV_BF16_Q4; }
// Bytes of one token's codes: 2r storage values, or r bytes of nibbles plus two bf16 scales (4-bit codes).
inline int code_row_bytes(const dkv_shape& s) { return is_q4(s) ? s.rank + 4 : 2 * s.rank * elem_bytes(s); }
inline int max_refs(int max_ctx, int R) { return static_cast<int>(ceil_div64(max_ctx, R)); }

struct CompressWs {
  int64_t max_ref_pad = 0;  // per (seq, kv head) reference rows, padded to a whole tile
  size_t xt = 0, refc = 0, invn = 0, pr = 0, bd = 0, counter = 0, total = 0;
};

// xt   [H_kv][total_new][2d]              centred new tokens (fp32 path only), head-major
// refc [num_seqs][H_kv][max_ref_pad][2d]  contiguous copy of every visible reference (storage dtype)
// invn [num_seqs][H_kv][max_ref_pad]      1/|r~_j| (fp32)
// pr   [num_seqs][H_kv][max_ref_pad][2r]  projections r~_j . blockdiag(B_K, B_V) (fp32)
// bd   [H_kv][2r][2d]                     blockdiag(B_K, B_V)^T (bf16; tensor-core operand)
// counter                                 int32 work counter of the search kernel (cleared by each call)
inline CompressWs compress_ws_layout(const dkv_shape& s, int num_seqs, int64_t total_new, int max_ctx) {
  CompressWs w;
  const int64_t H = s.num_kv_heads, d2 = 2 * s.head_dim, r2 = 2 * s.rank;
  const int es = elem_bytes(s);
  w.max_ref_pad = align_up(static_cast<size_t>(max_refs(max_ctx, s.ref_stride)), kRefTile);
  if (w.max_ref_pad == 0) w.max_ref_pad = kRefTile;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, kWsAlign);
    return o;
  };
  // the tensor-core (bf16) path centres its token tiles inside the search kernel and needs no copy
  w.xt = take(s.dtype == DKV_F32 ? static_cast<size_t>(H * total_new * d2 * es) : 0);
  const size_t nrows = static_cast<size_t>(num_seqs) * H * w.max_ref_pad;
  w.refc = take(nrows * d2 * es);
  w.invn = take(nrows * 4);
  w.pr = take(nrows * r2 * 4);
  w.bd = take(static_cast<size_t>(H * r2 * d2 * 2));
  w.counter = take(sizeof(int));
  w.total = off;
  return w;
}

// Tokens per shared-memory stage of the decode split kernel: about 16 KB of codes, 64..256 tokens.
constexpr int decode_stage_tokens(int rank, int elem) {
  return 16384 / (2 * rank * elem) < 64 ? 64 : (16384 / (2 * rank * elem) > 256 ? 256 : 16384 / (2 * rank * elem));
}

// Decode split-K plan.  The split kernel runs one or two CTAs per SM (slots); a CTA costs its tokens plus a
// fixed overhead (pipeline fill, per-reference mass write-out) worth about 256 tokens.  Among split counts n,
// pick the one minimising waves(n) * (tokens per split + 256), so that (seq, kv head, split) CTAs fill
// whole waves of the device's slots.  Split sizes are whole stages.
constexpr int kMaxSplitTokens = 8192;  // bounds the fixed-point per-reference mass of one split

inline void decode_split_plan(int units, int max_ctx, int stage_tokens, int slots_per_sm, int* tps_out,
                              int* nsplit_out) {
  int best_t = stage_tokens, best_n = 1;
  double best_cost = -1.0;
  const int nmax = static_cast<int>(ceil_div64(max_ctx > 0 ? max_ctx : 1, stage_tokens));
  const int sms = num_sms() * slots_per_sm;
  for (int n = 1; n <= nmax && n <= 4096; ++n) {
    const int64_t t = align_up(static_cast<size_t>(ceil_div64(max_ctx, n)), stage_tokens);
    if (t <= 0) break;
    if (t > kMaxSplitTokens) continue;
    const int64_t nn = ceil_div64(max_ctx, t);
    if (nn != n) continue;
    const int64_t waves = ceil_div64(static_cast<int64_t>(units) * nn, sms);
    const double cost = static_cast<double>(waves) * static_cast<double>(t + 256);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_t = static_cast<int>(t);
      best_n = n;
    }
  }
  *tps_out = best_t;
  *nsplit_out = best_n;
}

struct DecodeWs {
  int tps = 0, nsplit = 0, max_ref = 0, nchunk = 0;
  size_t qp = 0, qmu = 0, sref = 0, ml = 0, acc = 0, bins = 0, cpart = 0, cnt = 0, total = 0;
};

// qp    [num_seqs][H_q][r]            q.B_K, scaled by softmax_scale*log2(e) (fp32)
// qmu   [num_seqs][H_q]               q.mu_K, scaled
// sref  [num_seqs][H_kv][max_ref][G]  q.r~K_j, scaled
// ml    [num_seqs][H_q][nsplit][2]    per split: running max (log2 domain), softmax mass
// acc   [num_seqs][H_q][nsplit][r]    per split: sum p * cV
// bins  [num_seqs][H_kv][nsplit][max_ref][G]  per split: softmax mass per reference
// cpart [num_seqs][H_kv][nchunk][G][d]        combine partials: sum_j w_j r~V_j per chunk of refs
// cnt   [num_seqs][H_kv]              combine arrival counters (int32, cleared by each call)
// max_sel >= 0: sparse decode, whose splits run over a selected list of at most max_sel entries per sequence
// (the per-reference arrays still cover the whole context).
// slots_per_sm: split CTAs resident per SM (the tensor-core split kernel runs one or two).
inline DecodeWs decode_ws_layout(const dkv_shape& s, int num_seqs, int max_ctx, int max_sel = -1,
                                 int slots_per_sm = 1) {
  DecodeWs w;
  const int64_t Hq = s.num_q_heads, Hkv = s.num_kv_heads, G = Hq / Hkv, r = s.rank, d = s.head_dim;
  // splits are whole multiples of every stage size the split kernels use (64, 128 or 256 tokens)
  decode_split_plan(static_cast<int>(num_seqs * Hkv), max_sel >= 0 ? max_sel : max_ctx, 256, slots_per_sm, &w.tps,
                    &w.nsplit);
  w.max_ref = max_refs(max_ctx, s.ref_stride);
  if (w.max_ref < 1) w.max_ref = 1;
  w.nchunk = static_cast<int>(ceil_div64(w.max_ref, kCombineRefs));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, kWsAlign);
    return o;
  };
  const size_t S = static_cast<size_t>(num_seqs);
  w.qp = take(S * Hq * r * 4);
  w.qmu = take(S * Hq * 4);
  w.sref = take(S * Hkv * w.max_ref * G * 4);
  w.ml = take(S * Hq * w.nsplit * 2 * 4);
  w.acc = take(S * Hq * w.nsplit * r * 4);
  w.bins = take(S * Hkv * w.nsplit * static_cast<size_t>(w.max_ref) * G * 4);
  w.cpart = take(S * Hkv * w.nchunk * G * d * 4);
  w.cnt = take(S * Hkv * 4);
  w.total = off;
  return w;
}

}  // namespace dkv
