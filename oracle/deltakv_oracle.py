"""Plain CPU oracle of the DeltaKV hot path: compress (centre, search, code) and decode attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may import this module.  The product path (the CUDA library and its
Python binding) never does, and this module never imports the product package.

Everything is NumPy in float64 unless a step is defined in a narrower type.  Each function follows
the written definition step by step; there is no tiling, fusion or reordering beyond what a library
primitive (a matrix product, an argmax) does internally.

Source: "DeltaKV: Residual-Based KV Cache Compression via Long-Range Similarity" (Hao, Huang, Wang,
Zhang, Yu), as summarised on gist.science (English summary, Technical Summary §2 "Key Empirical
Observations" and §3 "Methodology"; French summary §2 "Méthodologie").  The summaries fix the method
only in outline; the concrete form implemented here is:

  centre    x~_t = RNE_S(fp32(x_t - mu))                     shared high-norm component removed
  search    idx(t) = argmax_{j : jR < t} <x~_t, r~_j> / |r~_j| (ties -> smallest j); refs: idx = t/R
  code      c_t = RNE_S( (x~_t - r~_idx)_K B_K ; (x~_t - r~_idx)_V B_V )   (0 for reference tokens)
  rebuild   K^_t = mu_K + r~K_idx + cK_t B_K^T   (likewise V)
  decode    out = softmax(scale * K^ q) V^,  lse = logsumexp(scale * K^ q)
  sparse    the same over a caller-given subset of the cached positions
  q4        codes stored as 4-bit integers with one bf16 scale per token and K/V half (absmax / 7)
  top-k L2  the pages' retrieval: the k references nearest by L2 distance, residual against their mean

Readings taken where the pages are silent or differ: cosine top-1 over every earlier reference
instead of the pages' k-nearest by L2 with a mean (k = 1 makes the mean the reference itself); one index per (token, kv head) from
the concatenated centred [k~ ; v~]; references stored centred; mu is an input parameter; a linear
rank-r compressor f_c(x) = x B, whose decompressor is f_d(z) = z B^T, so the residual in code space
f_c(x) - f_c(x^R) equals f_c(x - x^R); scale = 1/sqrt(d); zero-norm references score 0.

Pins (tests that fix this oracle to something other than itself) are in ``tests/test_oracle_pins.py``.
Parity pinned for every function here.  The pages' trained MLP compressors are out of scope (the linear
basis is an input), so nothing of them is claimed.
"""
from __future__ import annotations

import numpy as np

# --------------------------------------------------------------------------------------------------
# Storage rounding.  Both formats share fp32's exponent range; they differ in mantissa bits.
# --------------------------------------------------------------------------------------------------
_MANT_BITS = {"f32": 23, "bf16": 7}
_EMIN = -126  # smallest normal exponent of fp32 and bf16
_MAX = {"f32": float(np.finfo(np.float32).max), "bf16": float.fromhex("0x1.fe00000000000p+127")}


def round_to_storage(x, dtype: str) -> np.ndarray:
    """Round float64 values to the nearest value of the storage format, ties to even (IEEE RNE).

    The quantum at value x is 2^(max(e, -126) - m) with e = floor(log2|x|) and m mantissa bits; the
    rounding is rint(x / q) * q, which is exact in float64 for these formats.  Values whose rounded
    magnitude exceeds the format's largest finite value become +-inf; NaN stays NaN.
    """
    x = np.asarray(x, dtype=np.float64)
    m = _MANT_BITS[dtype]
    out = np.array(x, copy=True)
    fin = np.isfinite(x) & (x != 0)
    xf = x[fin]
    _, e2 = np.frexp(xf)  # xf = f * 2^e2 with 0.5 <= |f| < 1, so floor(log2|x|) = e2 - 1
    e = np.maximum(e2 - 1, _EMIN)
    q = np.ldexp(1.0, e - m)
    r = np.rint(xf / q) * q
    r = np.where(np.abs(r) > _MAX[dtype], np.copysign(np.inf, r), r)
    out[fin] = r
    return out


def storage_fp32_sub(x, mu) -> np.ndarray:
    """fp32(x - mu): IEEE single-precision subtraction of storage values and the fp32 shared component."""
    return (np.asarray(x, dtype=np.float64).astype(np.float32) - np.asarray(mu, dtype=np.float32)).astype(np.float64)


# --------------------------------------------------------------------------------------------------
# Compress.
# --------------------------------------------------------------------------------------------------
def center(x, mu, dtype: str) -> np.ndarray:
    """Remove the shared high-norm component: x~ = RNE_S(fp32(x - mu)).

    DeltaKV summary (en) §2, "Highly Shared Latent Components": a few high-norm directions are common to
    all tokens; subtracting them leaves low-magnitude residuals.  Here the shared part is one per-head
    vector mu (an input), subtracted in fp32 and rounded once to the storage type.
    """
    return round_to_storage(storage_fp32_sub(x, mu), dtype)


def is_reference(pos, R: int) -> np.ndarray:
    """Strided reference selection: token t is a reference iff t mod R == 0 (summary (en) §3)."""
    return np.asarray(pos) % R == 0


def visible_refs(t: int, R: int) -> int:
    """Number of references strictly before position t: #{j : j*R < t} = ceil(t / R)."""
    return -(-int(t) // R)


def ref_scores(xt_row, refs, t: int, R: int) -> np.ndarray:
    """Cosine-style scores <x~_t, r~_j> / |r~_j| (0 for a zero-norm r~_j) over the visible refs j < ceil(t/R)."""
    n = visible_refs(t, R)
    rr = np.asarray(refs, dtype=np.float64)[:n]
    dots = rr @ np.asarray(xt_row, dtype=np.float64)
    norms = np.sqrt(np.einsum("ij,ij->i", rr, rr))
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(norms > 0, dots / norms, 0.0)


def search(xt, refs, positions, R: int, chunk: int = 4096) -> np.ndarray:
    """Long-range similarity retrieval (summary (en) §3, "Strided Reference Selection"): each non-reference
    token takes the most similar earlier reference by cosine over the whole prefix; exact ties go to the
    smallest j; a reference token t takes idx = t / R.

    xt: [n, 2d] centred tokens at absolute ``positions``; refs: [n_ref, 2d] centred references of the same
    (sequence, kv head), ref j being the token at position j*R.  Returns int64 [n].
    """
    xt = np.asarray(xt, dtype=np.float64)
    refs = np.asarray(refs, dtype=np.float64)
    pos = np.asarray(positions, dtype=np.int64)
    idx = np.zeros(len(pos), dtype=np.int64)
    norms = np.sqrt(np.einsum("ij,ij->i", refs, refs))
    j = np.arange(len(refs), dtype=np.int64)
    for a in range(0, len(pos), chunk):
        b = min(a + chunk, len(pos))
        with np.errstate(divide="ignore", invalid="ignore"):
            sc = np.where(norms[None, :] > 0, (xt[a:b] @ refs.T) / norms[None, :], 0.0)
        vis = j[None, :] * R < pos[a:b, None]
        sc = np.where(vis, sc, -np.inf)
        idx[a:b] = np.argmax(sc, axis=1) if len(refs) else 0  # argmax returns the first (smallest j) maximum
    refm = is_reference(pos, R)
    idx[refm] = pos[refm] // R
    return idx


def codes(xt, refs, idx, BK, BV, dtype: str, rounded: bool = True) -> np.ndarray:
    """Residual encoding with a linear compressor (summary (en) §3, "Residual Encoding"):
    z = f_c(x) - f_c(x^R) with f_c(x) = x B, i.e. c_t = RNE_S([(x~_t - r~_idx)_K B_K ; (x~_t - r~_idx)_V B_V]).

    Reference tokens have a zero residual and so a zero code.  Returns float64 [n, 2r] of S values
    (``rounded=False``: the exact float64 projection before the final rounding to S).
    """
    xt = np.asarray(xt, dtype=np.float64)
    res = xt - np.asarray(refs, dtype=np.float64)[np.asarray(idx)]
    d = xt.shape[1] // 2
    cK = res[:, :d] @ np.asarray(BK, dtype=np.float64)
    cV = res[:, d:] @ np.asarray(BV, dtype=np.float64)
    c = np.concatenate([cK, cV], axis=1)
    return round_to_storage(c, dtype) if rounded else c


def compress(k, v, mu_k, mu_v, BK, BV, R: int, dtype: str, start: int = 0, prev_refs=None):
    """Compress the tokens at positions start..start+n-1 of one (sequence, kv head).

    k, v: [n, d] storage values; prev_refs: [ceil(start/R), 2d] centred refs already stored (or None).
    Returns (refs_all [n_ref_total, 2d], idx [n], codes [n, 2r], xt [n, 2d]).
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n = k.shape[0]
    pos = np.arange(start, start + n)
    xt = np.concatenate([center(k, mu_k, dtype), center(v, mu_v, dtype)], axis=1)
    new_refs = xt[is_reference(pos, R)]
    prev = np.zeros((0, xt.shape[1])) if prev_refs is None else np.asarray(prev_refs, dtype=np.float64)
    refs_all = np.concatenate([prev, new_refs], axis=0)
    idx = search(xt, refs_all, pos, R)
    c = codes(xt, refs_all, idx, BK, BV, dtype)
    return refs_all, idx, c, xt


# --------------------------------------------------------------------------------------------------
# The pages' own retrieval: the k nearest references by L2 distance, residual against their mean.
# --------------------------------------------------------------------------------------------------
def l2_scores(xt_row, refs, t: int, R: int) -> np.ndarray:
    """2<x~_t, r~_j> - |r~_j|^2 over the visible refs j < ceil(t/R): larger is nearer, since
    |x~_t - r~_j|^2 = |x~_t|^2 - (2<x~_t, r~_j> - |r~_j|^2) and |x~_t|^2 is the same for every j."""
    rr = np.asarray(refs, dtype=np.float64)[:visible_refs(t, R)]
    return 2.0 * (rr @ np.asarray(xt_row, dtype=np.float64)) - np.einsum("ij,ij->i", rr, rr)


def search_topk_l2(xt, refs, positions, R: int, k: int) -> np.ndarray:
    """k-nearest reference retrieval by L2 distance (summary (en) §3, "Strided Reference Selection" and "Residual
    Encoding"; summary (fr) §2): each non-reference token takes the k visible references nearest to it in L2
    distance on the centred [k~; v~] (ties: the smaller j first); with fewer than k visible references it takes
    all of them.  The chosen ordinals are stored in ascending order, unused slots as -1; a reference token t
    takes t / R in every slot.  Returns int64 [n, k]."""
    xt = np.asarray(xt, dtype=np.float64)
    pos = np.asarray(positions, dtype=np.int64)
    out = np.full((len(pos), k), -1, dtype=np.int64)
    for i, t in enumerate(pos):
        t = int(t)
        if t % R == 0:
            out[i] = t // R
            continue
        sc = l2_scores(xt[i], refs, t, R)
        order = np.lexsort((np.arange(len(sc)), -sc))  # by score descending, then j ascending
        sel = np.sort(order[:k])
        out[i, :len(sel)] = sel
    return out


def mean_refs(refs, idx_k) -> np.ndarray:
    """Mean of the references named by each row of idx_k (ignoring -1 slots): float64 [n, 2d]."""
    refs = np.asarray(refs, dtype=np.float64)
    idx_k = np.asarray(idx_k)
    valid = idx_k >= 0
    acc = np.zeros((idx_k.shape[0], refs.shape[1]))
    for c in range(idx_k.shape[1]):
        acc += np.where(valid[:, c:c + 1], refs[np.maximum(idx_k[:, c], 0)], 0.0)
    return acc / valid.sum(axis=1, keepdims=True)


def codes_topk(xt, refs, idx_k, BK, BV, dtype: str, rounded: bool = True) -> np.ndarray:
    """Residual against the mean of the retrieved references through the linear compressor:
    c_t = RNE_S([(x~_t - mean)_K B_K ; (x~_t - mean)_V B_V]) (summary (en) §3, "Residual Encoding")."""
    xt = np.asarray(xt, dtype=np.float64)
    res = xt - mean_refs(refs, idx_k)
    d = xt.shape[1] // 2
    c = np.concatenate([res[:, :d] @ np.asarray(BK, dtype=np.float64), res[:, d:] @ np.asarray(BV, dtype=np.float64)],
                       axis=1)
    return round_to_storage(c, dtype) if rounded else c


def compress_topk(k_, v_, mu_k, mu_v, BK, BV, R: int, dtype: str, k: int, start: int = 0, prev_refs=None):
    """compress() with the k-nearest-L2 retrieval.  Returns (refs_all, idx [n, k], codes [n, 2r], xt)."""
    k_ = np.asarray(k_, dtype=np.float64)
    v_ = np.asarray(v_, dtype=np.float64)
    n = k_.shape[0]
    pos = np.arange(start, start + n)
    xt = np.concatenate([center(k_, mu_k, dtype), center(v_, mu_v, dtype)], axis=1)
    prev = np.zeros((0, xt.shape[1])) if prev_refs is None else np.asarray(prev_refs, dtype=np.float64)
    refs_all = np.concatenate([prev, xt[is_reference(pos, R)]], axis=0)
    idx = search_topk_l2(xt, refs_all, pos, R, k)
    return refs_all, idx, codes_topk(xt, refs_all, idx, BK, BV, dtype), xt


def reconstruct_topk(mu_k, mu_v, refs, idx_k, cds, BK, BV):
    """K^_t = mu_K + mean_i r~K_{j_i} + cK_t B_K^T (likewise V): the rebuild with the mean of the references."""
    m = mean_refs(refs, idx_k)
    cds = np.asarray(cds, dtype=np.float64)
    BK = np.asarray(BK, dtype=np.float64)
    BV = np.asarray(BV, dtype=np.float64)
    d, r = BK.shape
    return (np.asarray(mu_k, dtype=np.float64)[None, :] + m[:, :d] + cds[:, :r] @ BK.T,
            np.asarray(mu_v, dtype=np.float64)[None, :] + m[:, d:] + cds[:, r:] @ BV.T)


def decode_topk(q, mu, refs, idx_k, cds, BK, BV, dtype: str, scale: float | None = None, rounded: bool = True):
    """GQA decode attention over a cache compressed with the k-nearest retrieval (explicit rebuild)."""
    q = np.asarray(q, dtype=np.float64)
    Hq, d = q.shape
    Hkv = len(refs)
    G = Hq // Hkv
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.zeros((Hq, d))
    lse = np.zeros(Hq)
    for g in range(Hkv):
        Kh, Vh = reconstruct_topk(mu[g][0], mu[g][1], refs[g], idx_k[g], cds[g], BK[g], BV[g])
        for hq in range(g * G, (g + 1) * G):
            out[hq], lse[hq] = attention(q[hq], Kh, Vh, sc)
    return (round_to_storage(out, dtype) if rounded else out), lse


# --------------------------------------------------------------------------------------------------
# 4-bit residual codes.
# --------------------------------------------------------------------------------------------------
Q4_MAX = 7  # symmetric 4-bit levels -7 .. 7 (the 16th pattern, -8, is never produced)


def quantize_q4(c, r: int):
    """4-bit quantisation of residual codes (summary (en) §5, "Memory Efficiency", and summary (es) §4: the 29%
    figure combines DeltaKV with 4-bit quantisation; the pages do not fix the scheme, so this is a symmetric
    absmax one).  Each K half (c[:, :r]) and V half (c[:, r:]) of a token gets one scale
        s = RNE_bf16(max_i |c_i| / 7)
    and integer codes q_i = clip(round_half_even(c_i / s), -7, 7) (all 0 when s = 0).  c: float64 [n, 2r] exact
    codes.  Returns (q int8 [n, 2r], s float64 [n, 2] of bf16 values: K scale, V scale)."""
    c = np.asarray(c, dtype=np.float64)
    n = c.shape[0]
    q = np.zeros((n, 2 * r), dtype=np.int8)
    s = np.zeros((n, 2))
    for half in range(2):
        ch = c[:, half * r:(half + 1) * r]
        sc = round_to_storage(np.max(np.abs(ch), axis=1) / Q4_MAX, "bf16") if n else np.zeros(0)
        with np.errstate(divide="ignore", invalid="ignore"):
            qq = np.where(sc[:, None] > 0, np.clip(np.rint(ch / sc[:, None]), -Q4_MAX, Q4_MAX), 0.0)
        q[:, half * r:(half + 1) * r] = qq.astype(np.int8)
        s[:, half] = sc
    return q, s


def dequantize_q4(q, s, r: int) -> np.ndarray:
    """Codes the 4-bit form stands for: c'_i = s_half * q_i (float64 [n, 2r])."""
    q = np.asarray(q, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    return np.concatenate([q[:, :r] * s[:, :1], q[:, r:] * s[:, 1:]], axis=1)


def compressed_bytes_per_token_q4(d: int, r: int, R: int, elem: int) -> float:
    """Bytes per token per kv head with 4-bit codes: 2r nibbles, two bf16 scales, the index, one ref per R."""
    return r + 2 * 2 + 4 + 2 * d * elem / R


# --------------------------------------------------------------------------------------------------
# Reconstruction and decode.
# --------------------------------------------------------------------------------------------------
def reconstruct(mu_k, mu_v, refs, idx, cds, BK, BV):
    """Reconstruction (summary (en) §3, "Reconstruction"; summary (fr) §2): KV^ = f_d(z) + KV^R with
    f_d(z) = z B^T, plus the shared component mu that was removed before encoding:
        K^_t = mu_K + r~K_idx(t) + cK_t B_K^T,   V^_t = mu_V + r~V_idx(t) + cV_t B_V^T.
    Returns float64 (K^ [T, d], V^ [T, d]).
    """
    refs = np.asarray(refs, dtype=np.float64)
    cds = np.asarray(cds, dtype=np.float64)
    BK = np.asarray(BK, dtype=np.float64)
    BV = np.asarray(BV, dtype=np.float64)
    d, r = BK.shape
    ri = refs[np.asarray(idx)]
    Kh = np.asarray(mu_k, dtype=np.float64)[None, :] + ri[:, :d] + cds[:, :r] @ BK.T
    Vh = np.asarray(mu_v, dtype=np.float64)[None, :] + ri[:, d:] + cds[:, r:] @ BV.T
    return Kh, Vh


def attention(q, K, V, scale: float):
    """Textbook softmax attention of one query over T keys/values (float64).

    s = scale * K q; out = sum_t softmax(s)_t V_t; lse = log sum_t exp(s_t).  T = 0 gives out = 0 and
    lse = -inf (softmax over an empty set is undefined; the library returns the same).
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(V.shape[1]), -np.inf
    s = scale * (K @ q)
    m = np.max(s)
    e = np.exp(s - m)
    L = np.sum(e)
    return (e @ V) / L, m + np.log(L)


def decode(q, mu, refs, idx, cds, BK, BV, dtype: str, scale: float | None = None, rounded: bool = True):
    """GQA decode attention over one sequence's compressed cache, rebuilt explicitly.

    q: [H_q, d]; mu: [H_kv, 2, d]; refs[h]: [n_ref, 2d]; idx[h]: [T]; cds[h]: [T, 2r];
    BK/BV: [H_kv, d, r] (stored values).  Query head h reads kv head h // (H_q / H_kv).
    Returns (out [H_q, d] rounded to S (``rounded=False``: exact float64), lse [H_q] float64).
    """
    q = np.asarray(q, dtype=np.float64)
    Hq, d = q.shape
    Hkv = len(refs)
    G = Hq // Hkv
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.zeros((Hq, d))
    lse = np.zeros(Hq)
    for g in range(Hkv):
        Kh, Vh = reconstruct(mu[g][0], mu[g][1], refs[g], idx[g], cds[g], BK[g], BV[g])
        for hq in range(g * G, (g + 1) * G):
            out[hq], lse[hq] = attention(q[hq], Kh, Vh, sc)
    return (round_to_storage(out, dtype) if rounded else out), lse


def decode_sparse(q, mu, refs, idx, cds, BK, BV, tokens, dtype: str, scale: float | None = None,
                  rounded: bool = True):
    """Decode attention over a selected subset of one sequence's cached tokens (summary (en) §3, "Sparse-vLLM
    Integration": only the tokens that the sparse attention keeps are reconstructed, on demand).

    Same arguments as ``decode`` plus ``tokens``: the selected positions (any order; a repeated position is
    attended twice).  Each kv head's K^ and V^ are rebuilt for the listed positions only and every query head
    of its group attends over exactly those rows.  An empty list gives out = 0, lse = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    Hq, d = q.shape
    Hkv = len(refs)
    G = Hq // Hkv
    sel = np.asarray(tokens, dtype=np.int64)
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.zeros((Hq, d))
    lse = np.zeros(Hq)
    for g in range(Hkv):
        Kh, Vh = reconstruct(mu[g][0], mu[g][1], refs[g], np.asarray(idx[g])[sel], np.asarray(cds[g])[sel], BK[g],
                             BV[g])
        for hq in range(g * G, (g + 1) * G):
            out[hq], lse[hq] = attention(q[hq], Kh, Vh, sc)
    return (round_to_storage(out, dtype) if rounded else out), lse


# --------------------------------------------------------------------------------------------------
# Closed-form sizes of the compressed layout (checked against the library's size queries).
# --------------------------------------------------------------------------------------------------
def compressed_bytes_per_token(d: int, r: int, R: int, elem: int) -> float:
    """Bytes per token per kv head of the compressed cache: codes 2r*elem + index 4 + one 2d*elem ref per R."""
    return 2 * r * elem + 4 + 2 * d * elem / R


def compressed_ratio(d: int, r: int, R: int, elem: int) -> float:
    """Compressed bytes over raw K+V bytes (2d*elem per token per kv head)."""
    return compressed_bytes_per_token(d, r, R, elem) / (2 * d * elem)


def raw_kv_bytes(layers: int, kv_heads: int, head_dim: int, tokens: int, batch: int, elem: int) -> int:
    """Raw KV-cache bytes: K and V, every layer, kv head and token."""
    return layers * kv_heads * head_dim * 2 * elem * tokens * batch
