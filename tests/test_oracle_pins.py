"""Pins of the CPU oracle to things other than itself (no GPU).

Each pin checks the oracle against a library routine, exact rational arithmetic, a closed form, an
identity the mathematics fixes, or a figure printed on the DeltaKV summary pages.  The mutation tests
at the end plant plausible mistakes in a copy of the oracle and check that some pin catches each one.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle.deltakv_oracle as O
from residual_kv_cache_delta_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "paper_figures.json")


# ------------------------------------------------------------------------------------------------
# Storage rounding pinned to torch's and NumPy's own conversions.
# ------------------------------------------------------------------------------------------------
def _bit_sweep_f32(n=200000, seed=0):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)
    # force ties (lower 16 bits = 0x8000), near-ties, subnormals and values next to the bf16 maximum
    bits[:5000] = (bits[:5000] & 0xFFFF0000) | 0x8000
    bits[5000:10000] = (bits[5000:10000] & 0xFFFF0000) | 0x7FFF
    bits[10000:12000] = bits[10000:12000] & 0x807FFFFF
    bits[12000:12010] = np.array([0x7F7F8000, 0x7F7FFFFF, 0xFF7F8000, 0x7F7F7FFF, 0x00000000, 0x80000000,
                                  0x00008000, 0x00018000, 0x3F808000, 0x3F818000], dtype=np.uint32)
    x = bits.view(np.float32)
    return x[np.isfinite(x)]


def check_bf16_rounding(rnd=O.round_to_storage):
    x = _bit_sweep_f32()
    ours = rnd(x.astype(np.float64), "bf16")
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).to(torch.float64).numpy()
    return np.array_equal(ours, ref, equal_nan=True)


def test_bf16_rounding_matches_torch():
    assert check_bf16_rounding()


def test_f32_rounding_matches_numpy():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(100000) * np.exp(rng.uniform(-80, 80, 100000))
    x = np.concatenate([x, [0.0, -0.0, 1e-45, 3e-39, 3.4e38, 3.4028235677973366e38]])
    with np.errstate(over="ignore"):
        ref = x.astype(np.float32).astype(np.float64)
    assert np.array_equal(O.round_to_storage(x, "f32"), ref)


def test_center_matches_torch_fp32_sub_then_bf16():
    rng = np.random.default_rng(2)
    x = torch.from_numpy(rng.standard_normal((64, 128)).astype(np.float32) * 8).to(torch.bfloat16)
    mu = torch.from_numpy(rng.standard_normal(128).astype(np.float32) * 3)
    ref = (x.float() - mu).to(torch.bfloat16).double().numpy()
    assert np.array_equal(O.center(x.double().numpy(), mu.numpy(), "bf16"), ref)


# ------------------------------------------------------------------------------------------------
# Search pinned to an exact-rational brute force (cosine compared without rounding).
# ------------------------------------------------------------------------------------------------
def _cos_greater(da, na, db, nb):
    """True iff da/sqrt(na) > db/sqrt(nb) exactly (Fractions); a zero norm scores 0."""
    sa = Fraction(0) if na == 0 else None
    sb = Fraction(0) if nb == 0 else None
    if sa is not None and sb is not None:
        return False
    if sa is not None:  # 0 > db/sqrt(nb)  <=>  db < 0
        return db < 0
    if sb is not None:
        return da > 0
    if (da >= 0) != (db >= 0):
        return da >= 0 and not (da == 0 and db == 0)
    if da >= 0:
        return da * da * nb > db * db * na
    return da * da * nb < db * db * na


def brute_force_idx(xt, refs, positions, R):
    xs = [[Fraction(float(v)) for v in row] for row in xt]
    rs = [[Fraction(float(v)) for v in row] for row in refs]
    nn = [sum(v * v for v in r) for r in rs]
    out = []
    for row, t in zip(xs, positions):
        t = int(t)
        if t % R == 0:
            out.append(t // R)
            continue
        best, bd, bn = None, None, None
        for j in range(len(rs)):
            if j * R >= t:
                break
            dj = sum(a * b for a, b in zip(row, rs[j]))
            if best is None or _cos_greater(dj, nn[j], bd, bn):
                best, bd, bn = j, dj, nn[j]
        out.append(best)
    return np.array(out)


def _tiny_case(seed, T=64, d=8, R=4):
    rng = np.random.default_rng(seed)
    x = O.round_to_storage(rng.standard_normal((T, 2 * d)) * 2, "bf16")
    pos = np.arange(T)
    refs = x[pos % R == 0].copy()
    # degenerate cases: a duplicated reference (exact tie), a zero-norm reference, a zero token
    refs[5] = refs[2]
    refs[7] = 0.0
    x[pos % R == 0] = refs
    x[33] = 0.0
    return x, refs, pos


def check_search_brute_force(search=O.search):
    for seed in range(4):
        x, refs, pos = _tiny_case(seed)
        if not np.array_equal(search(x, refs, pos, 4), brute_force_idx(x, refs, pos, 4)):
            return False
    return True


def test_search_matches_exact_rational_brute_force():
    assert check_search_brute_force()


def test_search_exact_tie_goes_to_smallest_j():
    x, refs, pos = _tiny_case(0)
    t = 6 * 4 + 1  # sees refs 0..6; make it point exactly along refs[2] == refs[5]
    x[t] = refs[2] * 3
    idx = O.search(x, refs, pos, 4)
    assert idx[t] == 2


def _exact_cos(row, ref):
    """<row, ref> / |ref| from exact rational dot products, rounded once to float64 (0 for a zero ref)."""
    xs = [Fraction(float(v)) for v in row]
    rs = [Fraction(float(v)) for v in ref]
    nn = sum(v * v for v in rs)
    if nn == 0:
        return 0.0
    return float(sum(a * b for a, b in zip(xs, rs))) / math.sqrt(float(nn))


def check_ref_scores(ref_scores=O.ref_scores):
    """ref_scores (the per-token score row the full-size parity tests take their argmax from) against exact
    arithmetic: one score per visible reference (j*R < t, so ceil(t/R) of them), each equal to the exact
    cosine numerator over |r~_j| to a few ulps, and its first maximum equal to the exact-rational argmax."""
    R = 4
    for seed in range(4):
        x, refs, pos = _tiny_case(seed)
        want = brute_force_idx(x, refs, pos, R)
        for t in pos:
            t = int(t)
            if t % R == 0:
                continue
            sc = ref_scores(x[t], refs, t, R)
            if len(sc) != sum(1 for j in range(len(refs)) if j * R < t):
                return False
            ex = np.array([_exact_cos(x[t], refs[j]) for j in range(len(sc))])
            if np.max(np.abs(sc - ex)) > 1e-12 * max(1.0, float(np.max(np.abs(ex)))):
                return False
            if int(np.argmax(sc)) != want[t]:
                return False
    return True


def test_ref_scores_matches_exact_cosines_and_brute_force():
    assert check_ref_scores()


def test_ref_scores_argmax_equals_search_on_long_context_sample():
    """The full-size parity tests take argmax(ref_scores) as the oracle's index of a sampled token; on a
    2048-token sample shaped like the long-context workload (R = 32, 1024 clusters, period 99991) that must be
    the index the pinned vectorised search returns for every token."""
    w = synth.workload(3, seq_len=2048, num_kv_heads=2, num_q_heads=8)
    for h in range(w.num_kv_heads):
        kk, vv, (mk, mv, BK, BV) = _compress_head(w, h)
        refs, idx, _, xt = O.compress(kk, vv, mk, mv, BK, BV, w.ref_stride, w.dtype)
        for t in range(w.seq_len):
            if t % w.ref_stride == 0:
                continue
            sc = O.ref_scores(xt[t], refs, t, w.ref_stride)
            assert len(sc) == O.visible_refs(t, w.ref_stride)
            assert int(np.argmax(sc)) == idx[t], (h, t)


def brute_force_topk_l2(xt, refs, positions, R, k):
    """Exact-rational k-nearest by squared L2 distance; ties to the smaller j; ascending ordinals, -1 padded."""
    xs = [[Fraction(float(v)) for v in row] for row in xt]
    rs = [[Fraction(float(v)) for v in row] for row in refs]
    out = []
    for row, t in zip(xs, positions):
        t = int(t)
        if t % R == 0:
            out.append([t // R] * k)
            continue
        d2 = [(sum((a - b) ** 2 for a, b in zip(row, rs[j])), j) for j in range(len(rs)) if j * R < t]
        sel = sorted(j for _, j in sorted(d2)[:k])
        out.append(sel + [-1] * (k - len(sel)))
    return np.array(out)


def check_topk_brute_force(search_topk=O.search_topk_l2):
    for seed in range(3):
        x, refs, pos = _tiny_case(seed)
        x[41] = refs[6] * 0.5 + refs[5] * 0.5  # equidistant from refs 2 (= 5) and 6: exact ties
        for k in (1, 2, 4):
            if not np.array_equal(search_topk(x, refs, pos, 4, k), brute_force_topk_l2(x, refs, pos, 4, k)):
                return False
    return True


def test_topk_l2_matches_exact_rational_brute_force():
    assert check_topk_brute_force()


def test_topk_l2_top1_equals_cosine_search_when_norms_are_equal():
    """With every reference of the same norm, the nearest in L2 is the most cosine-similar one."""
    rng = np.random.default_rng(4)
    refs = rng.standard_normal((40, 16))
    refs /= np.linalg.norm(refs, axis=1, keepdims=True)
    R = 8
    pos = np.arange(40 * R)
    x = rng.standard_normal((len(pos), 16))
    x[pos % R == 0] = refs
    top1 = O.search_topk_l2(x, refs, pos, R, 1)[:, 0]
    assert np.array_equal(top1, O.search(x, refs, pos, R))


def check_topk_codes_linear(codes_topk=O.codes_topk):
    """c_t = x~_t B - mean_i (r~_{j_i} B) with the projections formed separately (the mean counts only the filled
    slots: a token with fewer visible references than k averages those it has)."""
    w = synth.workload(1, seq_len=700)
    kk, vv, (mk, mv, BK, BV) = _compress_head(w, 1)
    for k in (2, 4):
        refs, idx, c, xt = O.compress_topk(kk, vv, mk, mv, BK, BV, w.ref_stride, w.dtype, k)
        c = codes_topk(xt, refs, idx, BK, BV, w.dtype)
        d = w.head_dim
        P = np.concatenate([xt[:, :d] @ BK, xt[:, d:] @ BV], axis=1)
        PR = np.concatenate([refs[:, :d] @ BK, refs[:, d:] @ BV], axis=1)
        want = np.zeros_like(P)
        for t in range(len(P)):
            js = [j for j in idx[t] if j >= 0]
            want[t] = P[t] - np.mean(PR[js], axis=0)
        if np.max(np.abs(c - want)) > np.max(np.abs(want)) * 2.0**-8:
            return False
    return True


def test_topk_codes_are_the_projection_minus_the_mean_projection():
    assert check_topk_codes_linear()


def test_topk_reference_tokens_and_full_rank_decode():
    """Reference tokens keep their own ordinal in every slot and a zero code; at r = d the rebuild is exact and
    decode equals textbook attention on the raw K/V."""
    w = synth.workload(0, rank=64, num_q_heads=4)
    mu, bs = synth.params(w, 0, rank=64)
    k, v = synth.kv_tokens(w, 0, 0, 0, w.seq_len)
    q = synth.queries(w, 0, 0)[0].double().numpy()
    refs, idx, cds = [], [], []
    for h in range(w.num_kv_heads):
        rr, ii, cc, _ = O.compress_topk(k[:, h].double().numpy(), v[:, h].double().numpy(), mu[h, 0].numpy(),
                                        mu[h, 1].numpy(), bs[h, 0].double().numpy(), bs[h, 1].double().numpy(),
                                        w.ref_stride, "f32", 2)
        pos = np.arange(w.seq_len)
        isref = pos % w.ref_stride == 0
        assert np.all(ii[isref] == (pos[isref] // w.ref_stride)[:, None]) and np.all(cc[isref] == 0)
        Kh, Vh = O.reconstruct_topk(mu[h, 0].numpy(), mu[h, 1].numpy(), rr, ii, cc, bs[h, 0].double().numpy(),
                                    bs[h, 1].double().numpy())
        assert np.linalg.norm(Kh - k[:, h].double().numpy()) / np.linalg.norm(k[:, h].double().numpy()) < 1e-5
        refs.append(rr), idx.append(ii), cds.append(cc)
    out, lse = O.decode_topk(q, mu.numpy(), refs, idx, cds, bs[:, 0].double().numpy(), bs[:, 1].double().numpy(), "f32")
    for hq in range(w.num_q_heads):
        h = hq // w.group
        o_ref, l_ref = _textbook(q[hq], k[:, h].double().numpy(), v[:, h].double().numpy(), 1 / math.sqrt(w.head_dim))
        assert np.linalg.norm(out[hq] - o_ref) / np.linalg.norm(o_ref) <= 1e-5
        assert abs(lse[hq] - l_ref) <= 1e-5 * abs(l_ref)


def test_search_cluster_invariant_tiny_workload():
    """Long-range recurrence: with sigma=0.1 a token's same-cluster reference has cosine ~0.99 vs ~0 for the
    others, so whenever an earlier reference of the token's cluster exists the search must pick one."""
    w = synth.workload(0)
    for h in range(w.num_kv_heads):
        mu, bs = synth.params(w, 0, rank=w.rank)
        k, v = synth.kv_tokens(w, 0, 0, 0, w.seq_len)
        refs, idx, _, _ = O.compress(k[:, h].double().numpy(), v[:, h].double().numpy(), mu[h, 0].numpy(),
                                     mu[h, 1].numpy(), bs[h, 0].double().numpy(), bs[h, 1].double().numpy(),
                                     w.ref_stride, w.dtype)
        pos = np.arange(w.seq_len)
        cl = synth.cluster_ids(pos, w.hash_mod, w.clusters)
        ref_cl = cl[:: w.ref_stride]
        checked = 0
        for t in pos[pos % w.ref_stride != 0]:
            nvis = O.visible_refs(t, w.ref_stride)
            if np.any(ref_cl[:nvis] == cl[t]):
                assert ref_cl[idx[t]] == cl[t], t
                checked += 1
        assert checked > 500


# ------------------------------------------------------------------------------------------------
# Codes and reconstruction: zero residual for references, exactness at full rank.
# ------------------------------------------------------------------------------------------------
def _compress_head(w, h, rank=None, T=None):
    T = w.seq_len if T is None else T
    mu, bs = synth.params(w, 0, rank=rank)
    k, v = synth.kv_tokens(w, 0, 0, 0, T)
    kk, vv = k[:, h].double().numpy(), v[:, h].double().numpy()
    args = (mu[h, 0].numpy(), mu[h, 1].numpy(), bs[h, 0].double().numpy(), bs[h, 1].double().numpy())
    return kk, vv, args


def test_reference_tokens_have_zero_code():
    w = synth.workload(1, seq_len=2048)
    kk, vv, args = _compress_head(w, 3)
    refs, idx, c, _ = O.compress(kk, vv, *args, w.ref_stride, w.dtype)
    pos = np.arange(len(kk))
    assert np.all(c[pos % w.ref_stride == 0] == 0)
    assert np.array_equal(idx[pos % w.ref_stride == 0], pos[pos % w.ref_stride == 0] // w.ref_stride)
    assert np.any(c[pos % w.ref_stride != 0] != 0)


def check_full_rank_reconstruction(compress=O.compress, reconstruct=O.reconstruct):
    """At r = d the basis is square orthonormal, so mu + r~ + (x~ - r~) B B^T = mu + fp32(x - mu) = x to fp32."""
    w = synth.workload(0, rank=64)
    for h in range(w.num_kv_heads):
        kk, vv, (mk, mv, BK, BV) = _compress_head(w, h, rank=64)
        refs, idx, c, _ = compress(kk, vv, mk, mv, BK, BV, w.ref_stride, "f32")
        Kh, Vh = reconstruct(mk, mv, refs, idx, c, BK, BV)
        for a, b in ((Kh, kk), (Vh, vv)):
            if np.linalg.norm(a - b) / np.linalg.norm(b) > 1e-5:
                return False
    return True


def test_full_rank_reconstruction_is_exact():
    assert check_full_rank_reconstruction()


def test_low_rank_reconstruction_error_shrinks_with_rank():
    """Adding rank can only shrink the part of the residual that the code misses: on tokens that have an
    earlier same-cluster reference, rebuilding with rank 32 beats rank 16, which beats the reference alone."""
    errs = []
    for r in (16, 32):
        w = synth.workload(0, rank=r)
        kk, vv, (mk, mv, BK, BV) = _compress_head(w, 0, rank=r)
        refs, idx, c, _ = O.compress(kk, vv, mk, mv, BK, BV, w.ref_stride, "f32")
        pos = np.arange(len(kk))
        cl = synth.cluster_ids(pos, w.hash_mod, w.clusters)
        sel = (pos % w.ref_stride != 0) & (cl[idx * w.ref_stride] == cl)
        Kh, _ = O.reconstruct(mk, mv, refs, idx, c, BK, BV)
        K0, _ = O.reconstruct(mk, mv, refs, idx, np.zeros_like(c), BK, BV)
        errs.append(np.linalg.norm((Kh - kk)[sel]))
        e_ref = np.linalg.norm((K0 - kk)[sel])
    assert errs[1] < errs[0] < e_ref


def test_codes_equal_projection_difference():
    """Linearity of f_c: the code is the difference of the token's and the reference's projections."""
    w = synth.workload(1, seq_len=1024)
    kk, vv, (mk, mv, BK, BV) = _compress_head(w, 1)
    refs, idx, c, xt = O.compress(kk, vv, mk, mv, BK, BV, w.ref_stride, w.dtype)
    d = w.head_dim
    P = np.concatenate([xt[:, :d] @ BK, xt[:, d:] @ BV], axis=1)
    PR = np.concatenate([refs[:, :d] @ BK, refs[:, d:] @ BV], axis=1)
    want = P - PR[idx]
    # c is rounded to bf16 (relative half-ulp 2^-9) after an exact fp64 difference
    assert np.max(np.abs(c - want)) <= np.max(np.abs(want)) * 2.0**-8


# ------------------------------------------------------------------------------------------------
# Decode pinned to textbook softmax attention (torch, float64) at full rank.
# ------------------------------------------------------------------------------------------------
def _textbook(q, K, V, scale):
    qt, Kt, Vt = (torch.from_numpy(np.asarray(a, dtype=np.float64)) for a in (q, K, V))
    s = scale * (Kt @ qt)
    return (torch.softmax(s, 0) @ Vt).numpy(), torch.logsumexp(s, 0).item()


def check_decode_full_rank(decode=O.decode, compress=O.compress):
    w = synth.workload(0, rank=64, num_q_heads=4)
    mu, bs = synth.params(w, 0, rank=64)
    k, v = synth.kv_tokens(w, 0, 0, 0, w.seq_len)
    q = synth.queries(w, 0, 0)[0].double().numpy()
    refs, idx, cds = [], [], []
    for h in range(w.num_kv_heads):
        rr, ii, cc, _ = compress(k[:, h].double().numpy(), v[:, h].double().numpy(), mu[h, 0].numpy(),
                                 mu[h, 1].numpy(), bs[h, 0].double().numpy(), bs[h, 1].double().numpy(),
                                 w.ref_stride, "f32")
        refs.append(rr), idx.append(ii), cds.append(cc)
    BK = bs[:, 0].double().numpy()
    BV = bs[:, 1].double().numpy()
    out, lse = decode(q, mu.numpy(), refs, idx, cds, BK, BV, "f32")
    scale = 1 / math.sqrt(w.head_dim)
    for hq in range(w.num_q_heads):
        h = hq // w.group
        o_ref, l_ref = _textbook(q[hq], k[:, h].double().numpy(), v[:, h].double().numpy(), scale)
        if np.linalg.norm(out[hq] - o_ref) / np.linalg.norm(o_ref) > 1e-5 or abs(lse[hq] - l_ref) > 1e-5 * abs(l_ref):
            return False
    return True


def test_decode_full_rank_equals_textbook_attention():
    assert check_decode_full_rank()


def check_decode_latent_identity(decode=O.decode):
    """The oracle's decode (explicit rebuild, then attention) equals the same attention written in latent space,
    the form the decode kernels compute (DeltaKV summary (en), §3 "Reconstruction": K^_t = mu_K + r~K_idx(t) +
    cK_t B_K^T, likewise V^):
        q.K^_t = q.mu_K + q.r~K_idx(t) + (q B_K).cK_t,
        sum_t p_t V^_t = mu_V + sum_j w_j r~V_j + (sum_t p_t cV_t) B_V^T,   w_j = sum over t with idx(t) = j of p_t,
    with a low-rank basis that is not orthonormal (r < d, B_K != B_V), arbitrary reference indices and a scale
    other than 1/sqrt(d), in float64."""
    rng = np.random.default_rng(11)
    Hq, Hkv, d, r, T, n_ref = 4, 2, 16, 4, 40, 5
    q = rng.standard_normal((Hq, d))
    mu = rng.standard_normal((Hkv, 2, d))
    BK, BV = rng.standard_normal((Hkv, d, r)), rng.standard_normal((Hkv, d, r))
    refs = [rng.standard_normal((n_ref, 2 * d)) for _ in range(Hkv)]
    idx = [rng.integers(0, n_ref, T) for _ in range(Hkv)]
    cds = [rng.standard_normal((T, 2 * r)) for _ in range(Hkv)]
    scale = 0.3
    out, lse = decode(q, mu, refs, idx, cds, BK, BV, "f32", scale=scale, rounded=False)
    G = Hq // Hkv
    for hq in range(Hq):
        g, qq = hq // G, q[hq]
        s = scale * (qq @ mu[g, 0] + refs[g][idx[g], :d] @ qq + cds[g][:, :r] @ (qq @ BK[g]))
        m = s.max()
        e = np.exp(s - m)
        p = e / e.sum()
        w = np.bincount(idx[g], weights=p, minlength=n_ref)
        o = mu[g, 1] + w @ refs[g][:, d:] + (p @ cds[g][:, r:]) @ BV[g].T
        if not np.allclose(out[hq], o, rtol=1e-12, atol=1e-12) or abs(lse[hq] - (m + np.log(e.sum()))) > 1e-12 * abs(lse[hq]):
            return False
    return True


def test_decode_equals_its_latent_space_form():
    assert check_decode_latent_identity()


def check_decode_topk_latent_identity(decode_topk=O.decode_topk):
    """The k-nearest decode (explicit rebuild against the mean of a token's filled slots; summary (en) §3,
    "Residual Encoding" and "Reconstruction") equals its latent-space form, with each token's softmax weight
    spread evenly over its filled slots:
        q.K^_t = q.mu_K + (1/|J_t|) sum_{j in J_t} q.r~K_j + (q B_K).cK_t,
        sum_t p_t V^_t = mu_V + sum_j w_j r~V_j + (sum_t p_t cV_t) B_V^T,   w_j = sum over t with j in J_t of p_t/|J_t|,
    for k = 4 slots of which some are unfilled (-1), at r < d with a basis that is not orthonormal, in float64."""
    rng = np.random.default_rng(12)
    Hq, Hkv, d, r, T, n_ref, k = 4, 2, 16, 4, 40, 6, 4
    q = rng.standard_normal((Hq, d))
    mu = rng.standard_normal((Hkv, 2, d))
    BK, BV = rng.standard_normal((Hkv, d, r)), rng.standard_normal((Hkv, d, r))
    refs = [rng.standard_normal((n_ref, 2 * d)) for _ in range(Hkv)]
    idx_k = []
    for _ in range(Hkv):
        rows = []
        for _t in range(T):
            n = int(rng.integers(1, k + 1))  # filled slots, ascending ordinals, -1 after them
            rows.append(list(np.sort(rng.choice(n_ref, n, replace=False))) + [-1] * (k - n))
        idx_k.append(np.array(rows, dtype=np.int64))
    cds = [rng.standard_normal((T, 2 * r)) for _ in range(Hkv)]
    scale = 0.3
    out, lse = decode_topk(q, mu, refs, idx_k, cds, BK, BV, "f32", scale=scale, rounded=False)
    G = Hq // Hkv
    for hq in range(Hq):
        g, qq = hq // G, q[hq]
        filled = idx_k[g] >= 0
        cnt = filled.sum(axis=1)
        sref = refs[g][:, :d] @ qq
        s_mean = np.array([sref[row[row >= 0]].sum() for row in idx_k[g]]) / cnt
        s = scale * (qq @ mu[g, 0] + s_mean + cds[g][:, :r] @ (qq @ BK[g]))
        m = s.max()
        e = np.exp(s - m)
        p = e / e.sum()
        w = np.zeros(n_ref)
        for t in range(T):
            for j in idx_k[g][t][filled[t]]:
                w[j] += p[t] / cnt[t]
        o = mu[g, 1] + w @ refs[g][:, d:] + (p @ cds[g][:, r:]) @ BV[g].T
        if not np.allclose(out[hq], o, rtol=1e-12, atol=1e-12) or abs(lse[hq] - (m + np.log(e.sum()))) > 1e-12 * abs(lse[hq]):
            return False
    return True


def test_decode_topk_equals_its_latent_space_form():
    assert check_decode_topk_latent_identity()


def check_decode_sparse(decode_sparse=O.decode_sparse):
    """Sparse decode at full rank (r = d, fp32) equals textbook softmax attention (torch) over the raw K/V rows
    of exactly the listed positions, for a random subset, an unsorted list with a repeated position (counted
    twice: its row appears twice in the textbook softmax) and a single position; an empty list gives 0, -inf."""
    w = synth.workload(0, rank=64, num_q_heads=4)
    mu, bs = synth.params(w, 0, rank=64)
    k, v = synth.kv_tokens(w, 0, 0, 0, w.seq_len)
    q = synth.queries(w, 0, 0)[0].double().numpy()
    refs, idx, cds = [], [], []
    for h in range(w.num_kv_heads):
        rr, ii, cc, _ = O.compress(k[:, h].double().numpy(), v[:, h].double().numpy(), mu[h, 0].numpy(),
                                   mu[h, 1].numpy(), bs[h, 0].double().numpy(), bs[h, 1].double().numpy(),
                                   w.ref_stride, "f32")
        refs.append(rr), idx.append(ii), cds.append(cc)
    BK, BV = bs[:, 0].double().numpy(), bs[:, 1].double().numpy()
    rng = np.random.default_rng(5)
    lists = [np.sort(rng.choice(w.seq_len, 100, replace=False)), np.array([900, 3, 517, 3, 1023, 0]), np.array([77])]
    scale = 1 / math.sqrt(w.head_dim)
    for sel in lists:
        out, lse = decode_sparse(q, mu.numpy(), refs, idx, cds, BK, BV, sel, "f32")
        for hq in range(w.num_q_heads):
            h = hq // w.group
            o_ref, l_ref = _textbook(q[hq], k[sel, h].double().numpy(), v[sel, h].double().numpy(), scale)
            if np.linalg.norm(out[hq] - o_ref) / np.linalg.norm(o_ref) > 1e-5 or abs(lse[hq] - l_ref) > 1e-5 * abs(l_ref):
                return False
    out, lse = decode_sparse(q, mu.numpy(), refs, idx, cds, BK, BV, np.zeros(0, np.int64), "f32")
    return bool(np.all(out == 0) and np.all(lse == -np.inf))


def test_decode_sparse_full_rank_equals_textbook_attention_on_the_listed_rows():
    assert check_decode_sparse()


def test_decode_sparse_over_every_token_equals_dense_decode():
    w = synth.workload(1, seq_len=700, num_kv_heads=2, num_q_heads=8)
    mu, bs = synth.params(w, 0)
    k, v = synth.kv_tokens(w, 0, 0, 0, w.seq_len)
    q = synth.queries(w, 0, 0)[0].double().numpy()
    st = [O.compress(k[:, h].double().numpy(), v[:, h].double().numpy(), mu[h, 0].numpy(), mu[h, 1].numpy(),
                     bs[h, 0].double().numpy(), bs[h, 1].double().numpy(), w.ref_stride, w.dtype)
          for h in range(w.num_kv_heads)]
    args = (q, mu.numpy(), [x[0] for x in st], [x[1] for x in st], [x[2] for x in st], bs[:, 0].double().numpy(),
            bs[:, 1].double().numpy())
    dense, dl = O.decode(*args, w.dtype, rounded=False)
    perm = np.random.default_rng(0).permutation(w.seq_len)  # the order of the list does not matter
    sp, sl = O.decode_sparse(*args, perm, w.dtype, rounded=False)
    assert np.allclose(sp, dense, rtol=0, atol=1e-12) and np.allclose(sl, dl, rtol=0, atol=1e-12)


def check_q4(quantize=O.quantize_q4, dequantize=O.dequantize_q4):
    """4-bit codes: exact on inputs that are multiples of a bf16 scale; zero codes stay zero; the round-trip error
    of random codes is at most half a step plus the scale's own bf16 rounding; every level is within -7 .. 7;
    the scale is the largest magnitude over 7 rounded to bf16 (checked against torch's bf16 cast)."""
    r = 32
    rng = np.random.default_rng(8)
    # exact case: c = k * s with a bf16 step s per half and integers k in -7..7 that reach +-7
    s_true = np.array([[0.0625, 0.01171875], [1.5, 0.75]])  # bf16-representable steps
    k = rng.integers(-7, 8, size=(2, 2 * r))
    k[:, 0] = 7
    k[:, r] = -7
    c = np.concatenate([k[:, :r] * s_true[:, :1], k[:, r:] * s_true[:, 1:]], axis=1)
    q, s = quantize(c, r)
    if not (np.array_equal(q, k) and np.array_equal(s, s_true)):
        return False
    if not np.array_equal(dequantize(q, s, r), c):
        return False
    z, zs = quantize(np.zeros((3, 2 * r)), r)
    if np.any(z != 0) or np.any(zs != 0) or np.any(dequantize(z, zs, r) != 0):
        return False
    c = rng.standard_normal((500, 2 * r)) * np.exp(rng.uniform(-3, 3, (500, 1)))
    q, s = quantize(c, r)
    if q.min() < -7 or q.max() > 7:
        return False
    want = torch.tensor(np.stack([np.abs(c[:, :r]).max(1), np.abs(c[:, r:]).max(1)], 1) / 7).to(torch.bfloat16)
    if not np.array_equal(s, want.double().numpy()):
        return False
    err = np.abs(dequantize(q, s, r) - c)
    bound = np.concatenate([np.repeat(s[:, :1], r, 1), np.repeat(s[:, 1:], r, 1)], 1) * (0.5 + 7 * 2.0**-8)
    return bool(np.all(err <= bound + 1e-15))


def test_q4_quantiser_exact_cases_and_error_bound():
    assert check_q4()


def test_q4_bytes_closed_form():
    # d=128, r=32, R=16: 32 B of nibbles + 4 B of scales + 4 B index + one 512 B reference per 16 tokens
    assert O.compressed_bytes_per_token_q4(128, 32, 16, 2) == 32 + 4 + 4 + 32
    assert round(O.compressed_bytes_per_token_q4(128, 32, 16, 2) / 512, 4) == 0.1406
    pages = _figure("kv_cache_fraction_after_deltakv")["value"]
    # context only: the pages' 29% (their stride, code width and model unstated) is above this layout's 14%
    assert O.compressed_bytes_per_token_q4(128, 32, 16, 2) / 512 < pages


def test_decode_single_token_returns_its_value():
    w = synth.workload(0)
    kk, vv, (mk, mv, BK, BV) = _compress_head(w, 0, T=1)
    refs, idx, c, _ = O.compress(kk, vv, mk, mv, BK, BV, w.ref_stride, "f32")
    q = np.ones((1, w.head_dim))
    out, lse = O.decode(q, np.stack([[mk, mv]]), [refs], [idx], [c], BK[None], BV[None], "f32")
    assert np.allclose(out[0], vv[0], rtol=0, atol=1e-5)
    assert np.isclose(lse[0], q[0] @ kk[0] / math.sqrt(w.head_dim), rtol=1e-6)


def test_decode_empty_context():
    out, lse = O.attention(np.ones(4), np.zeros((0, 4)), np.zeros((0, 4)), 0.5)
    assert np.all(out == 0) and lse == -np.inf


def test_chunked_compress_equals_one_shot():
    """Appending tokens in several calls gives the same refs, indices and codes as one call (the search sees
    every earlier reference, whether stored by an earlier call or centred in this one)."""
    w = synth.workload(1, seq_len=700)
    kk, vv, args = _compress_head(w, 2)
    refs1, idx1, c1, _ = O.compress(kk, vv, *args, w.ref_stride, w.dtype)
    refs, idx, cds = None, [], []
    for a, b in ((0, 333), (333, 334), (334, 512), (512, 700)):
        refs, ii, cc, _ = O.compress(kk[a:b], vv[a:b], *args, w.ref_stride, w.dtype, start=a, prev_refs=refs)
        idx.append(ii), cds.append(cc)
    assert np.array_equal(refs, refs1)
    assert np.array_equal(np.concatenate(idx), idx1)
    assert np.array_equal(np.concatenate(cds), c1)


# ------------------------------------------------------------------------------------------------
# Closed-form sizes against the pages' printed figures.
# ------------------------------------------------------------------------------------------------
def _figure(name):
    with open(GOLDEN) as f:
        return next(x for x in json.load(f)["figures"] if x["name"] == name)


def test_raw_kv_size_matches_pages_lower_bound():
    f = _figure("full_kv_llama31_8b_ctx128k_batch8_exceeds_gb")
    m = f["model"]
    b = O.raw_kv_bytes(m["layers"], m["kv_heads"], m["head_dim"], m["tokens"], m["batch"], m["elem_bytes"])
    assert b == 137438953472  # 2^37 bytes = 137.4 GB
    assert b / 1e9 > f["value"]


def test_compressed_ratio_closed_form_and_pages_figure():
    # d=128, r=32, bf16: codes 128 B + index 4 B + one 512 B reference per R tokens, over 512 B raw
    assert math.isclose(O.compressed_ratio(128, 32, 16, 2), (128 + 4 + 32) / 512)
    assert math.isclose(O.compressed_ratio(128, 32, 32, 2), (128 + 4 + 16) / 512)
    assert round(O.compressed_ratio(128, 32, 16, 2), 4) == 0.3203
    assert round(O.compressed_ratio(128, 32, 32, 2), 4) == 0.2891
    pages = _figure("kv_cache_fraction_after_deltakv")["value"]
    # context only: the pages' 29% (with 4-bit residuals, unstated stride/width) lies between our R=32 and R=16
    assert O.compressed_ratio(128, 32, 32, 2) < pages + 0.01 and pages < O.compressed_ratio(128, 32, 16, 2)
    assert 1 - _figure("kv_cache_reduction_up_to")["value"] == pytest.approx(pages)


# ------------------------------------------------------------------------------------------------
# Planted mistakes: every one must be caught by at least one pin above.
# ------------------------------------------------------------------------------------------------
def _mut_rounding_truncates(x, dtype):
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    b = x.astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    return b.view(np.float32).astype(np.float64)


def _mut_search_includes_self(xt, refs, positions, R, chunk=4096):
    pos = np.asarray(positions)
    idx = O.search(xt, refs, pos, R)
    norms = np.linalg.norm(refs, axis=1)
    for i, t in enumerate(pos):
        if t % R:
            n = min(-(-t // R) + 1, len(refs))  # off by one: also sees the next reference
            sc = (refs[:n] @ xt[i]) / np.where(norms[:n] > 0, norms[:n], 1)
            idx[i] = int(np.argmax(sc))
    return idx


def _mut_search_raw_dot(xt, refs, positions, R, chunk=4096):
    pos = np.asarray(positions)
    sc = xt @ refs.T  # forgets to divide by the reference norm
    idx = np.zeros(len(pos), dtype=np.int64)
    for i, t in enumerate(pos):
        n = -(-t // R)
        idx[i] = t // R if t % R == 0 else int(np.argmax(sc[i, :n]))
    return idx


def _mut_search_last_max(xt, refs, positions, R, chunk=4096):
    idx = O.search(xt, refs, positions, R)
    pos = np.asarray(positions)
    for i, t in enumerate(pos):
        if t % R:
            s = O.ref_scores(xt[i], refs, t, R)
            idx[i] = len(s) - 1 - int(np.argmax(s[::-1]))  # ties to the largest j
    return idx


def _mut_ref_scores_sees_next(xt_row, refs, t, R):
    n = O.visible_refs(t, R) + 1  # off by one: also scores the reference at position ceil(t/R)*R >= t
    rr = np.asarray(refs, dtype=np.float64)[:n]
    norms = np.sqrt(np.einsum("ij,ij->i", rr, rr))
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(norms > 0, (rr @ np.asarray(xt_row, dtype=np.float64)) / norms, 0.0)


def _mut_ref_scores_raw_dot(xt_row, refs, t, R):
    rr = np.asarray(refs, dtype=np.float64)[:O.visible_refs(t, R)]
    return rr @ np.asarray(xt_row, dtype=np.float64)  # forgets the reference norm


_ORIG_CODES = O.codes


def _mut_codes_swapped_bases(xt, refs, idx, BK, BV, dtype):
    return _ORIG_CODES(xt, refs, idx, BV, BK, dtype)  # V basis used for the K half and vice versa


def _mut_reconstruct_drops_mu(mu_k, mu_v, refs, idx, cds, BK, BV):
    return O.reconstruct(np.zeros_like(mu_k), np.zeros_like(mu_v), refs, idx, cds, BK, BV)


def _mut_reconstruct_minus(mu_k, mu_v, refs, idx, cds, BK, BV):
    return O.reconstruct(mu_k, mu_v, refs, idx, -np.asarray(cds), BK, BV)


def _mut_decode_wrong_group(q, mu, refs, idx, cds, BK, BV, dtype, scale=None):
    """Maps query head h to kv head h % H_kv instead of h // (H_q / H_kv)."""
    q = np.asarray(q, dtype=np.float64)
    Hq, d = q.shape
    out, lse = np.zeros((Hq, d)), np.zeros(Hq)
    for hq in range(Hq):
        g = hq % len(refs)
        Kh, Vh = O.reconstruct(mu[g][0], mu[g][1], refs[g], idx[g], cds[g], BK[g], BV[g])
        out[hq], lse[hq] = O.attention(q[hq], Kh, Vh, 1 / math.sqrt(d))
    return O.round_to_storage(out, dtype), lse


def _mut_decode_no_scale(q, mu, refs, idx, cds, BK, BV, dtype, scale=None):
    return O.decode(q, mu, refs, idx, cds, BK, BV, dtype, scale=1.0)


def _mut_decode_sparse_shifted(q, mu, refs, idx, cds, BK, BV, tokens, dtype, scale=None, rounded=True):
    t = np.minimum(np.asarray(tokens) + 1, len(idx[0]) - 1)  # off by one: attends the next position
    return O.decode_sparse(q, mu, refs, idx, cds, BK, BV, t, dtype, scale, rounded)


def _mut_decode_sparse_dense(q, mu, refs, idx, cds, BK, BV, tokens, dtype, scale=None, rounded=True):
    if len(tokens) == 0:
        return O.decode_sparse(q, mu, refs, idx, cds, BK, BV, tokens, dtype, scale, rounded)
    return O.decode(q, mu, refs, idx, cds, BK, BV, dtype, scale, rounded)  # ignores the selection


def _mut_q4_truncates(c, r):
    q, s = O.quantize_q4(c, r)
    c = np.asarray(c, dtype=np.float64)
    for half in range(2):
        ch = c[:, half * r:(half + 1) * r]
        with np.errstate(divide="ignore", invalid="ignore"):
            qq = np.where(s[:, half:half + 1] > 0, np.clip(np.trunc(ch / s[:, half:half + 1]), -7, 7), 0)
        q[:, half * r:(half + 1) * r] = qq  # rounds toward zero instead of to nearest
    return q, s


def _mut_q4_one_scale(c, r):
    q, s = O.quantize_q4(c, r)
    s2 = np.repeat(s[:, :1], 2, axis=1)  # the K scale used for the V half too
    c = np.asarray(c, dtype=np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(s2[:, :1] > 0, np.clip(np.rint(c / s2[:, :1]), -7, 7), 0).astype(np.int8)
    return q, s2


def _mut_topk_plus_norm(xt, refs, positions, R, k):
    saved = O.l2_scores
    try:
        O.l2_scores = lambda x, rf, t, R_: saved(x, rf, t, R_) + 2 * np.einsum(
            "ij,ij->i", np.asarray(rf)[:O.visible_refs(t, R_)], np.asarray(rf)[:O.visible_refs(t, R_)])
        return O.search_topk_l2(xt, refs, positions, R, k)  # + |r|^2 instead of - |r|^2
    finally:
        O.l2_scores = saved


def _mut_topk_codes_mean_over_k(xt, refs, idx_k, BK, BV, dtype, rounded=True):
    idx_k = np.asarray(idx_k)
    filled = np.where(idx_k >= 0, idx_k, 0)
    xt = np.asarray(xt, dtype=np.float64)
    m = np.mean(np.asarray(refs, dtype=np.float64)[filled], axis=1)  # counts -1 slots as reference 0
    d = xt.shape[1] // 2
    res = xt - m
    c = np.concatenate([res[:, :d] @ BK, res[:, d:] @ BV], axis=1)
    return O.round_to_storage(c, dtype) if rounded else c


_ORIG_RECONSTRUCT = O.reconstruct


def _mut_reconstruct_swapped_bases(mu_k, mu_v, refs, idx, cds, BK, BV):
    return _ORIG_RECONSTRUCT(mu_k, mu_v, refs, idx, cds, BV, BK)  # B_V rebuilds K and B_K rebuilds V


def _mut_reconstruct_no_v_reference(mu_k, mu_v, refs, idx, cds, BK, BV):
    Kh, Vh = _ORIG_RECONSTRUCT(mu_k, mu_v, refs, idx, cds, BK, BV)
    d = Kh.shape[1]
    return Kh, Vh - np.asarray(refs, dtype=np.float64)[np.asarray(idx)][:, d:]  # drops r~V_idx


def _mut_mean_refs_counts_empty_slots(refs, idx_k):
    idx_k = np.asarray(idx_k)
    filled = np.where(idx_k >= 0, idx_k, 0)
    return np.asarray(refs, dtype=np.float64)[filled].mean(axis=1)  # -1 slots read as reference 0


def test_planted_mistakes_are_caught(monkeypatch):
    assert not check_bf16_rounding(_mut_rounding_truncates)
    assert not check_search_brute_force(_mut_search_includes_self)
    assert not check_search_brute_force(_mut_search_raw_dot)
    assert not check_search_brute_force(_mut_search_last_max)
    assert not check_ref_scores(_mut_ref_scores_sees_next)
    assert not check_ref_scores(_mut_ref_scores_raw_dot)
    assert not check_decode_sparse(_mut_decode_sparse_shifted)
    assert not check_decode_sparse(_mut_decode_sparse_dense)
    assert not check_q4(quantize=_mut_q4_truncates)
    assert not check_q4(quantize=_mut_q4_one_scale)
    assert not check_topk_brute_force(_mut_topk_plus_norm)
    assert not check_topk_codes_linear(_mut_topk_codes_mean_over_k)
    assert not check_decode_full_rank(decode=_mut_decode_no_scale)
    assert not check_decode_full_rank(decode=_mut_decode_wrong_group)
    assert not check_full_rank_reconstruction(reconstruct=_mut_reconstruct_drops_mu)
    assert not check_full_rank_reconstruction(reconstruct=_mut_reconstruct_minus)
    with monkeypatch.context() as m:
        m.setattr(O, "codes", _mut_codes_swapped_bases)
        assert not check_full_rank_reconstruction()
    with monkeypatch.context() as m:
        m.setattr(O, "mean_refs", _mut_mean_refs_counts_empty_slots)
        assert not check_decode_topk_latent_identity()
    for mut in (_mut_reconstruct_swapped_bases, _mut_reconstruct_no_v_reference):
        with monkeypatch.context() as m:
            m.setattr(O, "reconstruct", mut)
            assert not check_decode_latent_identity()
