"""Helpers shared by the GPU parity tests: build seeded inputs, run the library, read the paged cache back
into per-(sequence, kv head) arrays, run the oracle on the same inputs and compare.

Tolerances (both must hold where two are given):
  refs (centred reference rows)  bit-exact
  ref_idx                        exact, except tokens whose oracle top-2 cosine gap is inside the fp32
                                 accumulation band eps_t = 2^-14 |x~_t| (bf16) / 2^-18 |x~_t| (fp32); there
                                 the GPU's j must score within eps_t of the best (counted, <= 0.1%)
  codes, decode out (bf16)       max-abs <= 2e-2 and normwise relative <= 1e-2 against the oracle's exact
                                 value (codes recomputed at the GPU's index)
  codes, decode out (fp32)       normwise relative <= 1e-5
  lse                            abs <= 1e-3 (bf16) / 1e-5 relative (fp32)
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

import oracle.deltakv_oracle as O
from residual_kv_cache_delta_b200 import deltakv as D
from residual_kv_cache_delta_b200 import synth

BAND = {"bf16": 2.0**-14, "f32": 2.0**-18}


def shape_of(w: synth.Workload, q4: bool = False) -> D.Shape:
    return D.Shape(w.num_q_heads, w.num_kv_heads, w.head_dim, w.rank, w.ref_stride, w.torch_dtype, q4=q4)


def unpack_q4(codes: torch.Tensor, R: int, r: int):
    """The 4-bit cache layout read back on the host: codes uint8 [nb, H, R*(r+4)] -> (levels int8 [nb, H, R, 2r],
    scales float64 [nb, H, R, 2]).  Nibble k of a little-endian 32-bit word holds code 2k and nibble k + 4 holds
    code 2k + 1 (two's complement), words in code order, the K half then the V half."""
    c = codes.cpu().numpy()
    nb, H = c.shape[:2]
    rows = np.ascontiguousarray(c[:, :, :R * r]).reshape(nb, H, R, r // 4, 4).view(np.uint32)[..., 0]
    q = np.zeros((nb, H, R, 2 * r), dtype=np.int8)
    for k in range(4):
        lo = (rows >> (4 * k)) & 15
        hi = (rows >> (4 * k + 16)) & 15
        q[..., 2 * k::8] = np.where(lo >= 8, lo.astype(np.int16) - 16, lo).astype(np.int8)
        q[..., 2 * k + 1::8] = np.where(hi >= 8, hi.astype(np.int16) - 16, hi).astype(np.int8)
    sc = torch.from_numpy(np.ascontiguousarray(c[:, :, R * r:])).view(torch.bfloat16).reshape(nb, H, R, 2)
    return q, sc.double().numpy()


@dataclass
class Layer:
    w: synth.Workload
    lens: list
    mu: torch.Tensor        # [H, 2, d] fp32 (cpu)
    basis: torch.Tensor     # [H, 2, d, r] storage (cpu)
    k: list = field(default_factory=list)  # per seq [T, H, d] storage (cpu)
    v: list = field(default_factory=list)
    bt: np.ndarray = None
    num_blocks: int = 0


def make_layer(w: synth.Workload, lens, layer: int = 0, extra_blocks: int = 0, paged_random=None) -> Layer:
    mu, basis = synth.params(w, layer)
    L = Layer(w, [int(x) for x in lens], mu, basis)
    for s, T in enumerate(L.lens):
        k, v = synth.kv_tokens(w, layer, s, 0, T)
        L.k.append(k)
        L.v.append(v)
    wp = w if paged_random is None else synth.dataclasses.replace(w, paged_random=paged_random)
    L.bt, nb = synth.block_tables(wp, np.array(L.lens), extra_tokens=0)
    L.num_blocks = nb + extra_blocks
    return L


def gpu_compress(L: Layer, schedule=None, cache=None, device="cuda", q4=False):
    """Run deltakv_compress over ``schedule``: a list of calls, each a list of (seq, start, end) ranges."""
    w = L.w
    shape = shape_of(w, q4)
    if cache is None:
        cache = D.alloc_cache(shape, L.num_blocks, device)
    if schedule is None:
        schedule = [[(s, 0, T) for s, T in enumerate(L.lens)]]
    bt_full = torch.from_numpy(L.bt).to(device)
    max_ctx = max(L.lens) if L.lens else 0
    max_ctx = max(max_ctx, 1)
    for call in schedule:
        seqs = [c for c in call if c[2] > c[1]]
        if not seqs:
            continue
        k = torch.cat([L.k[s][a:b] for s, a, b in seqs]).to(device)
        v = torch.cat([L.v[s][a:b] for s, a, b in seqs]).to(device)
        n = [b - a for _, a, b in seqs]
        cu = torch.tensor(np.concatenate([[0], np.cumsum(n)]), dtype=torch.int32, device=device)
        sp = torch.tensor([a for _, a, _ in seqs], dtype=torch.int32, device=device)
        bt = bt_full[[s for s, _, _ in seqs]].contiguous()
        ws = D.alloc_workspace(D.compress_workspace(shape, len(seqs), k.shape[0], max(n), max_ctx), device)
        D.deltakv_compress(shape, L.mu.to(device), L.basis.to(device), cache, k, v, cu, sp, bt, max(n), max_ctx, ws)
    torch.cuda.synchronize()
    return cache


def read_back(L: Layer, cache: D.Cache, s: int):
    """Per-sequence dense views of the paged cache: refs [H, n_ref, 2d], idx [H, T], codes [H, T, 2r] (float64)."""
    w = L.w
    T, R = L.lens[s], w.ref_stride
    nb = -(-T // R)
    blocks = torch.from_numpy(L.bt[s, :nb].astype(np.int64)).to(cache.codes.device)
    codes = cache.codes[blocks].permute(1, 0, 2, 3).reshape(w.num_kv_heads, nb * R, -1)[:, :T]
    idx = cache.ref_idx[blocks].permute(1, 0, 2).reshape(w.num_kv_heads, nb * R)[:, :T]
    refs = cache.refs[blocks].permute(1, 0, 2, 3).reshape(w.num_kv_heads, nb, -1)
    return (refs.double().cpu().numpy(), idx.long().cpu().numpy(), codes.double().cpu().numpy())


def oracle_compress(L: Layer, s: int, h: int):
    w = L.w
    k = L.k[s][:, h].double().numpy()
    v = L.v[s][:, h].double().numpy()
    return O.compress(k, v, L.mu[h, 0].numpy(), L.mu[h, 1].numpy(), L.basis[h, 0].double().numpy(),
                      L.basis[h, 1].double().numpy(), w.ref_stride, w.dtype)


@dataclass
class CompressReport:
    tokens: int = 0
    idx_mismatch: int = 0
    idx_band_ok: int = 0
    code_maxabs: float = 0.0
    code_num: float = 0.0
    code_den: float = 0.0
    code_bits_equal: int = 0
    code_total: int = 0

    @property
    def code_rel(self) -> float:
        return math.sqrt(self.code_num / max(self.code_den, 1e-300))


def compare_compress(L: Layer, cache: D.Cache, seqs=None, heads=None, token_sample=None, rep=None):
    """Compare the GPU cache with the oracle for the given sequences / heads (all by default).

    token_sample: optional int; compare only that many seeded random tokens per (seq, head) (plus all refs)
    """
    w = L.w
    rep = rep or CompressReport()
    seqs = range(len(L.lens)) if seqs is None else seqs
    heads = range(w.num_kv_heads) if heads is None else heads
    d = w.head_dim
    for s in seqs:
        if L.lens[s] == 0:
            continue
        g_refs, g_idx, g_codes = read_back(L, cache, s)
        for h in heads:
            refs, idx, cds, xt = oracle_compress(L, s, h)
            assert np.array_equal(g_refs[h], refs), f"refs differ (seq {s}, head {h})"
            T = L.lens[s]
            sel = np.arange(T)
            if token_sample is not None and token_sample < T:
                rng = np.random.default_rng(1000 * s + h)
                sel = np.unique(np.concatenate([rng.choice(T, token_sample, replace=False), np.arange(0, T, w.ref_stride)]))
            gi = g_idx[h][sel]
            oi = idx[sel]
            mism = np.nonzero(gi != oi)[0]
            for m in mism:
                t = int(sel[m])
                sc = O.ref_scores(xt[t], refs, t, w.ref_stride)
                assert 0 <= gi[m] < len(sc), f"GPU index {gi[m]} not visible to token {t}"
                eps = BAND[w.dtype] * np.linalg.norm(xt[t])
                assert sc.max() - sc[gi[m]] <= eps, (
                    f"seq {s} head {h} token {t}: GPU j={gi[m]} scores {sc[gi[m]]:.9g}, best j={oi[m]} "
                    f"{sc.max():.9g}, gap {sc.max() - sc[gi[m]]:.3g} > band {eps:.3g}")
                rep.idx_band_ok += 1
            rep.idx_mismatch += len(mism)
            rep.tokens += len(sel)
            exact = O.codes(xt[sel], refs, gi, L.basis[h, 0].double().numpy(), L.basis[h, 1].double().numpy(),
                            w.dtype, rounded=False)
            rounded = O.round_to_storage(exact, w.dtype)
            gc = g_codes[h][sel]
            diff = gc - exact
            rep.code_maxabs = max(rep.code_maxabs, float(np.max(np.abs(diff))) if diff.size else 0.0)
            rep.code_num += float(np.sum(diff * diff))
            rep.code_den += float(np.sum(exact * exact))
            rep.code_bits_equal += int(np.sum(gc == rounded))
            rep.code_total += gc.size
            # reference tokens: zero code, own index
            isref = (sel % w.ref_stride) == 0
            assert np.all(gc[isref] == 0) and np.array_equal(gi[isref], sel[isref] // w.ref_stride)
    return rep


def assert_compress_ok(rep: CompressReport, dtype: str):
    assert rep.idx_mismatch <= max(3, rep.tokens // 1000), f"{rep.idx_mismatch} near-tie index differences"
    if dtype == "bf16":
        assert rep.code_maxabs <= 2e-2, rep.code_maxabs
        assert rep.code_rel <= 1e-2, rep.code_rel
        assert rep.code_bits_equal >= 0.999 * rep.code_total, (rep.code_bits_equal, rep.code_total)
    else:
        assert rep.code_rel <= 1e-5, rep.code_rel


def gpu_decode(L: Layer, cache: D.Cache, q: torch.Tensor, lens=None, bt=None, device="cuda", scale=0.0, q4=False):
    """q [num_seqs, H_q, d] (cpu, storage dtype); returns (out float64 [S, H_q, d], lse [S, H_q])."""
    w = L.w
    shape = shape_of(w, q4)
    lens = L.lens if lens is None else lens
    bt = L.bt if bt is None else bt
    S = q.shape[0]
    max_ctx = max(max(lens), 1)
    out = torch.empty((S, w.num_q_heads, w.head_dim), dtype=w.torch_dtype, device=device)
    lse = torch.empty((S, w.num_q_heads), dtype=torch.float32, device=device)
    ws = D.alloc_workspace(D.decode_workspace(shape, S, max_ctx), device)
    D.deltakv_decode_attention(shape, L.mu.to(device), L.basis.to(device), cache, q.to(device).contiguous(),
                               torch.tensor(lens, dtype=torch.int32, device=device),
                               torch.from_numpy(np.ascontiguousarray(bt)).to(device), max_ctx, out, lse, ws,
                               softmax_scale=scale)
    torch.cuda.synchronize()
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


def oracle_decode_from_cache(L: Layer, cache: D.Cache, s: int, q: np.ndarray, T=None, scale=None):
    """Oracle decode over the GPU's compressed state of sequence s (first T tokens)."""
    w = L.w
    g_refs, g_idx, g_codes = read_back(L, cache, s)
    T = L.lens[s] if T is None else T
    nref = -(-T // w.ref_stride)
    refs = [g_refs[h][:nref] for h in range(w.num_kv_heads)]
    idx = [g_idx[h][:T] for h in range(w.num_kv_heads)]
    cds = [g_codes[h][:T] for h in range(w.num_kv_heads)]
    return O.decode(q, L.mu.numpy(), refs, idx, cds, L.basis[:, 0].double().numpy(), L.basis[:, 1].double().numpy(),
                    w.dtype, scale=scale, rounded=False)


def assert_out_close(out, ref, lse, ref_lse, dtype):
    diff = out - ref
    rel = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300)
    if dtype == "bf16":
        assert np.max(np.abs(diff)) <= 2e-2, np.max(np.abs(diff))
        assert rel <= 1e-2, rel
        assert np.max(np.abs(lse - ref_lse)) <= 1e-3, np.max(np.abs(lse - ref_lse))
    else:
        assert rel <= 1e-5, rel
        assert np.max(np.abs(lse - ref_lse) / np.maximum(np.abs(ref_lse), 1)) <= 1e-5


# --------------------------------------------------------------------------------------------------
# Sampled checks for full-size workloads (the oracle computes the sampled tokens one by one).
# --------------------------------------------------------------------------------------------------
def read_sampled(L: Layer, cache: D.Cache, s: int, sel: np.ndarray):
    """Reference rows [H, n_ref, 2d] of sequence s, and the index / codes of the tokens ``sel`` ([H, n])."""
    w = L.w
    R, T = w.ref_stride, L.lens[s]
    nref = -(-T // R)
    dev = cache.codes.device
    rblocks = torch.from_numpy(L.bt[s, :nref].astype(np.int64)).to(dev)
    refs = cache.refs[rblocks].permute(1, 0, 2, 3).reshape(w.num_kv_heads, nref, -1)
    tb = torch.from_numpy(L.bt[s, sel // R].astype(np.int64)).to(dev)
    to = torch.from_numpy((sel % R).astype(np.int64)).to(dev)
    idx = cache.ref_idx[tb, :, to].permute(1, 0)   # [H, n]
    cds = cache.codes[tb, :, to].permute(1, 0, 2)  # [H, n, 2r]
    return refs.double().cpu().numpy(), idx.long().cpu().numpy(), cds.double().cpu().numpy()


def check_sampled(L: Layer, cache: D.Cache, ks, vs, per_seq: int, rng, rep: CompressReport, seqs=None,
                  positions=None):
    """Every reference row (bit-exact) and a seeded token sample per (sequence, kv head): the index against the
    exact fp64 argmax over all of the token's visible references (near-tie band), the code against the oracle's
    exact code at the GPU's index.  ks / vs: per sequence raw K / V [T, H, d] (any device).  positions: per
    sequence, the tokens to check instead of the sample."""
    w = L.w
    H, R = w.num_kv_heads, w.ref_stride
    BK, BV = L.basis[:, 0].double().numpy(), L.basis[:, 1].double().numpy()
    for s in (range(len(L.lens)) if seqs is None else seqs):
        ksh = ks[s][::R].double().cpu().numpy()  # [n_ref, H, d] raw reference tokens
        vsh = vs[s][::R].double().cpu().numpy()
        Ts = L.lens[s]
        if positions is not None:
            sel = np.unique(np.asarray(positions[s], dtype=np.int64))
        else:
            extra = [t for t in (Ts - 1, Ts - 2, Ts - R, Ts - R + 1, 1, 2) if 0 <= t < Ts]
            sel = np.unique(np.concatenate([rng.choice(Ts, min(per_seq, Ts), replace=False), extra]))
        g_refs, g_sidx, g_scodes = read_sampled(L, cache, s, sel)
        ksel = ks[s][sel].double().cpu().numpy()
        vsel = vs[s][sel].double().cpu().numpy()
        for h in range(H):
            refs = np.concatenate([O.center(ksh[:, h], L.mu[h, 0].numpy(), w.dtype),
                                   O.center(vsh[:, h], L.mu[h, 1].numpy(), w.dtype)], axis=1)
            assert np.array_equal(g_refs[h], refs), f"reference rows differ (seq {s}, head {h})"
            xt = np.concatenate([O.center(ksel[:, h], L.mu[h, 0].numpy(), w.dtype),
                                 O.center(vsel[:, h], L.mu[h, 1].numpy(), w.dtype)], axis=1)
            gi = g_sidx[h]
            for n, t in enumerate(sel):
                if t % R == 0:
                    assert gi[n] == t // R
                    continue
                sc = O.ref_scores(xt[n], refs, int(t), R)
                oi = int(np.argmax(sc))  # first maximum = smallest j
                if gi[n] != oi:
                    assert 0 <= gi[n] < len(sc), (s, h, int(t), int(gi[n]))
                    eps = BAND[w.dtype] * np.linalg.norm(xt[n])
                    assert sc.max() - sc[gi[n]] <= eps, (s, h, int(t), int(gi[n]), oi)
                    rep.idx_band_ok += 1
                    rep.idx_mismatch += 1
            rep.tokens += len(sel)
            exact = O.codes(xt, refs, gi, BK[h], BV[h], w.dtype, rounded=False)
            isref = (sel % R) == 0
            exact[isref] = 0.0
            gc = g_scodes[h]
            diff = gc - exact
            rep.code_maxabs = max(rep.code_maxabs, float(np.max(np.abs(diff))))
            rep.code_num += float(np.sum(diff * diff))
            rep.code_den += float(np.sum(exact * exact))
            rep.code_bits_equal += int(np.sum(gc == O.round_to_storage(exact, w.dtype)))
            rep.code_total += gc.size
            assert np.all(gc[isref] == 0)
    return rep


def oracle_end_to_end_head(L: Layer, s: int, h: int, q: np.ndarray):
    """Oracle decode of kv head h's query-head group of sequence s from the raw K/V (the oracle's own
    compression, then the explicit rebuild).  q: [H_q, d].  Returns (out [G, d] float64, lse [G])."""
    w = L.w
    refs, idx, cds, _ = oracle_compress(L, s, h)
    G = w.group
    return O.decode(q[h * G:(h + 1) * G], L.mu[h:h + 1].numpy(), [refs], [idx], [cds],
                    L.basis[h:h + 1, 0].double().numpy(), L.basis[h:h + 1, 1].double().numpy(), w.dtype,
                    rounded=False)


# --------------------------------------------------------------------------------------------------
# Sparse decode (a caller-given token list per sequence).
# --------------------------------------------------------------------------------------------------
def gpu_decode_sparse(L: Layer, cache: D.Cache, q: torch.Tensor, lists, lens=None, device="cuda", ws_fill=None):
    """lists: per sequence an int array of positions.  Returns (out float64 [S, H_q, d], lse [S, H_q])."""
    w = L.w
    shape = shape_of(w)
    lens = L.lens if lens is None else lens
    S = q.shape[0]
    max_ctx = max(max(lens), 1)
    n = [len(x) for x in lists]
    max_sel = max(n) if n else 0
    tok = torch.tensor(np.concatenate([np.asarray(x, dtype=np.int64) for x in lists]) if sum(n) else
                       np.zeros(0), dtype=torch.int32, device=device)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(n)]), dtype=torch.int32, device=device)
    out = torch.full((S, w.num_q_heads, w.head_dim), float("nan"), dtype=w.torch_dtype, device=device)
    lse = torch.full((S, w.num_q_heads), float("nan"), dtype=torch.float32, device=device)
    ws = D.alloc_workspace(D.decode_sparse_workspace(shape, S, max_ctx, max_sel), device)
    if ws_fill is not None:
        ws.fill_(ws_fill)
    D.deltakv_decode_attention_sparse(shape, L.mu.to(device), L.basis.to(device), cache, q.to(device).contiguous(),
                                      torch.tensor(lens, dtype=torch.int32, device=device),
                                      torch.from_numpy(np.ascontiguousarray(L.bt)).to(device), tok, cu, max_sel,
                                      max_ctx, out, lse, ws)
    torch.cuda.synchronize()
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


def oracle_decode_sparse_from_cache(L: Layer, cache: D.Cache, s: int, q: np.ndarray, sel):
    """Oracle sparse decode over the GPU's compressed state of sequence s."""
    w = L.w
    g_refs, g_idx, g_codes = read_back(L, cache, s)
    return O.decode_sparse(q, L.mu.numpy(), list(g_refs), list(g_idx), list(g_codes),
                           L.basis[:, 0].double().numpy(), L.basis[:, 1].double().numpy(), sel, w.dtype,
                           rounded=False)


# --------------------------------------------------------------------------------------------------
# 4-bit codes.
# --------------------------------------------------------------------------------------------------
def read_back_q4(L: Layer, cache: D.Cache, s: int):
    """Per-sequence views of a 4-bit cache: refs [H, n_ref, 2d], idx [H, T], levels [H, T, 2r], scales [H, T, 2]."""
    w = L.w
    T, R, r = L.lens[s], w.ref_stride, w.rank
    nb = -(-T // R)
    blocks = L.bt[s, :nb].astype(np.int64)
    q, sc = unpack_q4(cache.codes, R, r)
    H = w.num_kv_heads
    lev = q[blocks].transpose(1, 0, 2, 3).reshape(H, nb * R, 2 * r)[:, :T]
    scl = sc[blocks].transpose(1, 0, 2, 3).reshape(H, nb * R, 2)[:, :T]
    bl = torch.from_numpy(blocks).to(cache.ref_idx.device)
    idx = cache.ref_idx[bl].permute(1, 0, 2).reshape(H, nb * R)[:, :T]
    refs = cache.refs[bl].permute(1, 0, 2, 3).reshape(H, nb, -1)
    return refs.double().cpu().numpy(), idx.long().cpu().numpy(), lev, scl


@dataclass
class Q4Report:
    values: int = 0
    scales: int = 0
    scales_equal: int = 0
    levels_equal: int = 0
    levels_compared: int = 0
    idx_mismatch: int = 0
    tokens: int = 0


def compare_compress_q4(L: Layer, cache: D.Cache, rep=None):
    """4-bit compress against the oracle: reference rows bit-exact; indices equal outside the near-tie band; the
    scale of each half equal to the oracle's (computed from the exact code at the GPU's index) or one bf16 step
    away; levels within one of the oracle's where the scales agree; and every dequantised code within half a step
    (plus the scale's own rounding and fp32 accumulation) of the exact code."""
    w = L.w
    r, R = w.rank, w.ref_stride
    rep = rep or Q4Report()
    for s in range(len(L.lens)):
        if L.lens[s] == 0:
            continue
        g_refs, g_idx, g_lev, g_sc = read_back_q4(L, cache, s)
        for h in range(w.num_kv_heads):
            refs, idx, _, xt = oracle_compress(L, s, h)
            assert np.array_equal(g_refs[h], refs), f"refs differ (seq {s}, head {h})"
            T = L.lens[s]
            gi = g_idx[h]
            for t in np.nonzero(gi != idx)[0]:
                sc = O.ref_scores(xt[t], refs, int(t), R)
                assert 0 <= gi[t] < len(sc)
                assert sc.max() - sc[gi[t]] <= BAND[w.dtype] * np.linalg.norm(xt[t]), (s, h, int(t))
                rep.idx_mismatch += 1
            rep.tokens += T
            exact = O.codes(xt, refs, gi, L.basis[h, 0].double().numpy(), L.basis[h, 1].double().numpy(), w.dtype,
                            rounded=False)
            exact[np.arange(T) % R == 0] = 0.0
            qo, so = O.quantize_q4(exact, r)
            gs, gq = g_sc[h], g_lev[h].astype(np.int64)
            # scales: equal or one bf16 step apart
            step = np.ldexp(1.0, np.frexp(np.maximum(so, 1e-38))[1] - 8)
            assert np.all(np.abs(gs - so) <= step * 1.0001), np.max(np.abs(gs - so) / step)
            rep.scales += gs.size
            rep.scales_equal += int(np.sum(gs == so))
            for half in range(2):
                same = gs[:, half] == so[:, half]
                a = gq[same, half * r:(half + 1) * r]
                b = qo[same, half * r:(half + 1) * r].astype(np.int64)
                assert np.all(np.abs(a - b) <= 1), np.max(np.abs(a - b))
                rep.levels_equal += int(np.sum(a == b))
                rep.levels_compared += a.size
            deq = O.dequantize_q4(gq, gs, r)
            bound = np.concatenate([np.repeat(gs[:, :1], r, 1), np.repeat(gs[:, 1:], r, 1)], 1) * (0.5 + 8 * 2.0**-8)
            err = np.abs(deq - exact)
            assert np.all(err <= bound * 1.02 + 1e-4 * max(np.max(np.abs(exact)), 1e-30)), np.max(err - bound)
            rep.values += deq.size
            isref = np.arange(T) % R == 0
            assert np.all(gq[isref] == 0) and np.all(gs[isref] == 0)
    return rep


def assert_q4_ok(rep: Q4Report):
    assert rep.idx_mismatch <= max(3, rep.tokens // 1000), rep.idx_mismatch
    assert rep.scales_equal >= 0.999 * rep.scales, (rep.scales_equal, rep.scales)
    assert rep.levels_equal >= 0.99 * rep.levels_compared, (rep.levels_equal, rep.levels_compared)


def oracle_decode_from_q4_cache(L: Layer, cache: D.Cache, s: int, q: np.ndarray):
    """Oracle decode over the GPU's 4-bit state of sequence s (codes taken as scale x level)."""
    w = L.w
    g_refs, g_idx, g_lev, g_sc = read_back_q4(L, cache, s)
    cds = [O.dequantize_q4(g_lev[h], g_sc[h], w.rank) for h in range(w.num_kv_heads)]
    return O.decode(q, L.mu.numpy(), list(g_refs), list(g_idx), cds, L.basis[:, 0].double().numpy(),
                    L.basis[:, 1].double().numpy(), w.dtype, rounded=False)


# --------------------------------------------------------------------------------------------------
# The k-nearest (L2) retrieval.
# --------------------------------------------------------------------------------------------------
L2_BAND = 2.0**-13  # x (|x~_t| max|r~| + max|r~|^2): fp32 products of bf16 operands and the 6-bit column tags


def gpu_compress_topk(L: Layer, k: int, schedule=None, device="cuda"):
    w = L.w
    shape = shape_of(w)
    cache = D.alloc_cache(shape, L.num_blocks, device, topk=k)
    if schedule is None:
        schedule = [[(s, 0, T) for s, T in enumerate(L.lens)]]
    bt_full = torch.from_numpy(L.bt).to(device)
    max_ctx = max(max(L.lens), 1)
    for call in schedule:
        seqs = [c for c in call if c[2] > c[1]]
        if not seqs:
            continue
        kk = torch.cat([L.k[s][a:b] for s, a, b in seqs]).to(device)
        vv = torch.cat([L.v[s][a:b] for s, a, b in seqs]).to(device)
        n = [b - a for _, a, b in seqs]
        cu = torch.tensor(np.concatenate([[0], np.cumsum(n)]), dtype=torch.int32, device=device)
        sp = torch.tensor([a for _, a, _ in seqs], dtype=torch.int32, device=device)
        bt = bt_full[[s for s, _, _ in seqs]].contiguous()
        ws = D.alloc_workspace(D.compress_workspace(shape, len(seqs), kk.shape[0], max(n), max_ctx), device)
        D.deltakv_compress_topk(shape, k, L.mu.to(device), L.basis.to(device), cache, kk, vv, cu, sp, bt, max(n),
                                max_ctx, ws)
    torch.cuda.synchronize()
    return cache


def read_back_topk(L: Layer, cache: D.Cache, s: int):
    """refs [H, n_ref, 2d], slots [H, T, k], codes [H, T, 2r] of sequence s (float64 / int64)."""
    w = L.w
    T, R = L.lens[s], w.ref_stride
    nb = -(-T // R)
    blocks = torch.from_numpy(L.bt[s, :nb].astype(np.int64)).to(cache.codes.device)
    codes = cache.codes[blocks].permute(1, 0, 2, 3).reshape(w.num_kv_heads, nb * R, -1)[:, :T]
    k = cache.ref_idx.shape[-1]
    idx = cache.ref_idx[blocks].permute(1, 0, 2, 3).reshape(w.num_kv_heads, nb * R, k)[:, :T]
    refs = cache.refs[blocks].permute(1, 0, 2, 3).reshape(w.num_kv_heads, nb, -1)
    return refs.double().cpu().numpy(), idx.long().cpu().numpy(), codes.double().cpu().numpy()


def compare_compress_topk(L: Layer, cache: D.Cache, k: int, rep=None):
    """Reference rows bit-exact; every token's slots equal to the oracle's k nearest (ascending, -1 padded)
    unless they differ only by references within the L2 near-tie band of the oracle's k-th best; codes against
    the oracle's exact code for the GPU's slots (bf16 tolerance)."""
    w = L.w
    R = w.ref_stride
    rep = rep or CompressReport()
    for s in range(len(L.lens)):
        T = L.lens[s]
        if T == 0:
            continue
        g_refs, g_idx, g_codes = read_back_topk(L, cache, s)
        for h in range(w.num_kv_heads):
            kk = L.k[s][:, h].double().numpy()
            vv = L.v[s][:, h].double().numpy()
            refs, idx, _, xt = O.compress_topk(kk, vv, L.mu[h, 0].numpy(), L.mu[h, 1].numpy(),
                                               L.basis[h, 0].double().numpy(), L.basis[h, 1].double().numpy(), R,
                                               w.dtype, k)
            assert np.array_equal(g_refs[h], refs), f"refs differ (seq {s}, head {h})"
            gi = g_idx[h]
            mr = np.sqrt(np.max(np.einsum("ij,ij->i", refs, refs)))
            for t in np.nonzero(np.any(gi != idx, axis=1))[0]:
                t = int(t)
                assert t % R != 0, (s, h, t)
                sc = O.l2_scores(xt[t], refs, t, R)
                eps = L2_BAND * (np.linalg.norm(xt[t]) * mr + mr * mr)
                kth = np.sort(sc)[::-1][min(k, len(sc)) - 1]
                g = gi[t]
                filled = g[g >= 0]
                assert len(filled) == min(k, len(sc)) and len(np.unique(filled)) == len(filled), (s, h, t, g)
                assert np.all(np.diff(filled) > 0) and np.all(g[len(filled):] == -1), (s, h, t, g)
                assert np.all(filled < len(sc)) and np.all(sc[filled] >= kth - eps), (s, h, t, g, idx[t])
                rep.idx_band_ok += 1
                rep.idx_mismatch += 1
            rep.tokens += T
            exact = O.codes_topk(xt, refs, gi, L.basis[h, 0].double().numpy(), L.basis[h, 1].double().numpy(),
                                 w.dtype, rounded=False)
            gc = g_codes[h]
            diff = gc - exact
            rep.code_maxabs = max(rep.code_maxabs, float(np.max(np.abs(diff))))
            rep.code_num += float(np.sum(diff * diff))
            rep.code_den += float(np.sum(exact * exact))
            rep.code_bits_equal += int(np.sum(gc == O.round_to_storage(exact, w.dtype)))
            rep.code_total += gc.size
            isref = np.arange(T) % R == 0
            assert np.all(gc[isref] == 0) and np.all(gi[isref] == (np.arange(T)[isref] // R)[:, None])
    return rep


def gpu_decode_topk(L: Layer, cache: D.Cache, q: torch.Tensor, k: int, device="cuda"):
    w = L.w
    shape = shape_of(w)
    S = q.shape[0]
    max_ctx = max(max(L.lens), 1)
    out = torch.full((S, w.num_q_heads, w.head_dim), float("nan"), dtype=w.torch_dtype, device=device)
    lse = torch.full((S, w.num_q_heads), float("nan"), dtype=torch.float32, device=device)
    ws = D.alloc_workspace(D.decode_topk_workspace(shape, k, S, max_ctx), device)
    D.deltakv_decode_attention_topk(shape, k, L.mu.to(device), L.basis.to(device), cache, q.to(device).contiguous(),
                                    torch.tensor(L.lens, dtype=torch.int32, device=device),
                                    torch.from_numpy(np.ascontiguousarray(L.bt)).to(device), max_ctx, out, lse, ws)
    torch.cuda.synchronize()
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


def oracle_decode_topk_from_cache(L: Layer, cache: D.Cache, s: int, q: np.ndarray):
    w = L.w
    g_refs, g_idx, g_codes = read_back_topk(L, cache, s)
    return O.decode_topk(q, L.mu.numpy(), list(g_refs), list(g_idx), list(g_codes), L.basis[:, 0].double().numpy(),
                         L.basis[:, 1].double().numpy(), w.dtype, rounded=False)
