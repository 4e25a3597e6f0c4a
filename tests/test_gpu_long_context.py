"""GPU parity at full size on the two large workloads:
  - the long-context batch: 4 sequences x 131072 tokens, R = 32, r = 32, 1024 clusters with recurrence period
    up to 99991 tokens (references up to 4096 per sequence, many decode splits);
  - the paged serving mix: 64 sequences with log-uniform lengths in [4096, 131072] (about 2.3 M tokens), 16-token
    blocks at a random permutation of the pool.

The whole workload runs on the GPU as one compress call over the batch and one decode step.  The oracle then
checks what it can compute one by one:
  - every reference row of every (sequence, kv head), bit-exact;
  - the reference index and code of a seeded sample of tokens per (sequence, kv head), against the exact
    fp64 argmax over all of that token's visible references (near-tie band as in the other parity tests);
  - the decode output of two sequences (the first and the last) over their whole compressed context.
"""
import numpy as np
import pytest
import torch

import oracle.deltakv_oracle as O
from residual_kv_cache_delta_b200 import deltakv as D
from residual_kv_cache_delta_b200 import synth

import _cases as C  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from residual_kv_cache_delta_b200 import build
    build.build()
    D.load_library()
    yield
    assert D.deltakv_get_device_error() == 0


def _read_sampled(L, cache, s, sel):
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


@pytest.mark.parametrize("wl,per_seq", [(3, 192), (4, 24)])
def test_large_workload_full_size_sampled(wl, per_seq):
    w = synth.workload(wl)
    B, H, R, d = w.batch, w.num_kv_heads, w.ref_stride, w.head_dim
    lens = [int(x) for x in synth.seq_lengths(w)] if w.ragged else [w.seq_len] * B
    T = max(lens)
    dev = torch.device("cuda")
    shape = C.shape_of(w)
    mu, basis = synth.params(w, 0)
    ks, vs = [], []
    for s in range(B):
        k, v = synth.kv_tokens(w, 0, s, 0, lens[s], backend="torch", device=dev)
        ks.append(k)
        vs.append(v)
    kk, vv = torch.cat(ks), torch.cat(vs)
    total = int(sum(lens))
    bt, nb = synth.block_tables(w, np.array(lens))
    cache = D.alloc_cache(shape, nb, dev)
    btd = torch.from_numpy(bt).to(dev)
    ws = D.alloc_workspace(D.compress_workspace(shape, B, total, T, T), dev)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
    D.deltakv_compress(shape, mu.to(dev), basis.to(dev), cache, kk, vv, cu, torch.zeros(B, dtype=torch.int32, device=dev),
                       btd, T, T, ws)
    torch.cuda.synchronize()
    assert D.deltakv_get_device_error() == 0

    L = C.Layer(w, lens, mu, basis)
    L.bt, L.num_blocks = bt, nb
    rep = C.CompressReport()
    rng = np.random.default_rng(31)
    BK, BV = basis[:, 0].double().numpy(), basis[:, 1].double().numpy()
    for s in range(B):
        ksh = ks[s][::R].double().cpu().numpy()  # [n_ref, H, d] raw reference tokens
        vsh = vs[s][::R].double().cpu().numpy()
        Ts = lens[s]
        sel = np.unique(np.concatenate([rng.choice(Ts, per_seq, replace=False), [Ts - 1, Ts - 2, Ts - R, Ts - R + 1, 1, 2]]))
        g_refs, g_sidx, g_scodes = _read_sampled(L, cache, s, sel)
        ksel = ks[s][sel].double().cpu().numpy()
        vsel = vs[s][sel].double().cpu().numpy()
        for h in range(H):
            refs = np.concatenate([O.center(ksh[:, h], mu[h, 0].numpy(), w.dtype),
                                   O.center(vsh[:, h], mu[h, 1].numpy(), w.dtype)], axis=1)
            assert np.array_equal(g_refs[h], refs), f"reference rows differ (seq {s}, head {h})"
            xt = np.concatenate([O.center(ksel[:, h], mu[h, 0].numpy(), w.dtype),
                                 O.center(vsel[:, h], mu[h, 1].numpy(), w.dtype)], axis=1)
            gi = g_sidx[h]
            for n, t in enumerate(sel):
                if t % R == 0:
                    assert gi[n] == t // R
                    continue
                sc = O.ref_scores(xt[n], refs, int(t), R)
                oi = int(np.argmax(sc))  # first maximum = smallest j
                if gi[n] != oi:
                    assert 0 <= gi[n] < len(sc)
                    eps = C.BAND[w.dtype] * np.linalg.norm(xt[n])
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
    C.assert_compress_ok(rep, w.dtype)

    # one decode step for the batch; the oracle checks two sequences over their whole context
    q = torch.from_numpy(np.random.default_rng(5).standard_normal((B, w.num_q_heads, d)).astype(np.float32))
    q = synth.to_storage(q.numpy(), w.dtype)
    out, lse = C.gpu_decode(L, cache, q)
    for s in (0, B - 1):
        ref, rl = C.oracle_decode_from_cache(L, cache, s, q[s].double().numpy())
        C.assert_out_close(out[s], ref, lse[s], rl, w.dtype)
