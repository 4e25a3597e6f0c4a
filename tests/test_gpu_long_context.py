"""GPU parity at full size on the three large workloads, and at the reference cap:
  - the full decode step: 32 layers of the Llama-3-8B shape, 8 sequences x 32768 tokens (seed 2);
  - the long-context batch: 4 sequences x 131072 tokens, R = 32, r = 32, 1024 clusters with recurrence period
    up to 99991 tokens (references up to 4096 per sequence, many decode splits);
  - the paged serving mix: 64 sequences with log-uniform lengths in [4096, 131072] (about 2.7 M tokens), 16-token
    blocks at a random permutation of the pool, decoded while newly arriving 2048-token prefills are compressed
    into the same pool on a second stream;
  - one sequence of 524288 tokens (32768 references at R = 16) with G = 4 and G = 8.

Every layer runs on the GPU through the C ABI.  The oracle then checks what it can compute one by one:
  - every reference row of every (sequence, kv head), bit-exact;
  - the reference index and code of a seeded sample of tokens per (sequence, kv head), against the exact
    fp64 argmax over all of that token's visible references (near-tie band as in the other parity tests);
  - the decode output of every sequence over its whole compressed context (the oracle's explicit rebuild on the
    GPU's compressed state), and, for one kv head, end to end from the raw K/V through the oracle's own
    compression.
"""
import numpy as np
import pytest
import torch

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


def _gen(w, layer, lens, seq_ids=None, dev="cuda"):
    ks, vs = [], []
    for i, T in enumerate(lens):
        s = i if seq_ids is None else seq_ids[i]
        k, v = synth.kv_tokens(w, layer, s, 0, T, backend="torch", device=dev)
        ks.append(k)
        vs.append(v)
    return ks, vs


def _compress(shape, mu, basis, cache, ks, vs, lens, bt, dev, stream=None):
    T = max(lens)
    total = int(sum(lens))
    B = len(lens)
    ws = D.alloc_workspace(D.compress_workspace(shape, B, total, T, T), dev)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
    D.deltakv_compress(shape, mu.to(dev), basis.to(dev), cache, torch.cat(ks), torch.cat(vs), cu,
                       torch.zeros(B, dtype=torch.int32, device=dev), bt, T, T, ws, stream=stream)
    return ws


def _queries(w, B, seed):
    q = np.random.default_rng(seed).standard_normal((B, w.num_q_heads, w.head_dim)).astype(np.float32)
    return synth.to_storage(q, w.dtype)


def _check_decode(L, cache, q, out, lse, seqs):
    for s in seqs:
        ref, rl = C.oracle_decode_from_cache(L, cache, s, q[s].double().numpy())
        C.assert_out_close(out[s], ref, lse[s], rl, L.w.dtype)


def test_full_decode_step_32_layers():
    """Workload 2: every layer compressed and decoded through the library; layers 0 and 31 checked element by
    element (all reference rows, 24 sampled tokens per (sequence, kv head), decode of all 8 sequences), and
    kv head 0 of sequence 0 end to end from raw K/V."""
    w = synth.workload(2)
    B, T = w.batch, w.seq_len
    lens = [T] * B
    dev = torch.device("cuda")
    shape = C.shape_of(w)
    bt, nb = synth.block_tables(w, np.array(lens))
    btd = torch.from_numpy(bt).to(dev)
    ctx = torch.tensor(lens, dtype=torch.int32, device=dev)
    wsd = D.alloc_workspace(D.decode_workspace(shape, B, T), dev)
    rng = np.random.default_rng(2)
    for layer in range(w.layers):
        mu, basis = synth.params(w, layer)
        ks, vs = _gen(w, layer, lens)
        cache = D.alloc_cache(shape, nb, dev)
        _compress(shape, mu, basis, cache, ks, vs, lens, btd, dev)
        q = _queries(w, B, 100 + layer)
        out = torch.empty((B, w.num_q_heads, w.head_dim), dtype=w.torch_dtype, device=dev)
        lse = torch.empty((B, w.num_q_heads), dtype=torch.float32, device=dev)
        D.deltakv_decode_attention(shape, mu.to(dev), basis.to(dev), cache, q.to(dev), ctx, btd, T, out, lse, wsd)
        torch.cuda.synchronize()
        assert D.deltakv_get_device_error() == 0, layer
        if layer not in (0, w.layers - 1):
            continue
        L = C.Layer(w, lens, mu, basis)
        L.bt, L.num_blocks = bt, nb
        rep = C.check_sampled(L, cache, ks, vs, 24, rng, C.CompressReport())
        C.assert_compress_ok(rep, w.dtype)
        o, ls = out.double().cpu().numpy(), lse.double().cpu().numpy()
        _check_decode(L, cache, q, o, ls, range(B))
        if layer == 0:
            L0 = C.Layer(w, [T], mu, basis, k=[ks[0].cpu()], v=[vs[0].cpu()])
            ref, rl = C.oracle_end_to_end_head(L0, 0, 0, q[0].double().numpy())
            G = w.group
            C.assert_out_close(o[0, :G], ref, ls[0, :G], rl, w.dtype)


def test_long_context_batch_full_size():
    """Workload 3: 4 x 131072 tokens in one compress call; 192 sampled tokens per (sequence, kv head); decode of
    all four sequences."""
    w = synth.workload(3)
    B = w.batch
    lens = [w.seq_len] * B
    dev = torch.device("cuda")
    shape = C.shape_of(w)
    mu, basis = synth.params(w, 0)
    ks, vs = _gen(w, 0, lens)
    bt, nb = synth.block_tables(w, np.array(lens))
    cache = D.alloc_cache(shape, nb, dev)
    _compress(shape, mu, basis, cache, ks, vs, lens, torch.from_numpy(bt).to(dev), dev)
    torch.cuda.synchronize()
    assert D.deltakv_get_device_error() == 0
    L = C.Layer(w, lens, mu, basis)
    L.bt, L.num_blocks = bt, nb
    C.assert_compress_ok(C.check_sampled(L, cache, ks, vs, 192, np.random.default_rng(31), C.CompressReport()),
                         w.dtype)
    q = _queries(w, B, 5)
    out, lse = C.gpu_decode(L, cache, q)
    _check_decode(L, cache, q, out, lse, range(B))


@pytest.mark.parametrize("G", [4, 8])
def test_half_million_token_sequence(G):
    """One sequence of 524288 tokens at R = 16: 32768 references, the reference cap.  Their per-reference masses do
    not fit in shared memory, so the split kernel keeps them in global memory.  Llama head geometry with one kv
    head and G query heads.  Compressed through the library (every reference row and 64 sampled tokens checked),
    then decoded against the oracle's rebuild of the GPU's compressed state."""
    w = synth.workload(1, num_q_heads=G, num_kv_heads=1, seq_len=524288, seed=11)
    lens = [w.seq_len]
    dev = torch.device("cuda")
    shape = C.shape_of(w)
    mu, basis = synth.params(w, 0)
    ks, vs = _gen(w, 0, lens)
    bt, nb = synth.block_tables(w, np.array(lens))
    cache = D.alloc_cache(shape, nb, dev)
    _compress(shape, mu, basis, cache, ks, vs, lens, torch.from_numpy(bt).to(dev), dev)
    torch.cuda.synchronize()
    assert D.deltakv_get_device_error() == 0
    L = C.Layer(w, lens, mu, basis)
    L.bt, L.num_blocks = bt, nb
    C.assert_compress_ok(C.check_sampled(L, cache, ks, vs, 64, np.random.default_rng(51), C.CompressReport()),
                         w.dtype)
    del ks, vs
    q = _queries(w, 1, 7)
    out, lse = C.gpu_decode(L, cache, q)
    assert D.deltakv_get_device_error() == 0
    _check_decode(L, cache, q, out, lse, [0])


def test_small_appends_at_long_context():
    """Two sequences compressed to 131072 - 40 tokens on the tensor-core path, then 40 more tokens each in calls of
    1 to 16 tokens (the append path reads the reference rows of the whole context from the paged cache).  Every
    appended token is checked against the exact argmax over its 8192 visible references, and both sequences'
    decode against the oracle."""
    w = synth.workload(1, batch=2, seq_len=131072, seed=13)
    T = w.seq_len
    lens = [T, T]
    dev = torch.device("cuda")
    shape = C.shape_of(w)
    mu, basis = synth.params(w, 0)
    ks, vs = _gen(w, 0, lens)
    bt, nb = synth.block_tables(w, np.array(lens))
    btd = torch.from_numpy(bt).to(dev)
    cache = D.alloc_cache(shape, nb, dev)
    start = T - 40
    _compress(shape, mu, basis, cache, [k[:start] for k in ks], [v[:start] for v in vs], [start, start], btd, dev)
    sizes = ([1, 16, 3, 1, 16, 3], [16, 1, 1, 16, 5, 1])
    pos = [start, start]
    ws = D.alloc_workspace(D.compress_workspace(shape, 2, 32, 16, T), dev)
    for a, b in zip(*sizes):
        n = [a, b]
        k = torch.cat([ks[s][pos[s]:pos[s] + n[s]] for s in range(2)])
        v = torch.cat([vs[s][pos[s]:pos[s] + n[s]] for s in range(2)])
        cu = torch.tensor([0, n[0], n[0] + n[1]], dtype=torch.int32, device=dev)
        sp = torch.tensor(pos, dtype=torch.int32, device=dev)
        D.deltakv_compress(shape, mu.to(dev), basis.to(dev), cache, k, v, cu, sp, btd, max(n), T, ws)
        pos = [pos[s] + n[s] for s in range(2)]
    torch.cuda.synchronize()
    assert pos == lens and D.deltakv_get_device_error() == 0
    L = C.Layer(w, lens, mu, basis)
    L.bt, L.num_blocks = bt, nb
    appended = {s: np.arange(start, T) for s in range(2)}
    C.assert_compress_ok(C.check_sampled(L, cache, ks, vs, 0, None, C.CompressReport(), positions=appended),
                         w.dtype)
    q = _queries(w, 2, 9)
    out, lse = C.gpu_decode(L, cache, q)
    _check_decode(L, cache, q, out, lse, range(2))


def test_serving_mix_decode_with_overlapped_prefills():
    """Workload 4: the 64 prefixes are compressed in one call (24 sampled tokens per (sequence, kv head) checked).
    Then 16 steps: the 64-query decode on the main stream while a new 2048-token sequence is compressed into
    freshly mapped blocks of the same pool on a second stream.  Afterwards every prefill must match the oracle
    on every token, and the decode of every step must match it for all 64 sequences."""
    w = synth.workload(4)
    B, P, NP = w.batch, w.prefill_len, 16
    lens = [int(x) for x in synth.seq_lengths(w)]
    T = max(lens)
    dev = torch.device("cuda")
    shape = C.shape_of(w)
    mu, basis = synth.params(w, 0)
    ks, vs = _gen(w, 0, lens)
    bt, nb = synth.block_tables(w, np.array(lens + [P] * NP))  # one pool, random placement
    cache = D.alloc_cache(shape, nb, dev)
    bt_dec = torch.from_numpy(np.ascontiguousarray(bt[:B])).to(dev)
    _compress(shape, mu, basis, cache, ks, vs, lens, bt_dec, dev)
    torch.cuda.synchronize()
    assert D.deltakv_get_device_error() == 0
    L = C.Layer(w, lens, mu, basis)
    L.bt, L.num_blocks = bt[:B], nb
    C.assert_compress_ok(C.check_sampled(L, cache, ks, vs, 24, np.random.default_rng(41), C.CompressReport()),
                         w.dtype)
    del ks, vs

    # prefills: raw K/V on the host (NumPy generator) for the oracle, copied to the device once
    pre = C.Layer(w, [P] * NP, mu, basis)
    for i in range(NP):
        k, v = synth.kv_tokens(w, 0, 1000 + i, 0, P)
        pre.k.append(k)
        pre.v.append(v)
    pre.bt, pre.num_blocks = bt[B:], nb
    pk = [x.to(dev) for x in pre.k]
    pv = [x.to(dev) for x in pre.v]
    bt_pre = [torch.from_numpy(np.ascontiguousarray(bt[B + i: B + i + 1])).to(dev) for i in range(NP)]
    ws_p = D.alloc_workspace(D.compress_workspace(shape, 1, P, P, P), dev)
    cu_p = torch.tensor([0, P], dtype=torch.int32, device=dev)
    st_p = torch.zeros(1, dtype=torch.int32, device=dev)

    q = _queries(w, B, 6)
    qd = q.to(dev)
    ctx = torch.tensor(lens, dtype=torch.int32, device=dev)
    wsd = D.alloc_workspace(D.decode_workspace(shape, B, T), dev)
    outs = [torch.empty((B, w.num_q_heads, w.head_dim), dtype=w.torch_dtype, device=dev) for _ in range(NP)]
    lses = [torch.empty((B, w.num_q_heads), dtype=torch.float32, device=dev) for _ in range(NP)]
    mud, bsd = mu.to(dev), basis.to(dev)
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    for i in range(NP):
        side.wait_stream(main)
        D.deltakv_compress(shape, mud, bsd, cache, pk[i], pv[i], cu_p, st_p, bt_pre[i], P, P, ws_p, stream=side)
        D.deltakv_decode_attention(shape, mud, bsd, cache, qd, ctx, bt_dec, T, outs[i], lses[i], wsd)
        main.wait_stream(side)
    torch.cuda.synchronize()
    assert D.deltakv_get_device_error() == 0

    rep = C.compare_compress(pre, cache)
    C.assert_compress_ok(rep, w.dtype)
    o0, l0 = outs[0].double().cpu().numpy(), lses[0].double().cpu().numpy()
    _check_decode(L, cache, q, o0, l0, range(B))
    for i in range(1, NP):  # every step decodes the same cache: within the parity tolerance of step 0
        C.assert_out_close(outs[i].double().cpu().numpy(), o0, lses[i].double().cpu().numpy(), l0, w.dtype)
