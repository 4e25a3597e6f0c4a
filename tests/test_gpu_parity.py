"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same seeded inputs.

Sizes are chosen so the oracle finishes in seconds while the GPU sees several tiles and ragged tails;
the Llama-3-8B single-layer workload (32768 tokens, 8 kv heads) runs at full size.
"""
import math

import numpy as np
import pytest
import torch

import oracle.deltakv_oracle as O
from residual_kv_cache_delta_b200 import deltakv as D
from residual_kv_cache_delta_b200 import synth

import _cases as C  # noqa: E402  (tests/ is on sys.path under pytest rootdir-relative import)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from residual_kv_cache_delta_b200 import build
    build.build()
    D.load_library()
    yield
    assert D.deltakv_get_device_error() == 0


def _queries(w, n, layer=0, seed=0):
    g = np.random.default_rng(seed).standard_normal((n, w.num_q_heads, w.head_dim)).astype(np.float32)
    return synth.to_storage(g, w.dtype)


def _decode_check(L, cache, q, lens=None, bt=None):
    lens = L.lens if lens is None else lens
    out, lse = C.gpu_decode(L, cache, q, lens=lens, bt=bt)
    qn = q.double().numpy()
    for s in range(q.shape[0]):
        ref, rl = C.oracle_decode_from_cache(L, cache, s if bt is None else 0, qn[s], T=lens[s])
        C.assert_out_close(out[s], ref, lse[s], rl, L.w.dtype)
    return out, lse


# --------------------------------------------------------------------------------------------------
def test_tiny_fp32_workload_compress_and_decode():
    w = synth.workload(0)
    L = C.make_layer(w, [w.seq_len])
    cache = C.gpu_compress(L)
    rep = C.compare_compress(L, cache)
    C.assert_compress_ok(rep, "f32")
    # four decode queries against the same cache (block tables alias the same blocks)
    q = synth.queries(w, 0, 0)
    bt = np.repeat(L.bt[:1], 4, axis=0)
    out, lse = C.gpu_decode(L, cache, q, lens=[w.seq_len] * 4, bt=bt)
    for i in range(4):
        ref, rl = C.oracle_decode_from_cache(L, cache, 0, q[i].double().numpy())
        C.assert_out_close(out[i], ref, lse[i], rl, "f32")
    # end to end from raw K/V through the oracle's own compression
    st = [C.oracle_compress(L, 0, h) for h in range(w.num_kv_heads)]
    for i in range(4):
        ref, rl = O.decode(q[i].double().numpy(), L.mu.numpy(), [x[0] for x in st], [x[1] for x in st],
                           [x[2] for x in st], L.basis[:, 0].double().numpy(), L.basis[:, 1].double().numpy(), "f32",
                           rounded=False)
        C.assert_out_close(out[i], ref, lse[i], rl, "f32")


def test_full_rank_fp32_decode_equals_textbook_attention():
    w = synth.workload(0, rank=64, num_q_heads=4)
    L = C.make_layer(w, [777])
    cache = C.gpu_compress(L)
    C.assert_compress_ok(C.compare_compress(L, cache), "f32")
    q = _queries(w, 1)
    out, lse = C.gpu_decode(L, cache, q)
    k, v = L.k[0].double().numpy(), L.v[0].double().numpy()
    for hq in range(w.num_q_heads):
        h = hq // w.group
        ref, rl = O.attention(q[0, hq].double().numpy(), k[:, h], v[:, h], 1 / math.sqrt(w.head_dim))
        assert np.linalg.norm(out[0, hq] - ref) / np.linalg.norm(ref) <= 1e-5
        assert abs(lse[0, hq] - rl) <= 1e-5 * max(1, abs(rl))


def test_bf16_llama_shape_ragged_tail():
    w = synth.workload(1, seq_len=4173)  # 260 full blocks + 13 tokens; spans 17 token tiles and 3 ref tiles
    L = C.make_layer(w, [w.seq_len])
    cache = C.gpu_compress(L)
    rep = C.compare_compress(L, cache)
    C.assert_compress_ok(rep, "bf16")
    q = _queries(w, 1)
    _decode_check(L, cache, q)


def test_bf16_batch_paged_random_placement():
    w = synth.workload(4, batch=6, seq_len=3000, min_len=1, prefill_len=0)
    lens = [1, 17, 300, 2048, 2999, 1100]
    L = C.make_layer(w, lens, extra_blocks=7, paged_random=True)
    cache = C.gpu_compress(L)
    C.assert_compress_ok(C.compare_compress(L, cache), "bf16")
    _decode_check(L, cache, _queries(w, len(lens)))


def test_bf16_small_appends_match_one_shot_oracle():
    """Calls of at most 16 new tokens per sequence take the append path (search and codes on CUDA cores over the
    paged reference rows).  From an empty cache: a first call of 5 tokens, then appends of 1 to 16 tokens that
    cross reference positions, sequences that skip calls, and one larger call in between on the tensor-core path.
    The result must match the oracle's one-shot compression of each whole sequence."""
    w = synth.workload(1, seq_len=700, num_kv_heads=4, num_q_heads=16)
    lens = [700, 301, 45]
    L = C.make_layer(w, lens, extra_blocks=3, paged_random=True)
    schedule = [[(0, 0, 5), (1, 0, 16), (2, 0, 1)]]
    pos = [5, 16, 1]
    steps = [(1, 1, 1), (16, 3, 0), (2, 0, 15), (7, 16, 1), (1, 1, 1), (0, 9, 16), (16, 16, 11)]
    for k in steps:
        call = []
        for s, n in enumerate(k):
            n = min(n, lens[s] - pos[s])
            if n > 0:
                call.append((s, pos[s], pos[s] + n))
                pos[s] += n
        schedule.append(call)
    schedule.append([(0, pos[0], 600), (1, pos[1], pos[1] + 1)])  # tensor-core path
    pos[0], pos[1] = 600, pos[1] + 1
    while any(p < T for p, T in zip(pos, lens)):  # the rest in appends of up to 16
        call = []
        for s in range(3):
            n = min(16 - 5 * s, lens[s] - pos[s])
            if n > 0:
                call.append((s, pos[s], pos[s] + n))
                pos[s] += n
        schedule.append(call)
    cache = C.gpu_compress(L, schedule)
    assert D.deltakv_get_device_error() == 0
    C.assert_compress_ok(C.compare_compress(L, cache), "bf16")
    _decode_check(L, cache, _queries(w, len(lens)))


def test_bf16_chunked_appends_match_one_shot_oracle():
    w = synth.workload(1, seq_len=1500, num_kv_heads=4, num_q_heads=16)
    lens = [1500, 900]
    L = C.make_layer(w, lens)
    schedule = [[(0, 0, 700), (1, 0, 1)], [(0, 700, 701), (1, 1, 512)], [(0, 701, 1500), (1, 512, 513)],
                [(1, 513, 900)]]
    cache = C.gpu_compress(L, schedule)
    C.assert_compress_ok(C.compare_compress(L, cache), "bf16")
    _decode_check(L, cache, _queries(w, 2))


@pytest.mark.parametrize("over", [
    dict(head_dim=64, rank=16, num_q_heads=8, num_kv_heads=4),    # two K-chunks on the tensor-core path
    dict(rank=16, num_q_heads=8, num_kv_heads=8),                 # G = 1
    dict(rank=64, num_q_heads=16, num_kv_heads=4),                # 2r = 128
    dict(num_q_heads=32, num_kv_heads=4),                         # G = 8
    dict(ref_stride=32, num_q_heads=8, num_kv_heads=2),
    dict(ref_stride=64, num_q_heads=8, num_kv_heads=2),
    dict(num_q_heads=8, num_kv_heads=8),                          # G = 1, r = 32: heads as MMA rows
    dict(num_q_heads=8, num_kv_heads=4),                          # G = 2, r = 32
    dict(rank=64, num_q_heads=4, num_kv_heads=2),                 # G = 2, r = 64
])
def test_bf16_shape_variants(over):
    w = synth.workload(1, seq_len=2600, **over)
    L = C.make_layer(w, [2600, 333])
    cache = C.gpu_compress(L)
    C.assert_compress_ok(C.compare_compress(L, cache), "bf16")
    _decode_check(L, cache, _queries(w, 2))


def test_decode_persistent_items_many_sequences_ragged():
    # 40 sequences of ragged lengths: the persistent split CTAs walk several (sequence, kv head, split) items
    # each, and the splits of short sequences that start past their context are skipped by every role
    w = synth.workload(1, seq_len=4096, num_kv_heads=4, num_q_heads=16)
    rng = np.random.default_rng(11)
    lens = [int(x) for x in rng.integers(1, 4097, size=40)]
    lens[0], lens[1], lens[2] = 4096, 1, 257
    L = C.make_layer(w, lens)
    cache = C.gpu_compress(L)
    q = _queries(w, len(lens), seed=3)
    out, lse = C.gpu_decode(L, cache, q)
    qn = q.double().numpy()
    for s in sorted(set([0, 1, 2] + [int(x) for x in rng.choice(len(lens), 5, replace=False)])):
        ref, rl = C.oracle_decode_from_cache(L, cache, s, qn[s], T=lens[s])
        C.assert_out_close(out[s], ref, lse[s], rl, "bf16")


def test_decode_edge_contexts():
    w = synth.workload(1, seq_len=1000, num_kv_heads=2, num_q_heads=8)
    L = C.make_layer(w, [1000, 1000, 1000, 1000])
    cache = C.gpu_compress(L)
    q = _queries(w, 4)
    lens = [0, 1, 17, 999]  # empty, single token, ragged, all but one
    out, lse = C.gpu_decode(L, cache, q, lens=lens)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    for s in range(1, 4):
        ref, rl = C.oracle_decode_from_cache(L, cache, s, q[s].double().numpy(), T=lens[s])
        C.assert_out_close(out[s], ref, lse[s], rl, "bf16")


def test_llama3_8b_single_layer_full_size():
    w = synth.workload(1)
    L = C.make_layer(w, [w.seq_len])
    cache = C.gpu_compress(L)
    rep = C.compare_compress(L, cache)
    C.assert_compress_ok(rep, "bf16")
    _decode_check(L, cache, synth.queries(w, 0, 0))


def test_device_error_word_records_bad_block_table():
    w = synth.workload(1, seq_len=300, num_kv_heads=2, num_q_heads=8)
    L = C.make_layer(w, [300])
    L.bt = L.bt.copy()
    L.bt[0, 5] = L.num_blocks + 100  # out of range: skipped and recorded, never dereferenced
    C.gpu_compress(L)
    assert D.deltakv_get_device_error() == 1
    assert D.deltakv_get_device_error() == 0  # cleared by the read


@pytest.mark.parametrize("wl,over,lens", [
    (1, dict(seq_len=2600), [2600, 1777, 333]),  # bf16, tensor-core split kernel
    (1, dict(seq_len=2600, rank=16), [2600, 1777, 333]),  # bf16, CUDA-core split kernel
    (0, dict(), [1024, 700, 45]),                 # fp32
])
def test_decode_reads_only_valid_cache_and_workspace(wl, over, lens):
    """Unused cache slots (the tail of each sequence's last block, blocks past the context) and the whole
    workspace are filled with NaN bit patterns before the calls; decode must not let any of it reach the
    result, on repeated calls (which also meet stale shared memory left by earlier kernels)."""
    w = synth.workload(wl, **over)
    L = C.make_layer(w, lens)
    shape = C.shape_of(w)
    cache = D.alloc_cache(shape, L.num_blocks, "cuda")
    for t in (cache.codes, cache.ref_idx, cache.refs):
        t.view(torch.uint8).fill_(0xFF)
    cache = C.gpu_compress(L, cache=cache)
    q = _queries(w, len(lens))
    dev = torch.device("cuda")
    ws = D.alloc_workspace(D.decode_workspace(shape, len(lens), max(lens)), dev)
    qd, ctx, bt = q.to(dev), torch.tensor(lens, dtype=torch.int32, device=dev), torch.from_numpy(L.bt).to(dev)
    refs = [C.oracle_decode_from_cache(L, cache, s, q[s].double().numpy(), T=lens[s]) for s in range(len(lens))]
    for _ in range(3):
        ws.fill_(0xFF)
        out = torch.full((len(lens), w.num_q_heads, w.head_dim), float("nan"), dtype=w.torch_dtype, device=dev)
        lse = torch.full((len(lens), w.num_q_heads), float("nan"), dtype=torch.float32, device=dev)
        D.deltakv_decode_attention(shape, L.mu.to(dev), L.basis.to(dev), cache, qd, ctx, bt, max(lens), out, lse, ws)
        torch.cuda.synchronize()
        o, l = out.double().cpu().numpy(), lse.double().cpu().numpy()
        for s in range(len(lens)):
            C.assert_out_close(o[s], refs[s][0], l[s], refs[s][1], w.dtype)
