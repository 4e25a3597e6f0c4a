"""GPU parity of the sparse decode entry point (deltakv_decode_attention_sparse) against the oracle.

Each sequence attends over a caller-given list of its cached positions only (the pages' selective
reconstruction).  The oracle rebuilds exactly the listed rows from the GPU's compressed state and runs textbook
softmax attention over them.  Lists: random 1%, 10% and 100% selections (sorted), an unsorted list with repeated
positions, a single position and an empty list, over ragged contexts that span several splits; every consumer
layout of the split kernels is covered (tensor-core G >= 4 and G < 4, r = 64, the CUDA-core r = 16 and fp32 paths).
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


def _queries(w, n, seed=0):
    g = np.random.default_rng(seed).standard_normal((n, w.num_q_heads, w.head_dim)).astype(np.float32)
    return synth.to_storage(g, w.dtype)


def _lists(lens, frac, rng):
    out = []
    for T in lens:
        k = max(1, int(round(frac * T))) if T > 0 else 0
        out.append(np.sort(rng.choice(T, min(k, T), replace=False)))
    return out


def _check(L, cache, q, lists):
    out, lse = C.gpu_decode_sparse(L, cache, q, lists)
    qn = q.double().numpy()
    for s, sel in enumerate(lists):
        if len(sel) == 0:  # softmax over nothing: zero output and lse = -inf, like the oracle
            assert np.all(out[s] == 0) and np.all(lse[s] == -np.inf)
            continue
        ref, rl = C.oracle_decode_sparse_from_cache(L, cache, s, qn[s], sel)
        C.assert_out_close(out[s], ref, lse[s], rl, L.w.dtype)
    return out, lse


SHAPES = [
    (1, dict(seq_len=9000, num_kv_heads=2, num_q_heads=8)),             # bf16 tensor-core split, G = 4
    (1, dict(seq_len=6000, num_kv_heads=2, num_q_heads=16)),            # G = 8
    (1, dict(seq_len=6000, num_kv_heads=2, num_q_heads=4)),             # G = 2 (heads as MMA rows)
    (1, dict(seq_len=5000, num_kv_heads=2, num_q_heads=8, rank=64)),    # r = 64 (two swizzled tiles)
    (1, dict(seq_len=5000, num_kv_heads=2, num_q_heads=8, rank=16)),    # bf16 CUDA-core split
    (1, dict(seq_len=5000, num_kv_heads=2, num_q_heads=8, ref_stride=32)),
    (0, dict()),                                                       # fp32 CUDA-core split
]


@pytest.mark.parametrize("wl,over", SHAPES)
def test_sparse_decode_random_selections(wl, over):
    w = synth.workload(wl, **over)
    T = w.seq_len
    lens = [T, T // 2 + 37, 1]
    L = C.make_layer(w, lens)
    cache = C.gpu_compress(L)
    q = _queries(w, len(lens), seed=3)
    rng = np.random.default_rng(11)
    for frac in (0.01, 0.1, 1.0):
        _check(L, cache, q, _lists(lens, frac, rng))


def test_sparse_decode_unsorted_repeated_single_and_empty_lists():
    w = synth.workload(1, seq_len=4000, num_kv_heads=2, num_q_heads=8)
    lens = [4000, 2500, 300, 700]
    L = C.make_layer(w, lens)
    cache = C.gpu_compress(L)
    q = _queries(w, len(lens), seed=4)
    rng = np.random.default_rng(12)
    unsorted = rng.choice(4000, 900, replace=True)  # repeats count twice
    lists = [unsorted, np.array([2499]), np.zeros(0, dtype=np.int64), np.arange(700)[::-1]]
    out, lse = _check(L, cache, q, lists)
    assert np.all(out[2] == 0) and np.all(lse[2] == -np.inf)


def test_sparse_over_every_position_matches_dense_decode():
    """The full list of positions must reproduce the dense entry point within the parity tolerance."""
    w = synth.workload(1, seq_len=7000, num_kv_heads=2, num_q_heads=8)
    lens = [7000, 3333]
    L = C.make_layer(w, lens)
    cache = C.gpu_compress(L)
    q = _queries(w, len(lens), seed=5)
    out_s, lse_s = C.gpu_decode_sparse(L, cache, q, [np.arange(T) for T in lens], ws_fill=0xFF)
    out_d, lse_d = C.gpu_decode(L, cache, q)
    for s in range(len(lens)):
        C.assert_out_close(out_s[s], out_d[s], lse_s[s], lse_d[s], w.dtype)


def test_sparse_decode_full_size_llama_shape():
    """The single-layer Llama-3-8B shape at 32768 tokens, 10% of the positions selected."""
    w = synth.workload(1)
    L = C.make_layer(w, [w.seq_len])
    cache = C.gpu_compress(L)
    q = _queries(w, 1, seed=6)
    _check(L, cache, q, _lists([w.seq_len], 0.1, np.random.default_rng(13)))
