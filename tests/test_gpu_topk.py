"""GPU parity of the pages' own retrieval (deltakv_compress_topk / deltakv_decode_attention_topk) against the
oracle: the k references nearest by L2 distance, the residual against their mean.

The tensor-core search ranks 2<x~, r~_j> - |r~_j|^2 in fp32 with 6-bit column tags; the GPU's slots must equal the
oracle's exact fp64 choice (ascending ordinals, -1 in unfilled slots) except for references inside the near-tie
band of the oracle's k-th best.  Codes are compared with the oracle's exact code for the GPU's slots, decode with
the oracle's explicit rebuild over the GPU's compressed state (bf16 tolerance 2e-2 max-abs, 1e-2 normwise).
"""
import numpy as np
import pytest

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


CASES = [
    (2, dict(seq_len=4000, num_kv_heads=2, num_q_heads=8), [4000, 1700, 30]),       # r = 32, G = 4
    (4, dict(seq_len=4000, num_kv_heads=2, num_q_heads=8), [4000, 60, 999]),         # first tokens see < 4 refs
    (2, dict(seq_len=3000, num_kv_heads=2, num_q_heads=8, rank=64), [3000, 1234]),   # r = 64
    (4, dict(seq_len=3000, num_kv_heads=2, num_q_heads=16), [3000, 777]),            # G = 8
    (2, dict(seq_len=5000, num_kv_heads=2, num_q_heads=8, ref_stride=32), [5000]),   # R = 32
    (1, dict(seq_len=3000, num_kv_heads=2, num_q_heads=8), [3000, 500]),             # L2 top-1
]


@pytest.mark.parametrize("k,over,lens", CASES)
def test_topk_compress_and_decode(k, over, lens):
    w = synth.workload(1, **over)
    L = C.make_layer(w, lens)
    cache = C.gpu_compress_topk(L, k)
    C.assert_compress_ok(C.compare_compress_topk(L, cache, k), w.dtype)
    q = _queries(w, len(lens), seed=12)
    out, lse = C.gpu_decode_topk(L, cache, q, k)
    for s in range(len(lens)):
        ref, rl = C.oracle_decode_topk_from_cache(L, cache, s, q[s].double().numpy())
        C.assert_out_close(out[s], ref, lse[s], rl, w.dtype)


def test_topk_chunked_appends():
    w = synth.workload(1, seq_len=2100, num_kv_heads=2, num_q_heads=8)
    L = C.make_layer(w, [2100, 300])
    schedule = [[(0, 0, 1500), (1, 0, 1)], [(0, 1500, 1501), (1, 1, 64)], [(0, 1501, 2100), (1, 64, 300)]]
    cache = C.gpu_compress_topk(L, 2, schedule=schedule)
    C.assert_compress_ok(C.compare_compress_topk(L, cache, 2), w.dtype)
