"""GPU parity of the 4-bit residual codes (dtype DKV_BF16_Q4) against the oracle's quantiser and decode.

Compress writes, per token and K/V half, a bf16 scale s = RNE(max|c| / 7) and levels clip(rint(c / s)) in
two's-complement nibbles.  The oracle applies its own quantiser to the exact code at the GPU's reference index;
the GPU's code comes from fp32 tensor-core accumulation, so scales may sit one bf16 step apart and levels one
apart (counted: at least 99.9% and 99% equal), and every dequantised code must lie within half a step of the
exact one.  Decode is compared with the oracle's explicit rebuild over the GPU's 4-bit state at the bf16
tolerance (2e-2 max-abs, 1e-2 normwise).
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


SHAPES = [
    (dict(seq_len=5000, num_kv_heads=2, num_q_heads=8), [5000, 2333, 17]),               # r = 32, G = 4
    (dict(seq_len=4000, num_kv_heads=2, num_q_heads=8, rank=64), [4000, 1500]),          # r = 64
    (dict(seq_len=4000, num_kv_heads=2, num_q_heads=16), [4000, 999]),                   # G = 8
    (dict(seq_len=6000, num_kv_heads=2, num_q_heads=8, ref_stride=32), [6000, 3001]),    # R = 32
    (dict(seq_len=40000, num_kv_heads=1, num_q_heads=4), [40000]),                       # one CTA per SM
]


@pytest.mark.parametrize("over,lens", SHAPES)
def test_q4_compress_and_decode(over, lens):
    w = synth.workload(1, **over)
    L = C.make_layer(w, lens)
    cache = C.gpu_compress(L, q4=True)
    C.assert_q4_ok(C.compare_compress_q4(L, cache))
    q = _queries(w, len(lens), seed=9)
    out, lse = C.gpu_decode(L, cache, q, q4=True)
    for s in range(len(lens)):
        ref, rl = C.oracle_decode_from_q4_cache(L, cache, s, q[s].double().numpy())
        C.assert_out_close(out[s], ref, lse[s], rl, w.dtype)


def test_q4_chunked_appends():
    """Appends (a prefix, then single tokens, then the rest, two sequences interleaved) against the oracle."""
    w = synth.workload(1, seq_len=2600, num_kv_heads=2, num_q_heads=8)
    L = C.make_layer(w, [2600, 700])
    schedule = [[(0, 0, 2048), (1, 0, 1)], [(0, 2048, 2049), (1, 1, 300)], [(0, 2049, 2600), (1, 300, 700)]]
    cache = C.gpu_compress(L, schedule=schedule, q4=True)
    C.assert_q4_ok(C.compare_compress_q4(L, cache))
    q = _queries(w, 2, seed=10)
    out, lse = C.gpu_decode(L, cache, q, q4=True)
    for s in range(2):
        ref, rl = C.oracle_decode_from_q4_cache(L, cache, s, q[s].double().numpy())
        C.assert_out_close(out[s], ref, lse[s], rl, w.dtype)
