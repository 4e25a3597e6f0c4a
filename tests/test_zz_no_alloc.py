"""The allocation-free decode entry point against the regular one (GPU).

deltakv_decode_attention_noalloc serves callers that may not allocate device memory: it takes its scratch
from one fixed array inside the library instead of a caller workspace.  Here it must reproduce
deltakv_decode_attention on the same compressed cache, on two calls in a row (the array keeps whatever the
previous call left in it, so the second call checks that nothing stale leaks into a result).

This file sorts last so that a run stopping at the first failure has already run every other test; it
also passes on its own in a fresh process.
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


def _close(a, b, dtype):
    diff = a - b
    rel = np.linalg.norm(diff) / max(np.linalg.norm(b), 1e-300)
    if dtype == "bf16":
        return np.max(np.abs(diff)) <= 2e-2 and rel <= 1e-2
    return rel <= 1e-5


@pytest.mark.parametrize("wl,over,lens", [
    (1, dict(seq_len=2600), [2600, 1777, 333]),     # bf16, tensor-core split kernel
    (0, dict(), [1024, 700]),                        # fp32
])
def test_noalloc_matches_workspace_entry_point_twice(wl, over, lens):
    w = synth.workload(wl, **over)
    L = C.make_layer(w, lens)
    cache = C.gpu_compress(L)
    dev = torch.device("cuda")
    shape = C.shape_of(w)
    S = len(lens)
    q = torch.from_numpy(np.random.default_rng(7).standard_normal((S, w.num_q_heads, w.head_dim))
                         .astype(np.float32)).to(w.torch_dtype).to(dev)
    ctx = torch.tensor(lens, dtype=torch.int32, device=dev)
    bt = torch.from_numpy(L.bt).to(dev)
    max_ctx = max(lens)
    mu, basis = L.mu.to(dev), L.basis.to(dev)
    assert D.decode_workspace(shape, S, max_ctx) <= D.NOALLOC_SCRATCH_BYTES

    ref_out = torch.empty((S, w.num_q_heads, w.head_dim), dtype=w.torch_dtype, device=dev)
    ref_lse = torch.empty((S, w.num_q_heads), dtype=torch.float32, device=dev)
    ws = D.alloc_workspace(D.decode_workspace(shape, S, max_ctx), dev)
    D.deltakv_decode_attention(shape, mu, basis, cache, q, ctx, bt, max_ctx, ref_out, ref_lse, ws)
    torch.cuda.synchronize()
    ref_out, ref_lse = ref_out.double().cpu().numpy(), ref_lse.double().cpu().numpy()

    for _ in range(2):
        out = torch.full((S, w.num_q_heads, w.head_dim), float("nan"), dtype=w.torch_dtype, device=dev)
        lse = torch.full((S, w.num_q_heads), float("nan"), dtype=torch.float32, device=dev)
        D.deltakv_decode_attention_noalloc(shape, mu, basis, cache, q, ctx, bt, max_ctx, out, lse)
        torch.cuda.synchronize()
        o, l = out.double().cpu().numpy(), lse.double().cpu().numpy()
        assert _close(o, ref_out, w.dtype)
        assert np.max(np.abs(l - ref_lse)) <= (1e-3 if w.dtype == "bf16" else 1e-5 * np.max(np.abs(ref_lse)))
    assert D.deltakv_get_device_error() == 0


def test_noalloc_rejects_requests_beyond_its_scratch():
    # 64 sequences of 131072 tokens need far more than the fixed scratch: refused before any launch
    w = synth.workload(1)
    shape = C.shape_of(w)
    assert D.decode_workspace(shape, 64, 131072) > D.NOALLOC_SCRATCH_BYTES
    dev = torch.device("cuda")
    cache = D.alloc_cache(shape, 1, dev)
    q = torch.zeros((64, w.num_q_heads, w.head_dim), dtype=w.torch_dtype, device=dev)
    ctx = torch.zeros(64, dtype=torch.int32, device=dev)
    bt = torch.zeros((64, 8192), dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    mu = torch.zeros((w.num_kv_heads, 2, w.head_dim), dtype=torch.float32, device=dev)
    basis = torch.zeros((w.num_kv_heads, 2, w.head_dim, w.rank), dtype=w.torch_dtype, device=dev)
    with pytest.raises(D.DeltaKVError) as e:
        D.deltakv_decode_attention_noalloc(shape, mu, basis, cache, q, ctx, bt, 131072, out, None)
    assert e.value.status == D.DKV_ERR_WORKSPACE
