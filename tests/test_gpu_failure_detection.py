"""Failure detection without a fault (GPU).

Every pipeline wait in the kernels is bounded by global time; a wait that runs out records
DKV_DEVERR_TIMEOUT in the device error word, raises the CTA's abort flag and lets the kernel return, so the
host reads an error status and the context stays usable.  deltakv_selftest_wait_timeout runs that same wait
loop, with a short limit, on an mbarrier phase that nothing completes (no arrival is ever made, no copy is in
flight).  Nothing faults, traps or hangs: the wait ends after its limit.
"""
import numpy as np
import pytest
import torch

from residual_kv_cache_delta_b200 import deltakv as D
from residual_kv_cache_delta_b200 import synth

import _cases as C  # noqa: E402

pytestmark = pytest.mark.gpu

DEVERR_TIMEOUT = 4


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from residual_kv_cache_delta_b200 import build
    build.build()
    D.load_library()


@pytest.mark.parametrize("limit_ns", [20_000, 2_000_000])
def test_wait_runs_out_and_the_context_stays_usable(limit_ns):
    assert D.deltakv_get_device_error() == 0
    res = torch.full((2,), -1, dtype=torch.int64, device="cuda")
    D.deltakv_selftest_wait_timeout(limit_ns, res)
    torch.cuda.synchronize()
    done, waited = res.cpu().tolist()
    assert done == 0                       # the phase never completes
    assert waited >= limit_ns              # the wait lasted its limit ...
    assert waited < limit_ns + 50_000_000  # ... and then ended
    assert D.deltakv_get_device_error() == DEVERR_TIMEOUT
    assert D.deltakv_get_device_error() == 0  # read and cleared
    # the context is usable: compress and decode right after match the oracle
    w = synth.workload(0)
    L = C.make_layer(w, [w.seq_len])
    cache = C.gpu_compress(L)
    C.assert_compress_ok(C.compare_compress(L, cache), "f32")
    q = synth.queries(w, 0, 0)
    out, lse = C.gpu_decode(L, cache, q[:1])
    ref, rl = C.oracle_decode_from_cache(L, cache, 0, q[0].double().numpy())
    C.assert_out_close(out[0], ref, lse[0], rl, "f32")
    assert D.deltakv_get_device_error() == 0
