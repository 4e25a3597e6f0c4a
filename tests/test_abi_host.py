"""Host-side tests of the C ABI (no GPU): the library loads, exports every declared symbol, and rejects
bad arguments with a status before touching the device."""
import ctypes
import os
import re

import pytest
import torch

import oracle.deltakv_oracle as O
from residual_kv_cache_delta_b200 import build as B
from residual_kv_cache_delta_b200 import deltakv as D

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
HEADER = os.path.join(INCLUDE, "deltakv.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return D.load_library()


def declared_functions(path=HEADER):
    src = open(path).read()
    return sorted(set(re.findall(r"^(?:const char\*|dkv_status|size_t|void|int32_t)\s+(deltakv_\w+)\s*\(", src, re.M)))


def test_exports_every_declared_symbol(lib):
    from residual_kv_cache_delta_b200 import pool as P
    names = declared_functions()
    assert len(names) >= 9
    assert set(names) == set(D.EXPORTED)
    headers = sorted(f for f in os.listdir(INCLUDE) if f.endswith(".h"))
    assert headers == ["deltakv.h", "deltakv_pool.h"]
    assert set(declared_functions(os.path.join(INCLUDE, "deltakv_pool.h"))) == set(P.EXPORTED)
    for h in headers:
        for n in declared_functions(os.path.join(INCLUDE, h)):
            assert hasattr(lib, n), n


def test_status_strings(lib):
    for s in range(6):
        assert D.status_string(s) != "unknown status"
    assert D.status_string(99) == "unknown status"


BF = torch.bfloat16


@pytest.mark.parametrize("shape,status", [
    (D.Shape(32, 8, 128, 32, 16, BF), D.DKV_OK),
    (D.Shape(2, 2, 64, 16, 16, torch.float32), D.DKV_OK),
    (D.Shape(32, 8, 128, 64, 32, BF), D.DKV_OK),
    (D.Shape(64, 8, 128, 32, 64, BF), D.DKV_OK),
    (D.Shape(32, 8, 96, 32, 16, BF), D.DKV_ERR_UNSUPPORTED),     # head_dim
    (D.Shape(32, 8, 128, 48, 16, BF), D.DKV_ERR_UNSUPPORTED),    # rank not a power of two
    (D.Shape(32, 8, 128, 32, 8, BF), D.DKV_ERR_UNSUPPORTED),     # stride
    (D.Shape(32, 8, 128, 128, 16, BF), D.DKV_ERR_UNSUPPORTED),   # 2r > 128 on the tensor-core path
    (D.Shape(96, 8, 128, 32, 16, BF), D.DKV_ERR_UNSUPPORTED),    # G = 12
    (D.Shape(30, 8, 128, 32, 16, BF), D.DKV_ERR_INVALID_ARG),    # H_q not a multiple of H_kv
    (D.Shape(32, 8, 64, 128, 16, BF), D.DKV_ERR_INVALID_ARG),    # rank > head_dim
    (D.Shape(0, 8, 128, 32, 16, BF), D.DKV_ERR_INVALID_ARG),
])
def test_shape_validation(lib, shape, status):
    assert D.check_shape(shape) == status


@pytest.mark.parametrize("d,r,R,dtype", [(128, 32, 16, BF), (128, 32, 32, BF), (64, 16, 16, torch.float32),
                                         (128, 64, 64, BF)])
def test_block_bytes_match_closed_form(lib, d, r, R, dtype):
    H = 8
    sh = D.Shape(32, H, d, r, R, dtype)
    es = 4 if dtype == torch.float32 else 2
    assert D.block_bytes(sh) == round(O.compressed_bytes_per_token(d, r, R, es) * R * H)
    c, i, f = D.cache_bytes(sh, 10)
    assert c + i + f == 10 * D.block_bytes(sh)
    assert (c, i, f) == (10 * H * R * 2 * r * es, 10 * H * R * 4, 10 * H * 2 * d * es)


def test_compressed_ratio_of_library_layout(lib):
    # bytes per token per kv head / raw 2*d*2: 32.03% at R=16 and 28.91% at R=32 (d=128, r=32, bf16)
    for R, want in ((16, 0.3203), (32, 0.2891)):
        sh = D.Shape(32, 8, 128, 32, R, BF)
        assert round(D.block_bytes(sh) / (8 * R * 2 * 128 * 2), 4) == want


def test_workspace_queries(lib):
    sh = D.Shape(32, 8, 128, 32, 16, BF)
    a = D.compress_workspace(sh, 1, 32768, 32768, 32768)
    # bf16: contiguous reference copies, but no copy of the centred tokens (the search kernel centres its
    # own tiles); fp32: the centred tokens too
    assert 8 * 2048 * 256 * 2 <= a < 8 * 32768 * 256 * 2
    sh32 = D.Shape(2, 2, 64, 16, 16, torch.float32)
    assert D.compress_workspace(sh32, 1, 1024, 1024, 1024) >= 2 * 1024 * 128 * 4
    b = D.decode_workspace(sh, 8, 32768)
    assert b > 0
    with pytest.raises(D.DeltaKVError) as e:
        D.decode_workspace(sh, 1, 32769 * 16)  # more than DKV_MAX_REFS references
    assert e.value.status == D.DKV_ERR_UNSUPPORTED
    with pytest.raises(D.DeltaKVError):
        D.compress_workspace(sh, -1, 10, 10, 10)


def test_decode_reference_cap_of_the_split_kernel(lib):
    # Dense bf16 decode with r in {32, 64} reaches DKV_MAX_REFS for every G: past what the shared-memory masses
    # hold (G = 8 with r = 32: 4208 references; G = 4 with r = 64: 4848), the split kernel keeps them in global
    # memory.  Sparse decode and the CUDA-core split kernel (fp32, r = 16) keep the shared-memory cap; the
    # workspace queries (and the calls) refuse a longer bound before any launch.
    g8 = D.Shape(64, 8, 128, 32, 16, BF)
    r64 = D.Shape(32, 8, 128, 64, 16, BF)
    for sh in (g8, r64, D.Shape(32, 8, 128, 32, 16, BF), D.Shape(8, 8, 128, 32, 16, BF)):
        assert D.decode_workspace(sh, 1, 32768 * 16) > 0
        with pytest.raises(D.DeltaKVError) as e:
            D.decode_workspace(sh, 1, 32769 * 16)
        assert e.value.status == D.DKV_ERR_UNSUPPORTED
    assert D.decode_sparse_workspace(g8, 1, 4208 * 16, 4208 * 16) > 0
    with pytest.raises(D.DeltaKVError):
        D.decode_sparse_workspace(g8, 1, 4209 * 16, 4209 * 16)
    assert D.decode_sparse_workspace(r64, 1, 4848 * 16, 4848 * 16) > 0
    with pytest.raises(D.DeltaKVError):
        D.decode_sparse_workspace(r64, 1, 4849 * 16, 4849 * 16)
    f32 = D.Shape(16, 2, 64, 16, 16, torch.float32)
    assert D.decode_workspace(f32, 1, 1024 * 16) > 0
    with pytest.raises(D.DeltaKVError):
        D.decode_workspace(f32, 1, 32768 * 16)
    # the benchmarked shapes reach the cap with shared-memory masses at 8192 references
    assert D.decode_workspace(D.Shape(32, 8, 128, 32, 16, BF), 64, 8192 * 16) > 0


def test_workspace_sizes_grow_with_their_bounds(lib):
    sh = D.Shape(32, 8, 128, 32, 16, BF)
    dec = [D.decode_workspace(sh, n, t) for n, t in ((1, 1024), (1, 32768), (4, 32768), (4, 131072))]
    assert dec == sorted(dec) and dec[0] < dec[-1]
    cmp_ = [D.compress_workspace(sh, n, n * t, t, t) for n, t in ((1, 1024), (1, 32768), (4, 32768))]
    assert cmp_ == sorted(cmp_) and cmp_[0] < cmp_[-1]


def _fake_call_compress(lib, ws_bytes, **over):
    sh = D.Shape(32, 8, 128, 32, 16, BF).c
    params = D.DkvParams(over.get("mu", 256), 256)
    cache = D.DkvCache(256, 256, 256, over.get("num_blocks", 4))
    fake = 256
    return lib.deltakv_compress(ctypes.byref(sh), ctypes.byref(params), ctypes.byref(cache), fake, fake, fake, fake,
                                fake, over.get("max_blocks", 4), 1, 64, 64, 64, over.get("ws", 256), ws_bytes, None)


def test_compress_rejects_before_launch(lib):
    # none of these reach the device: the status comes back from host validation
    assert _fake_call_compress(lib, 16) == D.DKV_ERR_WORKSPACE
    assert _fake_call_compress(lib, 1 << 40, mu=0) == D.DKV_ERR_INVALID_ARG
    assert _fake_call_compress(lib, 1 << 40, num_blocks=0) == D.DKV_ERR_INVALID_ARG
    assert _fake_call_compress(lib, 1 << 40, max_blocks=3) == D.DKV_ERR_INVALID_ARG  # 3 * 16 < max_ctx 64
    assert _fake_call_compress(lib, 1 << 40, ws=257) == D.DKV_ERR_INVALID_ARG  # misaligned workspace
    assert _fake_call_compress(lib, 1 << 40, mu=260) == D.DKV_ERR_INVALID_ARG  # mu is read in 16-byte vectors
    sh = D.Shape(32, 8, 128, 32, 16, BF).c
    assert lib.deltakv_compress(ctypes.byref(sh), None, None, 0, 0, 0, 0, 0, 1, 1, 1, 1, 1, 0, 0, None) == \
        D.DKV_ERR_INVALID_ARG


def test_decode_rejects_before_launch(lib):
    sh = D.Shape(32, 8, 128, 32, 16, BF).c
    params = D.DkvParams(256, 256)
    cache = D.DkvCache(256, 256, 256, 4)
    f = 256
    call = lambda ws_bytes, out=f, mb=4: lib.deltakv_decode_attention(  # noqa: E731
        ctypes.byref(sh), ctypes.byref(params), ctypes.byref(cache), f, f, f, mb, 1, 64, 0.0, out, None, f, ws_bytes,
        None)
    assert call(16) == D.DKV_ERR_WORKSPACE
    assert call(1 << 40, out=0) == D.DKV_ERR_INVALID_ARG
    assert call(1 << 40, mb=2) == D.DKV_ERR_INVALID_ARG
    params.mu = 260  # not 16-byte aligned
    assert call(1 << 40) == D.DKV_ERR_INVALID_ARG
    params.mu = 256
    bad = D.Shape(32, 8, 128, 32, 8, BF).c
    assert lib.deltakv_decode_attention(ctypes.byref(bad), ctypes.byref(params), ctypes.byref(cache), f, f, f, 4, 1,
                                        64, 0.0, f, None, f, 1 << 40, None) == D.DKV_ERR_UNSUPPORTED


def test_empty_calls_are_noops(lib):
    sh = D.Shape(32, 8, 128, 32, 16, BF).c
    params = D.DkvParams(256, 256)
    cache = D.DkvCache(256, 256, 256, 4)
    assert lib.deltakv_compress(ctypes.byref(sh), ctypes.byref(params), ctypes.byref(cache), 0, 0, 0, 0, 0, 4, 0, 0,
                                0, 64, 0, 0, None) == D.DKV_OK
    assert lib.deltakv_decode_attention(ctypes.byref(sh), ctypes.byref(params), ctypes.byref(cache), 0, 0, 0, 4, 0,
                                        64, 0.0, 0, None, 0, 0, None) == D.DKV_OK


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(D, "_lib", None)
    monkeypatch.setattr(D, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        D.load_library()


def test_q4_shape_support_and_sizes(lib):
    import oracle.deltakv_oracle as Ox
    sh = D.Shape(32, 8, 128, 32, 16, torch.bfloat16, q4=True)
    assert D.check_shape(sh) == D.DKV_OK
    assert D.check_shape(D.Shape(32, 8, 128, 16, 16, torch.bfloat16, q4=True)) == D.DKV_ERR_UNSUPPORTED
    # closed form: r nibble bytes + 2 bf16 scales + index per token, one 2d-wide bf16 reference per R tokens
    assert D.block_bytes(sh) == 8 * 16 * Ox.compressed_bytes_per_token_q4(128, 32, 16, 2)
    cb, ib, rb = D.cache_bytes(sh, 10)
    assert cb == 10 * 8 * 16 * (32 + 4) and ib == 10 * 8 * 16 * 4 and rb == 10 * 8 * 2 * 128 * 2
    # decode with 4-bit codes: G in {4, 8}; sparse decode reads unquantised codes only
    assert D.decode_workspace(sh, 2, 4096) > 0
    with pytest.raises(D.DeltaKVError) as e:
        D.decode_workspace(D.Shape(16, 8, 128, 32, 16, torch.bfloat16, q4=True), 2, 4096)
    assert e.value.status == D.DKV_ERR_UNSUPPORTED
    with pytest.raises(D.DeltaKVError) as e:
        D.decode_sparse_workspace(sh, 2, 4096, 100)
    assert e.value.status == D.DKV_ERR_UNSUPPORTED


def test_wait_selftest_rejects_bad_arguments_before_any_launch(lib):
    # a NULL or misaligned result, or a limit outside 1 us .. 2 s, is refused on the host (no GPU needed)
    assert lib.deltakv_selftest_wait_timeout(1_000_000, None, None) == D.DKV_ERR_INVALID_ARG
    assert lib.deltakv_selftest_wait_timeout(1_000_000, 4, None) == D.DKV_ERR_INVALID_ARG
    assert lib.deltakv_selftest_wait_timeout(999, 256, None) == D.DKV_ERR_INVALID_ARG
    assert lib.deltakv_selftest_wait_timeout(2_000_000_001, 256, None) == D.DKV_ERR_INVALID_ARG


def test_k_nearest_entry_points_reject_before_launch(lib):
    # k in {1, 2, 4}; k > 1 needs bf16 codes, r in {32, 64} and G in {4, 8}; all refused before any launch
    g4 = D.Shape(32, 8, 128, 32, 16, BF)
    assert D.decode_topk_workspace(g4, 2, 1, 1024) > 0 and D.decode_topk_workspace(g4, 4, 1, 1024) > 0
    for sh, k in ((g4, 3), (g4, 0), (D.Shape(16, 8, 128, 32, 16, BF), 2), (D.Shape(32, 8, 128, 16, 16, BF), 2),
                  (D.Shape(16, 4, 64, 16, 16, torch.float32), 2)):
        with pytest.raises(D.DeltaKVError) as e:
            D.decode_topk_workspace(sh, k, 1, 1024)
        assert e.value.status == D.DKV_ERR_UNSUPPORTED, (sh, k)
    params, cache, f = D.DkvParams(256, 256), D.DkvCache(256, 256, 256, 4), 256

    def compress(sh, k, ws_bytes):
        return lib.deltakv_compress_topk(ctypes.byref(sh.c), k, ctypes.byref(params), ctypes.byref(cache), f, f, f, f,
                                         f, 4, 1, 64, 64, 64, f, ws_bytes, None)

    def decode(sh, k, ws_bytes):
        return lib.deltakv_decode_attention_topk(ctypes.byref(sh.c), k, ctypes.byref(params), ctypes.byref(cache), f,
                                                 f, f, 4, 1, 64, 0.0, f, None, f, ws_bytes, None)

    assert compress(g4, 3, 1 << 40) == D.DKV_ERR_UNSUPPORTED
    assert compress(D.Shape(16, 4, 64, 16, 16, torch.float32), 2, 1 << 40) == D.DKV_ERR_UNSUPPORTED
    assert compress(g4, 2, 16) == D.DKV_ERR_WORKSPACE
    assert decode(g4, 3, 1 << 40) == D.DKV_ERR_UNSUPPORTED
    assert decode(D.Shape(16, 8, 128, 32, 16, BF), 2, 1 << 40) == D.DKV_ERR_UNSUPPORTED  # G = 2
    assert decode(g4, 2, 16) == D.DKV_ERR_WORKSPACE


def test_sparse_decode_rejects_before_launch(lib):
    sh = D.Shape(32, 8, 128, 32, 16, BF)
    params, cache, f = D.DkvParams(256, 256), D.DkvCache(256, 256, 256, 4), 256

    def call(ws_bytes, shape=sh, token_idx=f, cu_tokens=f, max_sel=16):
        return lib.deltakv_decode_attention_sparse(ctypes.byref(shape.c), ctypes.byref(params), ctypes.byref(cache),
                                                   f, f, f, 4, token_idx, cu_tokens, max_sel, 1, 64, 0.0, f, None, f,
                                                   ws_bytes, None)

    assert call(16) == D.DKV_ERR_WORKSPACE
    assert call(1 << 40, cu_tokens=None) == D.DKV_ERR_INVALID_ARG
    assert call(1 << 40, token_idx=None) == D.DKV_ERR_INVALID_ARG    # a list may be non-empty (max_sel > 0)
    assert call(1 << 40, max_sel=-1) == D.DKV_ERR_INVALID_ARG
    assert call(1 << 40, shape=D.Shape(32, 8, 128, 32, 16, BF, q4=True)) == D.DKV_ERR_UNSUPPORTED
    # the sparse workspace grows with the list bound, and the query refuses the same shapes
    assert D.decode_sparse_workspace(sh, 2, 4096, 100) < D.decode_sparse_workspace(sh, 2, 4096, 4096)
    with pytest.raises(D.DeltaKVError) as e:
        D.decode_sparse_workspace(sh, 2, 4096, -1)
    assert e.value.status == D.DKV_ERR_INVALID_ARG


def test_no_alloc_decode_checks_support_before_its_scratch_bound(lib):
    params, cache, f = D.DkvParams(256, 256), D.DkvCache(256, 256, 256, 1 << 20), 256

    def call(shape, num_seqs, max_ctx):
        mb = max_ctx // shape.ref_stride + 1
        return lib.deltakv_decode_attention_noalloc(ctypes.byref(shape.c), ctypes.byref(params), ctypes.byref(cache),
                                                    f, f, f, mb, num_seqs, max_ctx, 0.0, f, None, None)

    sh = D.Shape(32, 8, 128, 32, 16, BF)
    big = (64, 131072)
    assert D.decode_workspace(sh, *big) > D.NOALLOC_SCRATCH_BYTES
    assert call(sh, *big) == D.DKV_ERR_WORKSPACE          # supported, but past the fixed 16 MiB scratch
    assert call(sh, 64, 32769 * 16) == D.DKV_ERR_UNSUPPORTED  # past the reference cap: unsupported, not "workspace"
