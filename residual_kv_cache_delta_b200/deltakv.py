"""Thin ctypes binding of ``libdeltakv.so`` (argument marshalling only).

Every computation runs in the library's CUDA kernels.  This module converts torch tensors to raw
pointers and sizes, checks their dtypes/devices/contiguity, calls the C entry point of the same name and
raises on a non-OK status.  There is no fallback: if the library is missing or fails to load, every call
raises ``RuntimeError``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdeltakv.so")

DKV_OK, DKV_ERR_INVALID_ARG, DKV_ERR_UNSUPPORTED, DKV_ERR_WORKSPACE, DKV_ERR_CUDA, DKV_ERR_OUT_OF_BLOCKS = range(6)
DKV_F32, DKV_BF16, DKV_BF16_Q4 = 0, 1, 2
DEVERR_NAMES = {0: "none", 1: "block id out of range", 2: "reference index out of range",
                3: "length over host bound", 4: "pipeline wait timed out"}

# every symbol include/deltakv.h declares
EXPORTED = ("deltakv_status_string", "deltakv_check_shape", "deltakv_block_bytes", "deltakv_cache_bytes",
            "deltakv_compress_workspace", "deltakv_decode_workspace", "deltakv_compress",
            "deltakv_decode_attention", "deltakv_profile_kernel", "deltakv_profile_count",
            "deltakv_get_device_error", "deltakv_decode_attention_noalloc", "deltakv_decode_sparse_workspace",
            "deltakv_decode_attention_sparse", "deltakv_compress_topk", "deltakv_decode_topk_workspace",
            "deltakv_decode_attention_topk", "deltakv_selftest_wait_timeout")
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024
KERNEL_CENTER, KERNEL_REFPREP, KERNEL_SEARCH, KERNEL_DECODE_PROLOGUE, KERNEL_DECODE_SPLIT, KERNEL_DECODE_COMBINE = range(6)


class DkvShape(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("rank", ctypes.c_int32), ("ref_stride", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class DkvParams(ctypes.Structure):
    _fields_ = [("mu", ctypes.c_void_p), ("basis", ctypes.c_void_p)]


class DkvCache(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("ref_idx", ctypes.c_void_p), ("refs", ctypes.c_void_p),
                ("num_blocks", ctypes.c_int32)]


_lib = None


def load_library() -> ctypes.CDLL:
    """Load ``libdeltakv.so`` (built in-tree by ``build.py``); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libdeltakv.so not built ({LIB_PATH}); run residual_kv_cache_delta_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    pshape, pparams, pcache = ctypes.POINTER(DkvShape), ctypes.POINTER(DkvParams), ctypes.POINTER(DkvCache)
    lib.deltakv_status_string.argtypes = [ctypes.c_int]
    lib.deltakv_status_string.restype = ctypes.c_char_p
    lib.deltakv_check_shape.argtypes = [pshape]
    lib.deltakv_check_shape.restype = ctypes.c_int
    lib.deltakv_block_bytes.argtypes = [pshape]
    lib.deltakv_block_bytes.restype = SZ
    lib.deltakv_cache_bytes.argtypes = [pshape, I32, ctypes.POINTER(SZ), ctypes.POINTER(SZ), ctypes.POINTER(SZ)]
    lib.deltakv_cache_bytes.restype = ctypes.c_int
    lib.deltakv_compress_workspace.argtypes = [pshape, I32, I64, I32, I32, ctypes.POINTER(SZ)]
    lib.deltakv_compress_workspace.restype = ctypes.c_int
    lib.deltakv_decode_workspace.argtypes = [pshape, I32, I32, ctypes.POINTER(SZ)]
    lib.deltakv_decode_workspace.restype = ctypes.c_int
    lib.deltakv_compress.argtypes = [pshape, pparams, pcache, P, P, P, P, P, I32, I32, I64, I32, I32, P, SZ, P]
    lib.deltakv_compress.restype = ctypes.c_int
    lib.deltakv_decode_attention.argtypes = [pshape, pparams, pcache, P, P, P, I32, I32, I32, ctypes.c_float, P, P,
                                             P, SZ, P]
    lib.deltakv_decode_attention.restype = ctypes.c_int
    lib.deltakv_profile_kernel.argtypes = [I32, P, P, I32]
    lib.deltakv_profile_kernel.restype = ctypes.c_int
    lib.deltakv_profile_count.argtypes = [I32, ctypes.POINTER(I32)]
    lib.deltakv_profile_count.restype = ctypes.c_int
    lib.deltakv_decode_attention_noalloc.argtypes = [pshape, pparams, pcache, P, P, P, I32, I32, I32, ctypes.c_float,
                                                     P, P, P]
    lib.deltakv_decode_attention_noalloc.restype = ctypes.c_int
    lib.deltakv_decode_sparse_workspace.argtypes = [pshape, I32, I32, I32, ctypes.POINTER(SZ)]
    lib.deltakv_decode_sparse_workspace.restype = ctypes.c_int
    lib.deltakv_decode_attention_sparse.argtypes = [pshape, pparams, pcache, P, P, P, I32, P, P, I32, I32, I32,
                                                    ctypes.c_float, P, P, P, SZ, P]
    lib.deltakv_decode_attention_sparse.restype = ctypes.c_int
    lib.deltakv_compress_topk.argtypes = [pshape, I32, pparams, pcache, P, P, P, P, P, I32, I32, I64, I32, I32, P,
                                          SZ, P]
    lib.deltakv_compress_topk.restype = ctypes.c_int
    lib.deltakv_decode_topk_workspace.argtypes = [pshape, I32, I32, I32, ctypes.POINTER(SZ)]
    lib.deltakv_decode_topk_workspace.restype = ctypes.c_int
    lib.deltakv_decode_attention_topk.argtypes = [pshape, I32, pparams, pcache, P, P, P, I32, I32, I32, ctypes.c_float,
                                                  P, P, P, SZ, P]
    lib.deltakv_decode_attention_topk.restype = ctypes.c_int
    lib.deltakv_get_device_error.argtypes = [P, ctypes.POINTER(I32)]
    lib.deltakv_get_device_error.restype = ctypes.c_int
    lib.deltakv_selftest_wait_timeout.argtypes = [ctypes.c_uint64, P, P]
    lib.deltakv_selftest_wait_timeout.restype = ctypes.c_int
    _lib = lib
    return lib


class DeltaKVError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


def status_string(status: int) -> str:
    return load_library().deltakv_status_string(status).decode()


def _check(status: int, what: str):
    if status != DKV_OK:
        raise DeltaKVError(status, what)


@dataclass(frozen=True)
class Shape:
    """Head geometry of one layer (mirrors ``dkv_shape``)."""

    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    rank: int
    ref_stride: int
    dtype: torch.dtype = torch.bfloat16
    q4: bool = False  # 4-bit residual codes (bf16 storage otherwise; see include/deltakv.h)

    @property
    def c(self) -> DkvShape:
        dt = DKV_F32 if self.dtype == torch.float32 else (DKV_BF16_Q4 if self.q4 else DKV_BF16)
        return DkvShape(self.num_q_heads, self.num_kv_heads, self.head_dim, self.rank, self.ref_stride, dt)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


def check_shape(shape: Shape) -> int:
    return load_library().deltakv_check_shape(ctypes.byref(shape.c))


def block_bytes(shape: Shape) -> int:
    return int(load_library().deltakv_block_bytes(ctypes.byref(shape.c)))


def cache_bytes(shape: Shape, num_blocks: int) -> tuple[int, int, int]:
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(load_library().deltakv_cache_bytes(ctypes.byref(shape.c), num_blocks, ctypes.byref(a), ctypes.byref(b),
                                              ctypes.byref(c)), "deltakv_cache_bytes")
    return a.value, b.value, c.value


def compress_workspace(shape: Shape, num_seqs: int, total_new: int, max_new: int, max_ctx: int) -> int:
    n = ctypes.c_size_t()
    _check(load_library().deltakv_compress_workspace(ctypes.byref(shape.c), num_seqs, total_new, max_new, max_ctx,
                                                     ctypes.byref(n)), "deltakv_compress_workspace")
    return n.value


def decode_workspace(shape: Shape, num_seqs: int, max_ctx: int) -> int:
    n = ctypes.c_size_t()
    _check(load_library().deltakv_decode_workspace(ctypes.byref(shape.c), num_seqs, max_ctx, ctypes.byref(n)),
           "deltakv_decode_workspace")
    return n.value


def decode_sparse_workspace(shape: Shape, num_seqs: int, max_ctx: int, max_sel: int) -> int:
    n = ctypes.c_size_t()
    _check(load_library().deltakv_decode_sparse_workspace(ctypes.byref(shape.c), num_seqs, max_ctx, max_sel,
                                                          ctypes.byref(n)), "deltakv_decode_sparse_workspace")
    return n.value


@dataclass
class Cache:
    """Caller-owned device arrays of one layer's compressed cache (layout in include/deltakv.h)."""

    codes: torch.Tensor    # [num_blocks, H_kv, R, 2r] dtype
    ref_idx: torch.Tensor  # [num_blocks, H_kv, R] int32
    refs: torch.Tensor     # [num_blocks, H_kv, 2, d] dtype

    @property
    def num_blocks(self) -> int:
        return self.codes.shape[0]

    @property
    def c(self) -> DkvCache:
        return DkvCache(self.codes.data_ptr(), self.ref_idx.data_ptr(), self.refs.data_ptr(), self.num_blocks)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.codes, self.ref_idx, self.refs))


def alloc_cache(shape: Shape, num_blocks: int, device="cuda", topk: int = 0) -> Cache:
    """Zeroed cache arrays.  With 4-bit codes, ``codes`` is uint8 [num_blocks, H_kv, R*(r+4)] (per block and
    kv head: R packed rows of r bytes, then R pairs of bf16 scales).  topk > 0 (the k-nearest compress):
    ``ref_idx`` is [num_blocks, H_kv, R, k]."""
    H, R, r, d = shape.num_kv_heads, shape.ref_stride, shape.rank, shape.head_dim
    if topk > 0:
        return Cache(torch.zeros((num_blocks, H, R, 2 * r), dtype=shape.dtype, device=device),
                     torch.zeros((num_blocks, H, R, topk), dtype=torch.int32, device=device),
                     torch.zeros((num_blocks, H, 2, d), dtype=shape.dtype, device=device))
    if shape.q4:
        return Cache(torch.zeros((num_blocks, H, R * (r + 4)), dtype=torch.uint8, device=device),
                     torch.zeros((num_blocks, H, R), dtype=torch.int32, device=device),
                     torch.zeros((num_blocks, H, 2, d), dtype=shape.dtype, device=device))
    return Cache(torch.zeros((num_blocks, H, R, 2 * r), dtype=shape.dtype, device=device),
                 torch.zeros((num_blocks, H, R), dtype=torch.int32, device=device),
                 torch.zeros((num_blocks, H, 2, d), dtype=shape.dtype, device=device))


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte-aligned byte buffer (torch's caching allocator returns 512-byte-aligned blocks)."""
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)


def _ptr(t: Optional[torch.Tensor], dtype: Optional[torch.dtype] = None, name: str = "") -> int:
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def deltakv_compress(shape: Shape, mu: torch.Tensor, basis: torch.Tensor, cache: Cache, k_new: torch.Tensor,
                     v_new: torch.Tensor, cu_new: torch.Tensor, start_pos: torch.Tensor, block_tables: torch.Tensor,
                     max_new: int, max_ctx: int, workspace: torch.Tensor, stream=None) -> None:
    """Enqueue ``deltakv_compress`` (see include/deltakv.h).  Shapes: k_new/v_new [total_new, H_kv, d];
    cu_new [num_seqs+1]; start_pos [num_seqs]; block_tables [num_seqs, max_blocks] (all int32)."""
    sc = shape.c
    params = DkvParams(_ptr(mu, torch.float32, "mu"), _ptr(basis, shape.dtype, "basis"))
    cc = cache.c
    num_seqs, max_blocks = block_tables.shape
    st = load_library().deltakv_compress(
        ctypes.byref(sc), ctypes.byref(params), ctypes.byref(cc), _ptr(k_new, shape.dtype, "k_new"),
        _ptr(v_new, shape.dtype, "v_new"), _ptr(cu_new, torch.int32, "cu_new"),
        _ptr(start_pos, torch.int32, "start_pos"), _ptr(block_tables, torch.int32, "block_tables"), max_blocks,
        num_seqs, k_new.shape[0], max_new, max_ctx, _ptr(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream))
    _check(st, "deltakv_compress")


def deltakv_decode_attention(shape: Shape, mu: torch.Tensor, basis: torch.Tensor, cache: Cache, q: torch.Tensor,
                             context_lens: torch.Tensor, block_tables: torch.Tensor, max_ctx: int,
                             out: torch.Tensor, lse: Optional[torch.Tensor], workspace: torch.Tensor,
                             softmax_scale: float = 0.0, stream=None) -> None:
    """Enqueue ``deltakv_decode_attention``.  q/out [num_seqs, H_q, d]; lse [num_seqs, H_q] fp32 or None."""
    sc = shape.c
    params = DkvParams(_ptr(mu, torch.float32, "mu"), _ptr(basis, shape.dtype, "basis"))
    cc = cache.c
    num_seqs, max_blocks = block_tables.shape
    st = load_library().deltakv_decode_attention(
        ctypes.byref(sc), ctypes.byref(params), ctypes.byref(cc), _ptr(q, shape.dtype, "q"),
        _ptr(context_lens, torch.int32, "context_lens"), _ptr(block_tables, torch.int32, "block_tables"),
        max_blocks, num_seqs, max_ctx, float(softmax_scale), _ptr(out, shape.dtype, "out"),
        _ptr(lse, torch.float32, "lse"), _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
        _stream(stream))
    _check(st, "deltakv_decode_attention")


def deltakv_decode_attention_noalloc(shape: Shape, mu: torch.Tensor, basis: torch.Tensor, cache: Cache,
                                     q: torch.Tensor, context_lens: torch.Tensor, block_tables: torch.Tensor,
                                     max_ctx: int, out: torch.Tensor, lse: Optional[torch.Tensor],
                                     softmax_scale: float = 0.0, stream=None) -> None:
    """Enqueue ``deltakv_decode_attention_noalloc``: decode attention with the library's own fixed scratch
    array instead of a caller workspace (no device allocation anywhere; see include/deltakv.h)."""
    sc = shape.c
    params = DkvParams(_ptr(mu, torch.float32, "mu"), _ptr(basis, shape.dtype, "basis"))
    cc = cache.c
    num_seqs, max_blocks = block_tables.shape
    st = load_library().deltakv_decode_attention_noalloc(
        ctypes.byref(sc), ctypes.byref(params), ctypes.byref(cc), _ptr(q, shape.dtype, "q"),
        _ptr(context_lens, torch.int32, "context_lens"), _ptr(block_tables, torch.int32, "block_tables"),
        max_blocks, num_seqs, max_ctx, float(softmax_scale), _ptr(out, shape.dtype, "out"),
        _ptr(lse, torch.float32, "lse"), _stream(stream))
    _check(st, "deltakv_decode_attention_noalloc")


def deltakv_decode_attention_sparse(shape: Shape, mu: torch.Tensor, basis: torch.Tensor, cache: Cache,
                                    q: torch.Tensor, context_lens: torch.Tensor, block_tables: torch.Tensor,
                                    token_idx: torch.Tensor, cu_tokens: torch.Tensor, max_sel: int, max_ctx: int,
                                    out: torch.Tensor, lse: Optional[torch.Tensor], workspace: torch.Tensor,
                                    softmax_scale: float = 0.0, stream=None) -> None:
    """Enqueue ``deltakv_decode_attention_sparse``: decode over the positions token_idx[cu_tokens[s] ..
    cu_tokens[s+1]-1] of each sequence (int32 device tensors); other arguments as in the dense call."""
    sc = shape.c
    params = DkvParams(_ptr(mu, torch.float32, "mu"), _ptr(basis, shape.dtype, "basis"))
    cc = cache.c
    num_seqs, max_blocks = block_tables.shape
    tok = _ptr(token_idx, torch.int32, "token_idx") if token_idx.numel() > 0 else 0
    st = load_library().deltakv_decode_attention_sparse(
        ctypes.byref(sc), ctypes.byref(params), ctypes.byref(cc), _ptr(q, shape.dtype, "q"),
        _ptr(context_lens, torch.int32, "context_lens"), _ptr(block_tables, torch.int32, "block_tables"),
        max_blocks, tok, _ptr(cu_tokens, torch.int32, "cu_tokens"), max_sel, num_seqs, max_ctx,
        float(softmax_scale), _ptr(out, shape.dtype, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream))
    _check(st, "deltakv_decode_attention_sparse")


def decode_topk_workspace(shape: Shape, k: int, num_seqs: int, max_ctx: int) -> int:
    n = ctypes.c_size_t()
    _check(load_library().deltakv_decode_topk_workspace(ctypes.byref(shape.c), k, num_seqs, max_ctx, ctypes.byref(n)),
           "deltakv_decode_topk_workspace")
    return n.value


def deltakv_compress_topk(shape: Shape, k: int, mu: torch.Tensor, basis: torch.Tensor, cache: Cache,
                          k_new: torch.Tensor, v_new: torch.Tensor, cu_new: torch.Tensor, start_pos: torch.Tensor,
                          block_tables: torch.Tensor, max_new: int, max_ctx: int, workspace: torch.Tensor,
                          stream=None) -> None:
    """Enqueue ``deltakv_compress_topk`` (the k nearest references by L2, residual against their mean); the
    cache's ref_idx holds k slots per token (alloc_cache(..., topk=k))."""
    sc = shape.c
    params = DkvParams(_ptr(mu, torch.float32, "mu"), _ptr(basis, shape.dtype, "basis"))
    cc = cache.c
    num_seqs, max_blocks = block_tables.shape
    st = load_library().deltakv_compress_topk(
        ctypes.byref(sc), k, ctypes.byref(params), ctypes.byref(cc), _ptr(k_new, shape.dtype, "k_new"),
        _ptr(v_new, shape.dtype, "v_new"), _ptr(cu_new, torch.int32, "cu_new"),
        _ptr(start_pos, torch.int32, "start_pos"), _ptr(block_tables, torch.int32, "block_tables"), max_blocks,
        num_seqs, k_new.shape[0], max_new, max_ctx, _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
        _stream(stream))
    _check(st, "deltakv_compress_topk")


def deltakv_decode_attention_topk(shape: Shape, k: int, mu: torch.Tensor, basis: torch.Tensor, cache: Cache,
                                  q: torch.Tensor, context_lens: torch.Tensor, block_tables: torch.Tensor,
                                  max_ctx: int, out: torch.Tensor, lse: Optional[torch.Tensor],
                                  workspace: torch.Tensor, softmax_scale: float = 0.0, stream=None) -> None:
    """Enqueue ``deltakv_decode_attention_topk`` over a cache written by deltakv_compress_topk with the same k."""
    sc = shape.c
    params = DkvParams(_ptr(mu, torch.float32, "mu"), _ptr(basis, shape.dtype, "basis"))
    cc = cache.c
    num_seqs, max_blocks = block_tables.shape
    st = load_library().deltakv_decode_attention_topk(
        ctypes.byref(sc), k, ctypes.byref(params), ctypes.byref(cc), _ptr(q, shape.dtype, "q"),
        _ptr(context_lens, torch.int32, "context_lens"), _ptr(block_tables, torch.int32, "block_tables"),
        max_blocks, num_seqs, max_ctx, float(softmax_scale), _ptr(out, shape.dtype, "out"),
        _ptr(lse, torch.float32, "lse"), _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
        _stream(stream))
    _check(st, "deltakv_decode_attention_topk")


class KernelTimer:
    """Records CUDA events around the next ``n`` launches of one library kernel (deltakv_profile_kernel)."""

    def __init__(self, kernel_id: int, n: int):
        self.kernel_id = kernel_id
        self.starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        self.stops = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in self.starts + self.stops:
            e.record()  # materialise the underlying cudaEvent_t
        torch.cuda.synchronize()
        self._a = (ctypes.c_void_p * n)(*[e.cuda_event for e in self.starts])
        self._b = (ctypes.c_void_p * n)(*[e.cuda_event for e in self.stops])
        _check(load_library().deltakv_profile_kernel(kernel_id, self._a, self._b, n), "deltakv_profile_kernel")

    def count(self) -> int:
        c = ctypes.c_int32()
        _check(load_library().deltakv_profile_count(self.kernel_id, ctypes.byref(c)), "deltakv_profile_count")
        return c.value

    def times_ms(self) -> list:
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in zip(self.starts[: self.count()], self.stops[: self.count()])]

    def close(self):
        _check(load_library().deltakv_profile_kernel(self.kernel_id, None, None, 0), "deltakv_profile_kernel")


def deltakv_get_device_error(stream=None) -> int:
    """Synchronise ``stream`` and return (and clear) the device error word (0 = none)."""
    code = ctypes.c_int32()
    _check(load_library().deltakv_get_device_error(_stream(stream), ctypes.byref(code)), "deltakv_get_device_error")
    return code.value


def deltakv_selftest_wait_timeout(limit_ns: int, result: torch.Tensor, stream=None) -> None:
    """One bounded wait on a phase that nothing completes, with limit ``limit_ns``; ``result`` is a device int64
    tensor of 2 elements: [completed, waited ns]."""
    assert result.is_cuda and result.dtype == torch.int64 and result.numel() >= 2
    _check(load_library().deltakv_selftest_wait_timeout(int(limit_ns), _ptr(result), _stream(stream)),
           "deltakv_selftest_wait_timeout")
