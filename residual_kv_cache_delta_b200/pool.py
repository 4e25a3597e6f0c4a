"""ctypes binding of the host block pool and continuous-batching planner (include/deltakv_pool.h).

Argument marshalling only: every decision (which block, which request, preemption) is made by the C++ code
in ``libdeltakv.so``.  Block tables, ``cu_new``, ``start_pos`` and context lengths come back as NumPy arrays,
ready for ``torch.from_numpy(...).to(device)`` and the deltakv_compress / deltakv_decode_attention calls.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np

from . import deltakv as D

DKV_ERR_OUT_OF_BLOCKS = 5
EXPORTED = ("deltakv_pool_create", "deltakv_pool_destroy", "deltakv_pool_num_free", "deltakv_pool_open",
            "deltakv_pool_grow", "deltakv_pool_close", "deltakv_pool_seq_info", "deltakv_pool_block_tables",
            "deltakv_batcher_create", "deltakv_batcher_destroy", "deltakv_batcher_submit", "deltakv_batcher_plan",
            "deltakv_batcher_commit", "deltakv_batcher_counts")


class OutOfBlocks(D.DeltaKVError):
    pass


class DkvStepPlan(ctypes.Structure):
    _fields_ = [("num_compress", ctypes.c_int32), ("comp_req", ctypes.c_void_p), ("comp_seq", ctypes.c_void_p),
                ("cu_new", ctypes.c_void_p), ("start_pos", ctypes.c_void_p), ("comp_from", ctypes.c_void_p),
                ("num_decode", ctypes.c_int32), ("dec_req", ctypes.c_void_p), ("dec_seq", ctypes.c_void_p),
                ("context_len", ctypes.c_void_p), ("num_preempted", ctypes.c_int32)]


_bound = False


def _lib():
    global _bound
    lib = D.load_library()
    if not _bound:
        P, I32, I64, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
        pI32, pI64 = ctypes.POINTER(I32), ctypes.POINTER(I64)
        sig = {
            "deltakv_pool_create": ([I32, I32, I32, I32, U64, ctypes.POINTER(P)], ctypes.c_int),
            "deltakv_pool_destroy": ([P], None),
            "deltakv_pool_num_free": ([P], I32),
            "deltakv_pool_open": ([P, pI32], ctypes.c_int),
            "deltakv_pool_grow": ([P, I32, I32], ctypes.c_int),
            "deltakv_pool_close": ([P, I32], ctypes.c_int),
            "deltakv_pool_seq_info": ([P, I32, pI32, pI32], ctypes.c_int),
            "deltakv_pool_block_tables": ([P, P, I32, I32, P], ctypes.c_int),
            "deltakv_batcher_create": ([P, I32, I32, ctypes.POINTER(P)], ctypes.c_int),
            "deltakv_batcher_destroy": ([P], None),
            "deltakv_batcher_submit": ([P, I64, I32, I32], ctypes.c_int),
            "deltakv_batcher_plan": ([P, ctypes.POINTER(DkvStepPlan)], ctypes.c_int),
            "deltakv_batcher_commit": ([P, P, pI32], ctypes.c_int),
            "deltakv_batcher_counts": ([P, pI32, pI32, pI64], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _bound = True
    return lib


def _check(status: int, what: str):
    if status == DKV_ERR_OUT_OF_BLOCKS:
        raise OutOfBlocks(status, what)
    if status != D.DKV_OK:
        raise D.DeltaKVError(status, what)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


class BlockPool:
    """Physical blocks of a paged cache (ids 0 .. num_blocks-1), handed to sequences on the host."""

    def __init__(self, num_blocks: int, block_tokens: int, max_seqs: int, max_blocks_per_seq: int, seed: int = 0):
        self._h = ctypes.c_void_p()
        _check(_lib().deltakv_pool_create(num_blocks, block_tokens, max_seqs, max_blocks_per_seq, seed,
                                          ctypes.byref(self._h)), "deltakv_pool_create")
        self.num_blocks, self.block_tokens = num_blocks, block_tokens

    def close_pool(self):
        if self._h:
            _lib().deltakv_pool_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close_pool()
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    def num_free(self) -> int:
        return _lib().deltakv_pool_num_free(self._h)

    def open(self) -> int:
        s = ctypes.c_int32()
        _check(_lib().deltakv_pool_open(self._h, ctypes.byref(s)), "deltakv_pool_open")
        return s.value

    def grow(self, seq: int, new_len: int) -> None:
        _check(_lib().deltakv_pool_grow(self._h, seq, new_len), "deltakv_pool_grow")

    def close(self, seq: int) -> None:
        _check(_lib().deltakv_pool_close(self._h, seq), "deltakv_pool_close")

    def info(self, seq: int) -> tuple[int, int]:
        n, b = ctypes.c_int32(), ctypes.c_int32()
        _check(_lib().deltakv_pool_seq_info(self._h, seq, ctypes.byref(n), ctypes.byref(b)), "deltakv_pool_seq_info")
        return n.value, b.value

    def block_tables(self, seqs, max_blocks: int) -> np.ndarray:
        seqs = _i32(seqs)
        out = np.empty((len(seqs), max_blocks), dtype=np.int32)
        _check(_lib().deltakv_pool_block_tables(self._h, seqs.ctypes.data, len(seqs), max_blocks, out.ctypes.data),
               "deltakv_pool_block_tables")
        return out


@dataclass
class StepPlan:
    comp_req: np.ndarray
    comp_seq: np.ndarray
    cu_new: np.ndarray
    start_pos: np.ndarray
    comp_from: np.ndarray
    dec_req: np.ndarray
    dec_seq: np.ndarray
    context_len: np.ndarray
    num_preempted: int


class Batcher:
    """Continuous-batching planner over a BlockPool (see include/deltakv_pool.h for the policy)."""

    def __init__(self, pool: BlockPool, max_prefill_tokens: int, max_batch: int):
        self.pool, self.max_batch = pool, max_batch
        self._h = ctypes.c_void_p()
        _check(_lib().deltakv_batcher_create(pool.handle, max_prefill_tokens, max_batch, ctypes.byref(self._h)),
               "deltakv_batcher_create")

    def __del__(self):
        try:
            if self._h:
                _lib().deltakv_batcher_destroy(self._h)
                self._h = ctypes.c_void_p()
        except Exception:
            pass

    def submit(self, request_id: int, prompt_len: int, max_new_tokens: int) -> None:
        _check(_lib().deltakv_batcher_submit(self._h, request_id, prompt_len, max_new_tokens), "deltakv_batcher_submit")

    def plan(self) -> StepPlan:
        n = self.max_batch
        a = dict(comp_req=np.empty(n, np.int64), comp_seq=np.empty(n, np.int32), cu_new=np.empty(n + 1, np.int32),
                 start_pos=np.empty(n, np.int32), comp_from=np.empty(n, np.int32), dec_req=np.empty(n, np.int64),
                 dec_seq=np.empty(n, np.int32), context_len=np.empty(n, np.int32))
        p = DkvStepPlan(0, a["comp_req"].ctypes.data, a["comp_seq"].ctypes.data, a["cu_new"].ctypes.data,
                        a["start_pos"].ctypes.data, a["comp_from"].ctypes.data, 0, a["dec_req"].ctypes.data,
                        a["dec_seq"].ctypes.data, a["context_len"].ctypes.data, 0)
        _check(_lib().deltakv_batcher_plan(self._h, ctypes.byref(p)), "deltakv_batcher_plan")
        nc, nd = p.num_compress, p.num_decode
        return StepPlan(a["comp_req"][:nc].copy(), a["comp_seq"][:nc].copy(), a["cu_new"][:nc + 1].copy(),
                        a["start_pos"][:nc].copy(), a["comp_from"][:nc].copy(), a["dec_req"][:nd].copy(),
                        a["dec_seq"][:nd].copy(), a["context_len"][:nd].copy(), p.num_preempted)

    def commit(self) -> list:
        fin = np.empty(self.max_batch, np.int64)
        nf = ctypes.c_int32()
        _check(_lib().deltakv_batcher_commit(self._h, fin.ctypes.data, ctypes.byref(nf)), "deltakv_batcher_commit")
        return [int(x) for x in fin[:nf.value]]

    def counts(self) -> tuple[int, int, int]:
        w, r, f = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int64()
        _check(_lib().deltakv_batcher_counts(self._h, ctypes.byref(w), ctypes.byref(r), ctypes.byref(f)),
               "deltakv_batcher_counts")
        return w.value, r.value, f.value
