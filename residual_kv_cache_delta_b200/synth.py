"""Seeded synthetic inputs for the DeltaKV hot path.

This module only draws inputs: raw keys/values, queries, the per-head shared
component ``mu``, the rank-r bases and block tables.  It contains none of the
method's arithmetic (no centering, search, projection or attention), so both
the CUDA path and the CPU oracle can be fed from it without sharing any of the
computation they are compared on.

Data model (DeltaKV summaries, "Key Empirical Observations": long-range
inter-token similarity and highly shared high-norm latent components):

    x_t = mu + c_{cluster(t)} + sigma * eps_t,   cluster(t) = (t*7919 mod P) mod C

with ``mu`` a random direction scaled to a fixed norm (the shared high-norm
component), cluster centres ``c`` ~ N(0, 1) and noise ``eps`` ~ N(0, 1).  The
multiplicative hash makes tokens of the same cluster recur far apart, which is
the long-range similarity the method exploits.  K and V of one token share the
cluster id but use separate centre tables and separate ``mu``.

Random streams come from NumPy's PCG64 keyed by ``SeedSequence(seed,
spawn_key=(role, layer, seq, head, kv))``.  Large workloads can draw the noise
with ``torch.randn`` on a CUDA device instead (``backend="torch"``); those
values differ from the NumPy ones but are still seeded and reproducible.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

ROLE_MU, ROLE_CENTERS, ROLE_NOISE, ROLE_BASIS, ROLE_QUERY, ROLE_PERM, ROLE_LENS = range(7)
KEY, VALUE = 0, 1


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, generator constants and seed."""

    name: str
    seed: int
    layers: int
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    seq_len: int  # context length per sequence (max length for ragged mixes)
    dtype: str  # "f32" or "bf16": storage type of K, V, codes, refs and outputs
    ref_stride: int  # R: every R-th token is a reference; also the paged block size
    rank: int  # r: rank of the code basis
    hash_mod: int  # P in cluster(t) = (t*7919 mod P) mod C
    clusters: int  # C
    mu_norm: float
    sigma: float
    queries_per_seq: int = 1  # decode queries that read one sequence's cache
    ragged: bool = False  # lengths log-uniform in [min_len, seq_len]
    min_len: int = 0
    prefill_len: int = 0  # length of the prefills compressed beside decode
    paged_random: bool = False  # block tables are a random permutation of the pool

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


WORKLOADS = {
    0: Workload("tiny-fp32-d64-T1024", 0, 1, 1, 2, 2, 64, 1024, "f32", 16, 16, 97, 32, 10.0, 0.1,
                queries_per_seq=4),
    1: Workload("llama3-8b-1layer-T32k", 1, 1, 1, 32, 8, 128, 32768, "bf16", 16, 32, 257, 256, 20.0, 0.2),
    2: Workload("llama3-8b-32layer-B8-T32k", 2, 32, 8, 32, 8, 128, 32768, "bf16", 16, 32, 257, 256, 20.0, 0.2),
    3: Workload("llama3-8b-1layer-B4-T128k-R32", 3, 1, 4, 32, 8, 128, 131072, "bf16", 32, 32, 99991, 1024,
                20.0, 0.2),
    4: Workload("paged-mix-64seq-4k..128k", 4, 1, 64, 32, 8, 128, 131072, "bf16", 16, 32, 257, 256, 20.0, 0.2,
                ragged=True, min_len=4096, prefill_len=2048, paged_random=True),
}


def workload(idx: int, **overrides) -> Workload:
    """Workload ``idx`` with optional field overrides (smaller T for quick cases, etc.)."""
    return dataclasses.replace(WORKLOADS[idx], **overrides)


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(entropy=seed, spawn_key=tuple(key))))


def to_storage(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Cast float32 data to the storage type with torch's own conversion."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t if dtype == "f32" else t.to(torch.bfloat16)


def cluster_ids(positions: np.ndarray, hash_mod: int, clusters: int) -> np.ndarray:
    """cluster(t) = (t * 7919 mod P) mod C for absolute positions t."""
    p = np.asarray(positions, dtype=np.int64)
    return ((p * 7919) % hash_mod) % clusters


def shared_mu(w: Workload, layer: int, head: int, kv: int) -> np.ndarray:
    """Per-(layer, kv head, K/V) shared component: random direction of norm ``mu_norm`` (float32)."""
    g = _rng(w.seed, ROLE_MU, layer, 0, head, kv).standard_normal(w.head_dim)
    return (g / np.linalg.norm(g) * w.mu_norm).astype(np.float32)


def centers(w: Workload, layer: int, head: int, kv: int) -> np.ndarray:
    return _rng(w.seed, ROLE_CENTERS, layer, 0, head, kv).standard_normal((w.clusters, w.head_dim)).astype(
        np.float32)


def basis(w: Workload, layer: int, head: int, kv: int, rank: Optional[int] = None) -> np.ndarray:
    """Orthonormal d x r basis: QR of a Gaussian matrix with column signs fixed so diag(R) > 0 (float64)."""
    r = w.rank if rank is None else rank
    g = _rng(w.seed, ROLE_BASIS, layer, 0, head, kv).standard_normal((w.head_dim, r))
    qm, rm = np.linalg.qr(g)
    return qm * np.sign(np.diag(rm))[None, :]


def seq_lengths(w: Workload) -> np.ndarray:
    """Context length of each sequence (log-uniform for ragged mixes)."""
    if not w.ragged:
        return np.full(w.batch, w.seq_len, dtype=np.int64)
    u = _rng(w.seed, ROLE_LENS, 0, 0, 0, 0).random(w.batch)
    lens = np.exp(np.log(w.min_len) + u * (np.log(w.seq_len) - np.log(w.min_len)))
    return np.floor(lens).astype(np.int64)


def raw_kv_np(w: Workload, layer: int, seq: int, head: int, kv: int, t0: int, t1: int) -> np.ndarray:
    """float32 [t1-t0, d] raw K (kv=0) or V (kv=1) rows for absolute positions t0..t1-1 (before storage cast).

    The noise stream is keyed by (layer, seq, head, kv) and drawn for positions 0..t1-1, so a row does not
    depend on how the positions are split into calls.
    """
    mu = shared_mu(w, layer, head, kv)
    c = centers(w, layer, head, kv)
    noise = _rng(w.seed, ROLE_NOISE, layer, seq, head, kv).standard_normal((t1, w.head_dim))[t0:t1]
    cid = cluster_ids(np.arange(t0, t1), w.hash_mod, w.clusters)
    return (mu[None, :] + c[cid] + np.float32(w.sigma) * noise.astype(np.float32)).astype(np.float32)


def kv_tokens(w: Workload, layer: int, seq: int, t0: int, t1: int, backend: str = "numpy",
              device: str = "cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """K and V of one sequence for positions t0..t1-1, token-major ``[n, H_kv, d]`` in storage dtype.

    backend "numpy": PCG64 streams (reproducible on any host).  backend "torch": noise from
    ``torch.randn`` on ``device`` with a generator seeded from the same key (for workloads too large to
    draw on the host); centres and mu still come from the NumPy streams.
    """
    n, H, d = t1 - t0, w.num_kv_heads, w.head_dim
    if backend == "numpy":
        out = []
        for kv in (KEY, VALUE):
            rows = np.stack([raw_kv_np(w, layer, seq, h, kv, t0, t1) for h in range(H)], axis=1)
            out.append(to_storage(rows, w.dtype).to(device))
        return out[0], out[1]
    out = []
    pos = torch.arange(t0, t1, device=device, dtype=torch.int64)
    cid = ((pos * 7919) % w.hash_mod) % w.clusters
    for kv in (KEY, VALUE):
        x = torch.empty((n, H, d), device=device, dtype=torch.float32)
        for h in range(H):
            gen = torch.Generator(device=device)
            gen.manual_seed(int(np.random.SeedSequence(entropy=w.seed, spawn_key=(ROLE_NOISE, layer, seq, h, kv))
                                .generate_state(1, np.uint64)[0] & 0x7FFFFFFFFFFFFFFF))
            noise = torch.randn((t1, d), generator=gen, device=device, dtype=torch.float32)[t0:t1]
            mu = torch.from_numpy(shared_mu(w, layer, h, kv)).to(device)
            c = torch.from_numpy(centers(w, layer, h, kv)).to(device)
            x[:, h, :] = mu[None, :] + c[cid] + w.sigma * noise
        out.append(x if w.dtype == "f32" else x.to(torch.bfloat16))
    return out[0], out[1]


def params(w: Workload, layer: int, rank: Optional[int] = None) -> tuple[torch.Tensor, torch.Tensor]:
    """(mu [H_kv, 2, d] float32, basis [H_kv, 2, d, r] storage dtype) for one layer."""
    r = w.rank if rank is None else rank
    mu = np.stack([np.stack([shared_mu(w, layer, h, kv) for kv in (KEY, VALUE)]) for h in range(w.num_kv_heads)])
    bs = np.stack([np.stack([basis(w, layer, h, kv, r) for kv in (KEY, VALUE)]) for h in range(w.num_kv_heads)])
    return torch.from_numpy(mu.astype(np.float32)), to_storage(bs.astype(np.float32), w.dtype)


def queries(w: Workload, layer: int, seq: int) -> torch.Tensor:
    """Decode queries ``[queries_per_seq, H_q, d]`` ~ N(0, 1) in storage dtype."""
    g = _rng(w.seed, ROLE_QUERY, layer, seq, 0, 0).standard_normal((w.queries_per_seq, w.num_q_heads, w.head_dim))
    return to_storage(g.astype(np.float32), w.dtype)


def block_tables(w: Workload, lens: np.ndarray, extra_tokens: int = 0) -> tuple[np.ndarray, int]:
    """Block tables ``[batch, max_blocks]`` (int32, -1 = unused) and the pool size.

    Each sequence gets ceil((len + extra_tokens) / R) blocks.  Contiguous workloads use identity placement
    (sequence s owns a consecutive range); paged mixes place blocks at a seeded random permutation of the pool.
    """
    R = w.ref_stride
    nb = [(int(L) + extra_tokens + R - 1) // R for L in lens]
    total, mx = sum(nb), max(nb) if nb else 0
    ids = np.arange(total, dtype=np.int64)
    if w.paged_random:
        ids = _rng(w.seed, ROLE_PERM, 0, 0, 0, 0).permutation(total)
    bt = np.full((len(lens), max(mx, 1)), -1, dtype=np.int32)
    off = 0
    for s, n in enumerate(nb):
        bt[s, :n] = ids[off:off + n]
        off += n
    return bt, total


def log_uniform_note(w: Workload) -> str:
    lens = seq_lengths(w)
    return f"{len(lens)} seqs, sum {int(lens.sum())}, mean {lens.mean():.0f}, min {lens.min()}, max {lens.max()}"


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def n_refs(T: int, R: int) -> int:
    return ceil_div(T, R) if T > 0 else 0


__all__ = [name for name in dir() if not name.startswith("_") and name not in ("annotations", "math")]
