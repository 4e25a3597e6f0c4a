"""Benchmark of the DeltaKV hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2] [--impl ours|reference]

One step is one pass of the whole path over one batch:
  - workloads 0..3: compress every sequence's full prefix (centre, search, codes) for every layer, then one
    decode-attention step over the compressed cache for every layer;
  - workload 4 (paged serving mix): one decode step of the 64-sequence continuous batch on the main stream
    while a newly arriving 2048-token prefill is compressed into the same block pool on a second stream
    (the 64 prefixes are compressed once before timing).

Prints one JSON line (rank 0).  ``value`` is decode throughput: sequences decoded per second over all layers
(batch / device time of the decode part of a step), summed over ranks (each rank runs an independent replica
on its own sequences: weak scaling, no collective on the data path).  Compress throughput is the separate
``compress`` key (token-layers per second).  Both come from the same K timed steps: the steps are one CUDA
graph with event nodes at the phase boundaries.  Inputs are resident in HBM when the timed region starts and
larger than the 126 MB L2 (one layer's K+V is 1.07 GB on the default workload), so L2 is not flushed.
``e2e`` is decode throughput through the public API with each step's queries copied from pinned host memory
and each layer's output read back, inside the timed region.  ``roofline`` is the search kernel (the dominant
kernel of a step) and carries the decode path beside it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from residual_kv_cache_delta_b200 import synth  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "search_traffic.json")
CSRC = os.path.join(ROOT, "residual_kv_cache_delta_b200", "csrc")
# device code the search kernel is built from: compress.cuh up to its host-side launch code, and common.cuh
KERNEL_SRC = ((os.path.join(CSRC, "compress.cuh"), "// Host side."), (os.path.join(CSRC, "common.cuh"), None))
METRIC = "decode tok/s over compressed KV (HBM GB/s, % peak); compress tokens/s"
KERNEL_NAMES = ("center", "refprep", "search", "decode_prologue", "decode_split", "decode_combine")
PROFILED_KERNELS = tuple(range(len(KERNEL_NAMES)))
DEFAULT_WORKLOAD = 2  # the largest single-GPU workload: 32 layers x 8 sequences x 32768 tokens
PREFILL_SEQS = 16     # distinct arriving prefills of the serving mix, cycled over the steps


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS),
                   help="index of the synthetic workload")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--layers", type=int, default=None, help="override the workload's layer count (smaller cases)")
    p.add_argument("--select", type=float, default=None,
                   help="decode over a seeded random fraction of each sequence's positions (sparse entry point)")
    p.add_argument("--q4", action="store_true", help="4-bit residual codes (dtype DKV_BF16_Q4)")
    p.add_argument("--topk", type=int, default=0, choices=[0, 1, 2, 4],
                   help="the k-nearest L2 retrieval (deltakv_compress_topk / deltakv_decode_attention_topk)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--append", action="store_true",
                   help="also report the compress latency of 1-, 16- and 2048-token appends at a 131072-token context")
    return p.parse_args(argv)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def shard_sequences(rank: int, batch: int) -> list:
    """Sequence ids of one rank's replica: every (sequence, layer, kv head) is independent, so rank k
    simply owns sequences k*batch .. k*batch + batch - 1 of the job (weak scaling, no data exchange)."""
    return [rank * batch + s for s in range(batch)]


def max_over_ranks(x: float, device, world: int) -> float:
    """Maximum of a per-rank time over all ranks (the job's time is its slowest rank's)."""
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------------------
# Algorithmic work (closed form)
# ------------------------------------------------------------------------------------------------
def search_pairs(T: int, R: int, start: int = 0) -> int:
    """sum over non-reference positions t in [start, T) of ceil(t / R) (causal token-reference pairs)."""
    t = np.arange(start, T, dtype=np.int64)
    t = t[t % R != 0]
    return int(np.sum((t + R - 1) // R))


def search_flops(w: synth.Workload, T: int) -> int:
    """Per (sequence, layer, kv head): 2*(2d) per pair for the scores + 2*(2d)*r per token for the projection."""
    d2 = 2 * w.head_dim
    return 2 * d2 * search_pairs(T, w.ref_stride) + 2 * d2 * w.rank * T


def code_bytes(w: synth.Workload, q4: bool = False) -> int:
    """Bytes of one token's codes: 2r storage values, or r bytes of 4-bit levels and two bf16 scales."""
    return w.rank + 4 if q4 else 2 * w.rank * w.elem_bytes


def decode_bytes(w: synth.Workload, T: int, q4: bool = False, topk: int = 0) -> int:
    """Per (sequence, layer, kv head): codes + index slots per token, the K and V reference rows, the block
    table, the parameters (mu in fp32, the basis in storage precision), and the queries / outputs of the head
    group."""
    es, d, r, R, G = w.elem_bytes, w.head_dim, w.rank, w.ref_stride, w.group
    n_ref = -(-T // R)
    return (T * (code_bytes(w, q4) + 4 * max(topk, 1)) + n_ref * 2 * d * es + n_ref * 4 + 2 * d * 4 + 2 * d * r * es
            + 2 * G * d * es)


def decode_bytes_sparse(w: synth.Workload, T: int, n_sel: int) -> int:
    """Per (sequence, layer, kv head) of a sparse decode over n_sel listed positions: each listed token's codes,
    index, list entry and block-table entry, every K and V reference row of the context (a listed token may point
    at any of them), the parameters, and the queries / outputs of the head group."""
    es, d, r, R, G = w.elem_bytes, w.head_dim, w.rank, w.ref_stride, w.group
    n_ref = -(-T // R)
    return n_sel * (2 * r * es + 4 + 4 + 4) + n_ref * 2 * d * es + 2 * d * 4 + 2 * d * r * es + 2 * G * d * es


def decode_split_bytes(w: synth.Workload, T: int, q4: bool = False, topk: int = 0) -> int:
    """Per (sequence, layer, kv head): what the split kernel alone must stream (codes, indices, block table)."""
    return T * (code_bytes(w, q4) + 4 * max(topk, 1)) + (-(-T // w.ref_stride)) * 4


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained") or p["bf16_tflops"], "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def kernel_src_hash() -> str:
    """Hash of the search kernel's device source (comments and blank lines removed), so that a stored ncu
    traffic figure is dropped once that code changes, and survives changes to commentary or host code."""
    lines = []
    for path, stop in KERNEL_SRC:
        with open(path) as f:
            for ln in f:
                if stop is not None and ln.startswith(stop):
                    break
                ln = ln.split("//", 1)[0].rstrip()
                if ln:
                    lines.append(ln)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()[:16]


def search_traffic(w: synth.Workload, lens) -> float | None:
    """DRAM bytes of one search-kernel launch of this workload's layer, from the stored ncu capture.

    The capture is of one (sequence, kv head)-uniform launch; its bytes are scaled by the number of
    (sequence, kv head) units when this workload has the same per-unit shape (T, R, r, d), since the kernel's
    traffic grows in proportion to the units.  None when the kernel source changed since the capture, or the
    per-unit shape differs."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        tr = json.load(f)
    if tr.get("kernel_src_sha256_16") != kernel_src_hash():
        return None
    unit = tr.get("unit", {})
    if any(int(x) != unit.get("seq_len") for x in lens):
        return None
    if (unit.get("ref_stride"), unit.get("rank"), unit.get("head_dim")) != (w.ref_stride, w.rank, w.head_dim):
        return None
    return tr["bytes_per_launch"] / tr["units"] * len(lens) * w.num_kv_heads


# ------------------------------------------------------------------------------------------------
# Clock sampling during the timed region
# ------------------------------------------------------------------------------------------------
class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-i", str(self.dev), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# CPU oracle timing (baseline leg and reference arm)
# ------------------------------------------------------------------------------------------------
def seq_lens(w: synth.Workload) -> list:
    return [int(x) for x in synth.seq_lengths(w)]


ORACLE_SAMPLE_TOKENS = 32768  # longest prefix the oracle sample compresses (about 5-20 s on 8-16 host cores)


def oracle_sample_len(w: synth.Workload) -> int:
    return min(seq_lens(w)[0], ORACLE_SAMPLE_TOKENS)


def decode_units(w: synth.Workload) -> float:
    """(sequence, layer, kv head) decode units of one step in multiples of the oracle sample (the first
    ``oracle_sample_len`` tokens of sequence 0, one kv head): decode time grows linearly with the context."""
    return w.layers * w.num_kv_heads * sum(seq_lens(w)) / oracle_sample_len(w)


def oracle_setup(w: synth.Workload):
    """Inputs of the oracle sample: a prefix of sequence 0, layer 0, kv head 0 and its query-head group."""
    T = oracle_sample_len(w)
    k, v = synth.kv_tokens(w, 0, 0, 0, T)
    mu, bs = synth.params(w, 0)
    q = synth.queries(w, 0, 0)[0]
    h = 0
    return dict(k=k[:, h].double().numpy(), v=v[:, h].double().numpy(), mk=mu[h, 0].numpy(), mv=mu[h, 1].numpy(),
                BK=bs[h, 0].double().numpy(), BV=bs[h, 1].double().numpy(), mu=mu[:1].numpy(),
                q=q[: w.group].double().numpy(), T=T)


def oracle_compress(w, s):
    import oracle.deltakv_oracle as O
    t0 = time.perf_counter()
    st = O.compress(s["k"], s["v"], s["mk"], s["mv"], s["BK"], s["BV"], w.ref_stride, w.dtype)
    return time.perf_counter() - t0, st


def oracle_decode(w, s, st, select=None):
    """Seconds of one oracle decode of the sample (dense, or over a seeded random ``select`` fraction of it)."""
    import oracle.deltakv_oracle as O
    refs, idx, cds, _ = st
    args = (s["q"], s["mu"], [refs], [idx], [cds], s["BK"][None], s["BV"][None])
    if select is not None:
        sel = np.sort(np.random.default_rng(10007).choice(s["T"], max(1, int(round(select * s["T"]))), replace=False))
    t0 = time.perf_counter()
    if select is None:
        O.decode(*args, w.dtype)
    else:
        O.decode_sparse(*args, sel, w.dtype)
    return time.perf_counter() - t0


def oracle_sample_desc(w, s) -> str:
    return (f"oracle on the first {s['T']} tokens of sequence 0, layer 0, kv head 0 with its {w.group} query "
            f"heads; decode time scaled by {decode_units(w):.1f} sample-sized units per step (the step's "
            f"sum over layers, kv heads and sequences of context length / {s['T']}); compress rate = sample "
            f"tokens / (sample time x {w.num_kv_heads} kv heads)")


def oracle_rates(w, t_compress: float, t_decode: float, sample_tokens: int) -> tuple:
    """(decode tok/s, compress token-layers/s) that the oracle's per-unit times imply for the whole step.

    Decode: one step decodes every sequence once, which is ``decode_units`` units of the sampled one.
    Compress: the sample compresses ``sample_tokens`` tokens of one of the H kv heads of one layer."""
    return w.batch / (t_decode * decode_units(w)), sample_tokens / (t_compress * w.num_kv_heads)


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [x.get("num_threads", 1) for x in threadpool_info() if x.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def run_reference(args, w):
    """The reference arm: the CPU oracle as it stands, on a bounded sample of the same workload.  Each step is
    the oracle's decode of one (sequence, layer, kv head) unit (measured, reported as ms_per_step); the value
    scales it to the whole step's units, stated in ``sample_scale``."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    s = oracle_setup(w)
    t_c, st = oracle_compress(w, s)
    for _ in range(max(0, args.warmup)):
        oracle_decode(w, s, st)
    steps = max(1, args.steps)
    dts = [oracle_decode(w, s, st) for _ in range(steps)]
    t_d = float(np.mean(dts))
    dec, cmp = oracle_rates(w, t_c, t_d, s["T"])
    line = {"metric": METRIC, "value": dec, "unit": "tok/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": steps, "warmup": args.warmup, "ms_per_step": t_d * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "layers": w.layers, "batch": w.batch, "seq_len": w.seq_len},
            "sample_scale": {"units_per_step": decode_units(w), "unit": "(sequence, layer, kv head) decode",
                             "step_is": "one unit's decode; value = batch / (ms_per_step x units_per_step)"},
            "compress": {"tokens_per_s": cmp, "sample_s": t_c, "sample_tokens": s["T"]},
            "cpu_baseline": {"value": dec, "unit": "tok/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": oracle_sample_desc(w, s)},
            "e2e": {"value": dec, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# Our arm
# ------------------------------------------------------------------------------------------------
class Replica:
    """All device state of one rank's replica of the workload."""

    def __init__(self, w: synth.Workload, rank: int, device, select: float | None = None, q4: bool = False,
                 topk: int = 0):
        from residual_kv_cache_delta_b200 import deltakv as D
        self.D, self.w, self.dev, self.q4, self.topk = D, w, device, q4, topk
        self.shape = D.Shape(w.num_q_heads, w.num_kv_heads, w.head_dim, w.rank, w.ref_stride, w.torch_dtype, q4=q4)
        B, H = w.batch, w.num_kv_heads
        self.lens = seq_lens(w)
        T = max(self.lens)
        self.max_ctx = T
        self.total = int(sum(self.lens))
        big = w.layers * self.total * H * w.head_dim > 2**31
        backend = "torch" if big else "numpy"
        seqs = shard_sequences(rank, B)
        self.n_prefill = PREFILL_SEQS if w.prefill_len > 0 else 0
        plen = [w.prefill_len] * self.n_prefill
        bt, nb = synth.block_tables(w, np.array(self.lens + plen))
        self.bt = torch.from_numpy(bt[:B]).to(device)
        self.bt_pre = [torch.from_numpy(bt[B + i: B + i + 1]).to(device) for i in range(self.n_prefill)]
        self.k, self.v, self.mu, self.basis, self.cache, self.q = [], [], [], [], [], []
        for layer in range(w.layers):
            ks, vs = [], []
            for s, T_s in zip(seqs, self.lens):
                k, v = synth.kv_tokens(w, layer, s, 0, T_s, backend=backend, device=device)
                ks.append(k.to(device))
                vs.append(v.to(device))
            self.k.append(torch.cat(ks))
            self.v.append(torch.cat(vs))
            mu, bs = synth.params(w, layer)
            self.mu.append(mu.to(device))
            self.basis.append(bs.to(device))
            self.cache.append(D.alloc_cache(self.shape, nb, device, topk=topk))
            self.q.append(torch.cat([synth.queries(w, layer, s)[:1] for s in seqs]).to(device))
        self.cu = torch.tensor(np.concatenate([[0], np.cumsum(self.lens)]), dtype=torch.int32, device=device)
        self.start = torch.zeros(B, dtype=torch.int32, device=device)
        self.ctx = torch.tensor(self.lens, dtype=torch.int32, device=device)
        self.ws_c = D.alloc_workspace(D.compress_workspace(self.shape, B, self.total, T, T), device)
        self.select = select
        if select is not None:  # seeded random selection of each sequence's positions, sorted
            rng = np.random.default_rng(10007 + rank)
            self.lists = [np.sort(rng.choice(L, max(1, int(round(select * L))), replace=False)) for L in self.lens]
            self.n_sel = [len(x) for x in self.lists]
            self.max_sel = max(self.n_sel)
            self.tok = torch.tensor(np.concatenate(self.lists), dtype=torch.int32, device=device)
            self.cu_tok = torch.tensor(np.concatenate([[0], np.cumsum(self.n_sel)]), dtype=torch.int32, device=device)
            self.ws_d = D.alloc_workspace(D.decode_sparse_workspace(self.shape, B, T, self.max_sel), device)
        elif topk > 0:
            self.ws_d = D.alloc_workspace(D.decode_topk_workspace(self.shape, topk, B, T), device)
        else:
            self.ws_d = D.alloc_workspace(D.decode_workspace(self.shape, B, T), device)
        self.out = torch.empty((B, w.num_q_heads, w.head_dim), dtype=w.torch_dtype, device=device)
        self.lse = torch.empty((B, w.num_q_heads), dtype=torch.float32, device=device)
        if self.n_prefill:
            P = w.prefill_len
            self.pk, self.pv = [], []
            for i in range(self.n_prefill):
                k, v = synth.kv_tokens(w, 0, 10**6 + rank * PREFILL_SEQS + i, 0, P, backend=backend, device=device)
                self.pk.append(k.to(device))
                self.pv.append(v.to(device))
            self.pcu = torch.tensor([0, P], dtype=torch.int32, device=device)
            self.pstart = torch.zeros(1, dtype=torch.int32, device=device)
            self.ws_p = D.alloc_workspace(D.compress_workspace(self.shape, 1, P, P, P), device)
            self.side = torch.cuda.Stream(device=device)
        self.step_no = 0

    # one step's launches: 3 per compress call (centre, reference prep, search) and 3 per decode call
    # (prologue, split, combine); memsets are not counted
    @property
    def launches_per_step(self) -> int:
        return 6 if self.n_prefill else self.w.layers * 6

    def compress_all(self):
        D, w = self.D, self.w
        for layer in range(w.layers):
            if self.topk > 0:
                D.deltakv_compress_topk(self.shape, self.topk, self.mu[layer], self.basis[layer], self.cache[layer],
                                        self.k[layer], self.v[layer], self.cu, self.start, self.bt, self.max_ctx,
                                        self.max_ctx, self.ws_c)
            else:
                D.deltakv_compress(self.shape, self.mu[layer], self.basis[layer], self.cache[layer], self.k[layer],
                                   self.v[layer], self.cu, self.start, self.bt, self.max_ctx, self.max_ctx, self.ws_c)

    def decode_layer(self, layer: int):
        D = self.D
        if self.topk > 0:
            D.deltakv_decode_attention_topk(self.shape, self.topk, self.mu[layer], self.basis[layer], self.cache[layer],
                                            self.q[layer], self.ctx, self.bt, self.max_ctx, self.out, self.lse,
                                            self.ws_d)
        elif self.select is None:
            D.deltakv_decode_attention(self.shape, self.mu[layer], self.basis[layer], self.cache[layer],
                                       self.q[layer], self.ctx, self.bt, self.max_ctx, self.out, self.lse, self.ws_d)
        else:
            D.deltakv_decode_attention_sparse(self.shape, self.mu[layer], self.basis[layer], self.cache[layer],
                                              self.q[layer], self.ctx, self.bt, self.tok, self.cu_tok, self.max_sel,
                                              self.max_ctx, self.out, self.lse, self.ws_d)

    def decode_all(self):
        for layer in range(self.w.layers):
            self.decode_layer(layer)

    def prefill(self, i: int, stream):
        D, P = self.D, self.w.prefill_len
        D.deltakv_compress(self.shape, self.mu[0], self.basis[0], self.cache[0], self.pk[i], self.pv[i], self.pcu,
                           self.pstart, self.bt_pre[i], P, P, self.ws_p, stream=stream)

    def step(self, ev=None):
        """One step.  ``ev``: optional list of external events [start, compress done, decode done (, prefill
        start, prefill done)] recorded at the phase boundaries."""
        main = torch.cuda.current_stream()
        if ev is not None:
            ev[0].record(main)
        if not self.n_prefill:
            self.compress_all()
            if ev is not None:
                ev[1].record(main)
            self.decode_all()
            if ev is not None:
                ev[2].record(main)
        else:
            i = self.step_no % self.n_prefill
            self.step_no += 1
            self.side.wait_stream(main)
            with torch.cuda.stream(self.side):
                if ev is not None:
                    ev[3].record(self.side)
                self.prefill(i, self.side)
                if ev is not None:
                    ev[4].record(self.side)
            if ev is not None:
                ev[1].record(main)
            self.decode_all()
            if ev is not None:
                ev[2].record(main)
            main.wait_stream(self.side)

    def setup(self):
        """Workload 4: the 64 prefixes are compressed once before timing (decode reads them every step)."""
        if self.n_prefill:
            self.compress_all()


def _events(n):
    return [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n)]


def append_latency(D, device, ctx: int = 131072, sizes=(2048, 16, 1), reps: int = 20) -> dict:
    """Device time of one compress call that appends n tokens to a sequence of ctx - n tokens, for each n in sizes
    (Llama-3-8B head geometry: 8 kv heads, d = 128, r = 32, R = 16; one sequence).  The prefix is compressed once;
    each call is timed as the mean of `reps` back-to-back calls of the same n tokens in one CUDA graph, each of
    which rewrites the same cache rows with the same values.  Calls of at most 16 tokens take the append path (search and codes on
    CUDA cores over the paged reference rows), longer ones the reference prep and the tensor-core search."""
    w = synth.workload(1, seq_len=ctx, seed=17)
    shape = D.Shape(w.num_q_heads, w.num_kv_heads, w.head_dim, w.rank, w.ref_stride, w.torch_dtype)
    mu, basis = (x.to(device) for x in synth.params(w, 0))
    k, v = synth.kv_tokens(w, 0, 0, 0, ctx, backend="torch", device=device)
    bt, nb = synth.block_tables(w, np.array([ctx]))
    btd = torch.from_numpy(bt).to(device)
    cache = D.alloc_cache(shape, nb, device)

    def args_of(a, b):
        return (torch.tensor([0, b - a], dtype=torch.int32, device=device),
                torch.tensor([a], dtype=torch.int32, device=device))

    def call(a, b, ws, cu, sp):
        D.deltakv_compress(shape, mu, basis, cache, k[a:b], v[a:b], cu, sp, btd, b - a, ctx, ws)

    p0 = ctx - max(sizes)
    call(0, p0, D.alloc_workspace(D.compress_workspace(shape, 1, p0, p0, ctx), device), *args_of(0, p0))
    out = {}
    for n in sorted(sizes, reverse=True):
        ws = D.alloc_workspace(D.compress_workspace(shape, 1, n, n, ctx), device)
        cu, sp = args_of(ctx - n, ctx)
        for _ in range(3):
            call(ctx - n, ctx, ws, cu, sp)
        torch.cuda.synchronize()
        # the reps calls as one CUDA graph: device time without the host's launch gaps
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                call(ctx - n, ctx, ws, cu, sp)
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        out[str(n)] = e0.elapsed_time(e1) * 1e3 / reps
        del g
    err = D.deltakv_get_device_error()
    if err:
        raise RuntimeError(f"device error word {err}: {D.DEVERR_NAMES.get(err)}")
    return {"context": ctx, "kv_heads": w.num_kv_heads, "batch": 1, "us_per_call": out,
            "what": "device time of one compress call appending n tokens at this context (mean of back-to-back calls in a CUDA graph)"}


def run_ours(args, w):
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    from residual_kv_cache_delta_b200 import build
    if rank == 0:
        build.build()
    if world > 1:
        torch.distributed.barrier()
    from residual_kv_cache_delta_b200 import deltakv as D
    D.load_library()
    if args.topk and (args.q4 or args.select is not None or w.prefill_len):
        raise SystemExit("--topk runs alone (no --q4, --select or serving-mix prefills)")
    rep = Replica(w, rank, device, select=args.select, q4=args.q4, topk=args.topk)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    def check_err():
        err = D.deltakv_get_device_error()
        if err:
            raise RuntimeError(f"device error word {err}: {D.DEVERR_NAMES.get(err)}")

    rep.setup()
    W = max(args.warmup, 3)
    for _ in range(W):
        rep.step()
    torch.cuda.synchronize()
    check_err()

    K = args.steps
    nev = 5 if rep.n_prefill else 3
    evs = [_events(nev) for _ in range(K)]
    # The K timed steps are captured once into a CUDA graph (the library allocates nothing and never
    # synchronises, so its calls capture as plain kernel / memset nodes) and replayed as one launch; event
    # nodes mark each step's phases.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(K):
            rep.step(evs[i])
    graph.replay()  # upload + warm replay
    torch.cuda.synchronize()
    clocks = Clocks(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    del graph
    check_err()
    ms_max = max_over_ranks(ms, device, world)
    dec_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))  # decode part of a step
    cmp_ms = (float(np.mean([e[0].elapsed_time(e[1]) for e in evs])) if not rep.n_prefill
              else float(np.mean([e[3].elapsed_time(e[4]) for e in evs])))
    dec_ms_max = max_over_ranks(dec_ms, device, world)
    cmp_ms_max = max_over_ranks(cmp_ms, device, world)

    # Per-kernel breakdown: a second graph of the same K steps with the library's timing hook, which puts
    # an event pair around every launch of each kernel (kept out of the graph timed above).
    per_step = {k: (w.layers if k >= 3 or not rep.n_prefill else 1) for k in PROFILED_KERNELS}
    timers = {kid: D.KernelTimer(kid, K * per_step[kid]) for kid in PROFILED_KERNELS}
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(K):
            rep.step()
    graph.replay()  # upload + warm replay; the replay below overwrites every event
    torch.cuda.synchronize()
    barrier()
    graph.replay()
    torch.cuda.synchronize()
    barrier()
    kernel_ms = {}
    for kid, t in timers.items():
        times = t.times_ms()
        kernel_ms[kid] = float(np.mean(times)) if times else float("nan")
        t.close()
    del graph

    # Decode alone (workload 4: without the concurrent prefill), for its fraction of HBM in isolation.
    iso_ms = None
    if rep.n_prefill:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(K):
                rep.decode_all()
        g.replay()
        torch.cuda.synchronize()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        g.replay()
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        iso_ms = max_over_ranks(f0.elapsed_time(f1) / K, device, world)
        del g

    # end to end through the public API with host buffers: each step copies every layer's queries from
    # pinned host memory, decodes, and reads every layer's output back
    e2e = None
    if not args.no_e2e:
        hq = [x.cpu().pin_memory() for x in rep.q]
        hout = [torch.empty(rep.out.shape, dtype=rep.out.dtype).pin_memory() for _ in range(w.layers)]
        bi = sum(x.numel() * x.element_size() for x in hq)
        bo = sum(x.numel() * x.element_size() for x in hout)
        E = max(K, 10)
        for it in range(W + E):
            if it == W:
                barrier()
                torch.cuda.synchronize()
                f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                f0.record(stream)
            for layer in range(w.layers):
                rep.q[layer].copy_(hq[layer], non_blocking=True)
                rep.decode_layer(layer)
                hout[layer].copy_(rep.out, non_blocking=True)
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(f0.elapsed_time(f1), device, world)
        e2e = {"value": w.batch * world * E / (e_ms / 1e3), "unit": "tok/s", "h2d_bytes_per_step": bi,
               "d2h_bytes_per_step": bo, "steps": E,
               "what": "decode of every layer through deltakv_decode_attention with q from pinned host memory "
                       "and the output copied back to pinned host memory, per layer and step"}

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    hbm, tf_burst, tf_sust, peak_kind = load_peaks()
    lens = rep.lens
    units = len(lens) * w.num_kv_heads
    # search kernel: flops of one launch (one layer of the prefix compress; workload 4: one prefill)
    if rep.n_prefill:
        flops_launch = w.num_kv_heads * search_flops(w, w.prefill_len)
        traffic = None
    else:
        flops_launch = w.num_kv_heads * sum(search_flops(w, T) for T in lens)
        traffic = search_traffic(w, lens)
    s_ms = kernel_ms[D.KERNEL_SEARCH]
    s_tf = flops_launch / (s_ms / 1e3) / 1e12
    # a step lasts long enough (tens of ms) for the power cap to act: the sustained bf16 figure is the peak
    peak_tf = tf_sust
    if rep.select is None:
        dec_bytes = w.num_kv_heads * sum(decode_bytes(w, T, rep.q4, rep.topk) for T in lens)  # per layer
    else:
        dec_bytes = w.num_kv_heads * sum(decode_bytes_sparse(w, T, n) for T, n in zip(lens, rep.n_sel))
    if rep.select is None:
        split_bytes = w.num_kv_heads * sum(decode_split_bytes(w, T, rep.q4, rep.topk) for T in lens)
    else:  # listed tokens' codes, indices, list entries and block-table entries
        split_bytes = w.num_kv_heads * sum(rep.n_sel) * (2 * w.rank * w.elem_bytes + 12)
    d_path_ms = sum(kernel_ms[k] for k in (D.KERNEL_DECODE_PROLOGUE, D.KERNEL_DECODE_SPLIT, D.KERNEL_DECODE_COMBINE))
    dec_layer_ms = dec_ms_max / w.layers  # device time of one layer's decode inside the timed steps
    dec_gbs = dec_bytes / (dec_layer_ms / 1e3) / 1e9
    split_ms = kernel_ms[D.KERNEL_DECODE_SPLIT]
    cmp_tokens = w.prefill_len if rep.n_prefill else w.layers * rep.total
    line = {
        "metric": METRIC,
        "value": w.batch * world / (dec_ms_max / 1e3),
        "unit": "tok/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": ms_max / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "layers": w.layers, "batch": w.batch, "seq_len": w.seq_len,
                   "kv_heads": w.num_kv_heads, "q_heads": w.num_q_heads, "head_dim": w.head_dim, "rank": w.rank,
                   "ref_stride": w.ref_stride, "parallelism": f"replica-per-gpu x{world}",
                   "context_tokens": rep.total, "prefill_len": w.prefill_len,
                   "codes": "4-bit levels with a bf16 scale per token and K/V half" if rep.q4 else w.dtype,
                   "retrieval": (f"the {rep.topk} nearest references by L2, residual against their mean"
                                 if rep.topk else "cosine top-1"),
                   "decode": "dense" if rep.select is None else
                             f"sparse: a seeded random {rep.select:g} of each sequence's positions "
                             f"({sum(rep.n_sel)} tokens), through deltakv_decode_attention_sparse",
                   "l2": "inputs larger than L2 (one layer's decode reads %.0f MB, compress %.0f MB), no flush" %
                         (dec_bytes / 1e6, rep.k[0].numel() * 4 / 1e6)},
        "value_is": "decode tok/s = batch / device time of the decode part of a step (all layers), max over ranks",
        "decode": {"ms_per_step": dec_ms_max, "ms_per_layer": dec_layer_ms,
                   "algorithmic_bytes_per_layer": dec_bytes, "gbs": dec_gbs, "frac_hbm": dec_gbs / hbm,
                   "kernels_ms_per_layer": d_path_ms, "split_ms_per_launch": split_ms, "split_bytes": split_bytes,
                   "split_gbs": split_bytes / (split_ms / 1e3) / 1e9,
                   "split_frac_hbm": split_bytes / (split_ms / 1e3) / 1e9 / hbm},
        "compress": {"tokens_per_s": cmp_tokens * world / (cmp_ms_max / 1e3), "unit": "token-layers/s",
                     "ms_per_step": cmp_ms_max, "search_ms_per_launch": s_ms, "search_tflops": s_tf},
        "kernel_ms_per_launch": {KERNEL_NAMES[k]: v for k, v in kernel_ms.items()},
        "roofline": {"kernel": "search_tc_kernel", "bound": "tensor", "achieved": s_tf, "peak": peak_tf,
                     "peak_kind": f"bf16 dense sustained, {peak_kind}", "unit": "TFLOP/s", "frac": s_tf / peak_tf,
                     "frac_of_burst": s_tf / tf_burst, "traffic": traffic, "flops_per_launch": flops_launch,
                     "decode": {"kernels": "decode_prologue + decode_split_mma + decode_combine", "bound": "hbm",
                                "achieved": dec_gbs, "peak": hbm, "unit": "GB/s", "frac": dec_gbs / hbm,
                                "bytes_per_launch": dec_bytes, "peak_kind": f"HBM copy, {peak_kind}",
                                "timed": "decode part of the timed steps, per layer"}},
        "gpu_launches": rep.launches_per_step * K,
        "clocks": clk,
    }
    if iso_ms is not None:
        iso_gbs = dec_bytes / (iso_ms / w.layers / 1e3) / 1e9
        line["decode"]["isolated"] = {"ms_per_step": iso_ms, "gbs": iso_gbs, "frac_hbm": iso_gbs / hbm,
                                      "tok_per_s": w.batch * world / (iso_ms / 1e3)}
    if e2e is not None:
        line["e2e"] = e2e
    if args.append and rank == 0:
        line["append"] = append_latency(D, device)
    if not args.no_cpu_baseline:
        s = oracle_setup(w)
        t_c, st = oracle_compress(w, s)
        t_d = float(np.median([oracle_decode(w, s, st, args.select) for _ in range(3)]))
        dec, cmp = oracle_rates(w, t_c, t_d, s["T"])  # a selection scales the sample and the step alike
        line["cpu_baseline"] = {"value": dec, "unit": "tok/s", "cores": cpu_threads(), "kind": "oracle",
                                "sample": oracle_sample_desc(w, s), "compress_tokens_per_s": cmp,
                                "sample_s": {"compress": t_c, "decode": t_d}}
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def main():
    args = parse()
    w = synth.workload(args.workload)
    if args.layers is not None:
        w = synth.dataclasses.replace(w, layers=args.layers, name=f"{w.name}-{args.layers}layer")
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
