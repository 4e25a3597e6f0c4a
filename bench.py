"""Benchmark of the DeltaKV hot path on B200: one step = compress a full prefix (centre, search, codes)
and run one decode-attention step over the compressed cache, for every layer of the workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 1] [--impl ours|reference]

Prints one JSON line (rank 0).  ``value`` is whole-job throughput in tokens/s: (prefix tokens compressed +
tokens decoded) per second, summed over ranks (each rank runs an independent replica of the workload on
its own sequences: weak scaling, no collective on the data path).  Inputs are resident in HBM when the
timed region starts; the K/V inputs of the default workload (134 MB) exceed the 126 MB L2.  ``e2e`` is
the same metric with the inputs copied from pinned host memory and the decode output copied back inside
the timed region.  ``roofline`` is for the dominant kernel (the tensor-core similarity search).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
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


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", type=int, default=1, help="index of the synthetic workload (0..3)")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    return p.parse_args()


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


def decode_bytes(w: synth.Workload, T: int) -> int:
    """Per (sequence, layer, kv head): codes + index per token, the K and V reference rows, the block table,
    the parameters, and the queries / outputs of the head group."""
    es, d, r, R, G = w.elem_bytes, w.head_dim, w.rank, w.ref_stride, w.group
    n_ref = -(-T // R)
    return T * (2 * r * es + 4) + n_ref * 2 * d * es + n_ref * 4 + (2 * d + 2 * d * r) * es + 2 * G * d * es


def decode_split_bytes(w: synth.Workload, T: int) -> int:
    """Per (sequence, layer, kv head): what the split kernel alone must stream (codes, indices, block table)."""
    es, r, R = w.elem_bytes, w.rank, w.ref_stride
    return T * (2 * r * es + 4) + (-(-T // R)) * 4


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained"), "measured"
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
def cpu_oracle_sample(w: synth.Workload, seq_len: int):
    """Times the oracle (as it stands) on one kv head of one layer over the full prefix plus the decode of its
    query-head group; returns (seconds, tokens that sample represents of the full step, description)."""
    import oracle.deltakv_oracle as O
    k, v = synth.kv_tokens(w, 0, 0, 0, seq_len)
    mu, bs = synth.params(w, 0)
    q = synth.queries(w, 0, 0)[0]
    h = 0
    kk, vv = k[:, h].double().numpy(), v[:, h].double().numpy()
    BK, BV = bs[h, 0].double().numpy(), bs[h, 1].double().numpy()
    t0 = time.perf_counter()
    refs, idx, cds, _ = O.compress(kk, vv, mu[h, 0].numpy(), mu[h, 1].numpy(), BK, BV, w.ref_stride, w.dtype)
    O.decode(q[: w.group].double().numpy(), mu[:1].numpy(), [refs], [idx], [cds], BK[None], BV[None], w.dtype)
    dt = time.perf_counter() - t0
    frac = 1.0 / w.num_kv_heads  # one kv head of the layer
    desc = (f"oracle on kv head 0 of {w.num_kv_heads}, layer 0 of {w.layers}, sequence 0 of {w.batch}: compress "
            f"{seq_len} tokens + decode {w.group} query heads; scaled by {w.num_kv_heads * w.layers * w.batch}")
    return dt, frac, desc


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [x.get("num_threads", 1) for x in threadpool_info() if x.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def tokens_per_step(w: synth.Workload) -> int:
    return w.layers * w.batch * (w.seq_len + 1)


def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    steps = max(1, min(args.steps, 3))
    dt_all = []
    for _ in range(max(0, min(args.warmup, 1))):
        cpu_oracle_sample(w, w.seq_len)
    for _ in range(steps):
        dt, frac, desc = cpu_oracle_sample(w, w.seq_len)
        dt_all.append(dt)
    dt = float(np.mean(dt_all))
    per_step_equiv = dt / frac * w.layers * w.batch  # seconds the oracle would need for one whole step
    value = tokens_per_step(w) / per_step_equiv
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": steps, "warmup": args.warmup, "ms_per_step": per_step_equiv * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "layers": w.layers, "batch": w.batch, "seq_len": w.seq_len},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# Our arm
# ------------------------------------------------------------------------------------------------
class Replica:
    """All device state of one rank's replica of the workload."""

    def __init__(self, w: synth.Workload, rank: int, device):
        from residual_kv_cache_delta_b200 import deltakv as D
        self.D, self.w, self.dev = D, w, device
        self.shape = D.Shape(w.num_q_heads, w.num_kv_heads, w.head_dim, w.rank, w.ref_stride, w.torch_dtype)
        T, B, H = w.seq_len, w.batch, w.num_kv_heads
        big = w.layers * B * T * H * w.head_dim > 2**31
        backend = "torch" if big else "numpy"
        self.k, self.v, self.mu, self.basis, self.cache, self.q = [], [], [], [], [], []
        lens = np.full(B, T)
        bt, nb = synth.block_tables(w, lens)
        self.bt = torch.from_numpy(bt).to(device)
        seqs = shard_sequences(rank, B)
        for layer in range(w.layers):
            ks, vs = [], []
            for s in seqs:
                k, v = synth.kv_tokens(w, layer, s, 0, T, backend=backend, device=device)
                ks.append(k.to(device))
                vs.append(v.to(device))
            self.k.append(torch.cat(ks))
            self.v.append(torch.cat(vs))
            mu, bs = synth.params(w, layer)
            self.mu.append(mu.to(device))
            self.basis.append(bs.to(device))
            self.cache.append(D.alloc_cache(self.shape, nb, device))
            self.q.append(torch.cat([synth.queries(w, layer, s)[:1] for s in seqs]).to(device))
        self.cu = torch.arange(0, (B + 1) * T, T, dtype=torch.int32, device=device)
        self.start = torch.zeros(B, dtype=torch.int32, device=device)
        self.ctx = torch.full((B,), T, dtype=torch.int32, device=device)
        self.ws_c = D.alloc_workspace(D.compress_workspace(self.shape, B, B * T, T, T), device)
        self.ws_d = D.alloc_workspace(D.decode_workspace(self.shape, B, T), device)
        self.out = torch.empty((B, w.num_q_heads, w.head_dim), dtype=w.torch_dtype, device=device)
        self.lse = torch.empty((B, w.num_q_heads), dtype=torch.float32, device=device)
        self.launches_per_step = w.layers * (3 + 3)  # centre, refprep, search; prologue, split, combine

    def step(self, k=None, v=None):
        D, w = self.D, self.w
        for layer in range(w.layers):
            D.deltakv_compress(self.shape, self.mu[layer], self.basis[layer], self.cache[layer],
                               self.k[layer] if k is None else k, self.v[layer] if v is None else v, self.cu,
                               self.start, self.bt, w.seq_len, w.seq_len, self.ws_c)
        for layer in range(w.layers):
            D.deltakv_decode_attention(self.shape, self.mu[layer], self.basis[layer], self.cache[layer], self.q[layer],
                                       self.ctx, self.bt, w.seq_len, self.out, self.lse, self.ws_d)


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
    rep = Replica(w, rank, device)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(max(args.warmup, 3)):
        rep.step()
    torch.cuda.synchronize()
    err = D.deltakv_get_device_error()
    if err:
        raise RuntimeError(f"device error word {err}: {D.DEVERR_NAMES.get(err)}")

    K = args.steps
    # The K timed steps are captured once into a CUDA graph (the library allocates nothing and never
    # synchronises, so its calls capture as plain kernel / memset nodes) and replayed as one launch.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(K):
            rep.step()
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
    err = D.deltakv_get_device_error()
    if err:
        raise RuntimeError(f"device error word {err}: {D.DEVERR_NAMES.get(err)}")
    ms_max = max_over_ranks(ms, device, world)

    # Per-kernel breakdown: a second graph of the same K steps with the library's timing hook, which puts
    # an event pair around every launch of each kernel (kept out of the graph timed above).
    timers = {kid: D.KernelTimer(kid, K * w.layers) for kid in PROFILED_KERNELS}
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
    search_ms = [kernel_ms[D.KERNEL_SEARCH]]
    split_ms = [kernel_ms[D.KERNEL_DECODE_SPLIT]]

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        hk = [x.cpu().pin_memory() for x in rep.k]
        hv = [x.cpu().pin_memory() for x in rep.v]
        hq = [x.cpu().pin_memory() for x in rep.q]
        hout = torch.empty(rep.out.shape, dtype=rep.out.dtype).pin_memory()
        dk = [torch.empty_like(x) for x in rep.k]
        dv = [torch.empty_like(x) for x in rep.v]
        bi = sum(x.numel() * x.element_size() for x in hk + hv + hq)
        bo = hout.numel() * hout.element_size() * w.layers
        for it in range(max(args.warmup, 3) + K):
            if it == max(args.warmup, 3):
                barrier()
                torch.cuda.synchronize()
                f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                f0.record(stream)
            for layer in range(w.layers):
                dk[layer].copy_(hk[layer], non_blocking=True)
                dv[layer].copy_(hv[layer], non_blocking=True)
                rep.q[layer].copy_(hq[layer], non_blocking=True)
                D.deltakv_compress(rep.shape, rep.mu[layer], rep.basis[layer], rep.cache[layer], dk[layer], dv[layer],
                                   rep.cu, rep.start, rep.bt, w.seq_len, w.seq_len, rep.ws_c)
            for layer in range(w.layers):
                D.deltakv_decode_attention(rep.shape, rep.mu[layer], rep.basis[layer], rep.cache[layer],
                                           rep.q[layer], rep.ctx, rep.bt, w.seq_len, rep.out, rep.lse, rep.ws_d)
                hout.copy_(rep.out, non_blocking=True)
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(f0.elapsed_time(f1), device, world)
        e2e = {"value": tokens_per_step(w) * world * K / (e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo}

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    hbm, tf_burst, tf_sust, peak_kind = load_peaks()
    flops_launch = w.batch * w.num_kv_heads * search_flops(w, w.seq_len)
    s_ms = float(np.mean(search_ms)) if search_ms else float("nan")
    achieved = flops_launch / (s_ms / 1e3) / 1e12
    traffic = None
    if os.path.exists(TRAFFIC_FILE):
        with open(TRAFFIC_FILE) as f:
            tr = json.load(f)
        if tr.get("kernel_src_sha256_16") == kernel_src_hash() and tr.get("workload") == w.name:
            traffic = tr.get("bytes_per_launch")
    dec_bytes = w.batch * w.num_kv_heads * decode_bytes(w, w.seq_len)
    split_bytes = w.batch * w.num_kv_heads * decode_split_bytes(w, w.seq_len)
    d_ms = float(np.mean(split_ms)) if split_ms else float("nan")
    dec_ms = sum(kernel_ms[k] for k in (D.KERNEL_DECODE_PROLOGUE, D.KERNEL_DECODE_SPLIT, D.KERNEL_DECODE_COMBINE))
    cmp_ms = sum(kernel_ms[k] for k in (D.KERNEL_CENTER, D.KERNEL_REFPREP, D.KERNEL_SEARCH))
    line = {
        "metric": METRIC,
        "value": tokens_per_step(w) * world * K / (ms_max / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_max / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "layers": w.layers, "batch": w.batch, "seq_len": w.seq_len,
                   "kv_heads": w.num_kv_heads, "q_heads": w.num_q_heads, "head_dim": w.head_dim, "rank": w.rank,
                   "ref_stride": w.ref_stride, "parallelism": f"replica-per-gpu x{world}",
                   "l2": "inputs larger than L2 (K+V %.0f MB per layer), no flush" %
                         (rep.k[0].numel() * 4 / 1e6)},
        "kernel_ms_per_launch": {KERNEL_NAMES[k]: v for k, v in kernel_ms.items()},
        "compress": {"tokens_per_s": w.batch * w.seq_len * world / (cmp_ms / 1e3),
                     "ms_per_layer": cmp_ms, "search_ms_per_launch": s_ms, "search_tflops": achieved},
        "decode": {"tok_per_s": w.batch * world / (dec_ms * w.layers / 1e3), "ms_per_layer": dec_ms,
                   "algorithmic_bytes_per_layer": dec_bytes,
                   "gbs": dec_bytes / (dec_ms / 1e3) / 1e9, "frac_hbm": dec_bytes / (dec_ms / 1e3) / 1e9 / hbm,
                   "split_ms_per_launch": d_ms, "split_bytes": split_bytes,
                   "split_gbs": split_bytes / (d_ms / 1e3) / 1e9,
                   "split_frac_hbm": split_bytes / (d_ms / 1e3) / 1e9 / hbm, "hbm_peak_gbs": hbm},
        "roofline": {"kernel": "search_tc_kernel", "bound": "tensor", "achieved": achieved, "peak": tf_burst,
                     "peak_kind": f"bf16 dense burst, {peak_kind}", "unit": "TFLOP/s", "frac": achieved / tf_burst,
                     "traffic": traffic, "flops_per_launch": flops_launch},
        "gpu_launches": rep.launches_per_step * K,
        "clocks": clk,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if not args.no_cpu_baseline:
        dt, frac, desc = cpu_oracle_sample(w, w.seq_len)
        per_step_equiv = dt / frac * w.layers * w.batch
        line["cpu_baseline"] = {"value": tokens_per_step(w) / per_step_equiv, "unit": "tokens/s",
                                "cores": cpu_threads(), "kind": "oracle", "sample": desc}
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def main():
    args = parse()
    w = synth.workload(args.workload)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
