"""Multi-process host logic of the replica-per-GPU bench, on CPU with the gloo backend (world size 2).

The path exchanges no data between GPUs: each rank compresses and decodes its own shard of sequences, and
the only collectives are the timing barrier and a MAX reduction of the step time.  These tests run that
host logic in two real processes.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    from residual_kv_cache_delta_b200 import synth
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, wsz, _ = bench.dist_env()
        seqs = bench.shard_sequences(r, 3)
        shards = [None] * wsz
        torch.distributed.all_gather_object(shards, seqs)
        slowest = bench.max_over_ranks(1.5 + r, torch.device("cpu"), wsz)
        w = synth.workload(0)
        k, _ = synth.kv_tokens(w, 0, seqs[0], 0, 64)
        with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
            json.dump({"rank": r, "world": wsz, "seqs": seqs, "shards": shards, "slowest": slowest,
                       "k0": np.asarray(k, dtype=np.float64).ravel()[:16].tolist()}, f)
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


def test_replica_shards_and_max_over_ranks_gloo(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [x["world"] for x in res] == [2, 2]
    # every rank sees the same shard map; shards are disjoint and cover 0 .. world*batch-1
    assert res[0]["shards"] == res[1]["shards"]
    flat = sum(res[0]["shards"], [])
    assert sorted(flat) == list(range(6)) and len(set(flat)) == 6
    # the job's time is the slowest rank's, on every rank
    assert res[0]["slowest"] == res[1]["slowest"] == 2.5
    # different shards mean different synthetic sequences (weak scaling, not N copies of one)
    assert res[0]["k0"] != res[1]["k0"]


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", LOCAL_RANK="0", MASTER_ADDR="127.0.0.1")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "0",
           "--steps", "1", "--warmup", "0", "--gpus", "2"]
    r1 = subprocess.run(cmd, env=dict(env, RANK="1"), capture_output=True, text=True, timeout=300)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = subprocess.run(cmd, env=dict(env, RANK="0"), capture_output=True, text=True, timeout=300)
    assert r0.returncode == 0, r0.stderr
    lines = [ln for ln in r0.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0 and line["n_gpus"] == 2
