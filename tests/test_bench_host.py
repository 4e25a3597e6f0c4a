"""Host logic of bench.py that decides what the JSON line may claim (CPU only).

The bench attaches a stored ncu DRAM-traffic figure for the search kernel only while the kernel's device
source matches the source the figure was captured from.  These tests pin that rule: commentary and host
launch code do not invalidate the figure, a change to device code does.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import pytest  # noqa: E402

DEVICE = """// kernels
__global__ void k(int* x) {  // a comment
  x[0] = 1;
}
"""
HOST = """// Host side.
void launch() { k<<<1, 1>>>(nullptr); }
"""
COMMON = """__device__ int helper() { return 2; }  // shared device helper
"""


def _write(tmp_path, device, host, common):
    comp, comm = tmp_path / "compress.cuh", tmp_path / "common.cuh"
    comp.write_text(device + host)
    comm.write_text(common)
    return ((str(comp), "// Host side."), (str(comm), None))


def test_hash_ignores_commentary_and_host_code(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "KERNEL_SRC", _write(tmp_path, DEVICE, HOST, COMMON))
    h0 = bench.kernel_src_hash()
    monkeypatch.setattr(bench, "KERNEL_SRC", _write(tmp_path, DEVICE.replace("a comment", "other words") + "\n\n",
                                                      HOST.replace("1, 1", "2, 64"), COMMON))
    assert bench.kernel_src_hash() == h0


def test_hash_follows_device_code(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "KERNEL_SRC", _write(tmp_path, DEVICE, HOST, COMMON))
    h0 = bench.kernel_src_hash()
    monkeypatch.setattr(bench, "KERNEL_SRC", _write(tmp_path, DEVICE.replace("x[0] = 1", "x[0] = 2"), HOST, COMMON))
    assert bench.kernel_src_hash() != h0
    monkeypatch.setattr(bench, "KERNEL_SRC", _write(tmp_path, DEVICE, HOST, COMMON.replace("2;", "3;")))
    assert bench.kernel_src_hash() != h0



def test_default_workload_is_the_largest_single_gpu_config():
    from residual_kv_cache_delta_b200 import synth
    args = bench.parse([])
    w = synth.workload(args.workload)
    assert (w.layers, w.batch, w.seq_len) == (32, 8, 32768)
    assert args.warmup >= 3


def test_stored_traffic_scales_by_units_and_is_dropped_for_other_shapes(tmp_path, monkeypatch):
    import json
    from residual_kv_cache_delta_b200 import synth
    f = tmp_path / "t.json"
    f.write_text(json.dumps({"kernel_src_sha256_16": bench.kernel_src_hash(), "bytes_per_launch": 800.0, "units": 8,
                             "unit": {"seq_len": 32768, "ref_stride": 16, "rank": 32, "head_dim": 128}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    w2 = synth.workload(2)
    assert bench.search_traffic(w2, [32768] * 8) == 800.0 / 8 * 64
    assert bench.search_traffic(synth.workload(3), [131072] * 4) is None  # other T and R
    assert bench.search_traffic(w2, [32768, 1000]) is None                # ragged


def test_oracle_rates_scale_the_sample_to_the_step():
    from residual_kv_cache_delta_b200 import synth
    w = synth.workload(2)
    dec, cmp = bench.oracle_rates(w, t_compress=2.0, t_decode=0.05, sample_tokens=32768)
    # 32 layers x 8 kv heads x 8 sequences of 32768 tokens = 2048 sample-sized decode units per step
    assert dec == pytest.approx(8 / (0.05 * 2048))
    assert cmp == pytest.approx(32768 / (2.0 * 8))
