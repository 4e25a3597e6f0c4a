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


def _reference_arm(env_extra):
    import json
    import subprocess
    env = dict(os.environ, **env_extra)
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "0",
                        "--steps", "2", "--warmup", "0"], capture_output=True, text=True, timeout=300, env=env,
                       cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    return [json.loads(line) for line in p.stdout.splitlines() if line.startswith("{")]


def test_reference_arm_prints_one_line_with_the_contract_keys():
    (line,) = _reference_arm({})
    assert line["impl"] == "reference" and line["unit"] == "tok/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 2 and line["dtype"] == "f64"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # the value is the sample's rate scaled to the whole step's units
    units = line["sample_scale"]["units_per_step"]
    from residual_kv_cache_delta_b200 import synth
    assert line["value"] == pytest.approx(synth.workload(0).batch / (line["ms_per_step"] / 1e3 * units), rel=1e-9)


def test_reference_arm_runs_on_rank_zero_only():
    assert _reference_arm({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []


def test_peaks_are_the_measured_file_else_the_stated_fallback(tmp_path, monkeypatch):
    import json
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps({"hbm_gbs": 6538.0, "bf16_tflops": 1630.4, "bf16_tflops_sustained": 1388.1}))
    monkeypatch.setattr(bench, "PEAKS_FILE", str(f))
    assert bench.load_peaks() == (6538.0, 1630.4, 1388.1, "measured")
    f.write_text(json.dumps({"hbm_gbs": 6538.0, "bf16_tflops": 1630.4}))  # no sustained figure: the burst one
    assert bench.load_peaks() == (6538.0, 1630.4, 1630.4, "measured")
    monkeypatch.setattr(bench, "PEAKS_FILE", str(tmp_path / "absent.json"))
    hbm, burst, sustained, kind = bench.load_peaks()
    assert (hbm, burst, kind) == (6650.0, 1590.0, "fallback") and sustained <= burst


def test_clock_samples_parse_to_median_and_active_reasons(monkeypatch):
    class FakeSmi:  # stands in for the nvidia-smi sampler process
        def __init__(self, out):
            self.out = out

        def terminate(self):
            pass

        def communicate(self, timeout=None):
            return self.out, ""

    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    rows = ["0, 1700, 1965, 980.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
            "0, 1740, 1965, 990.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
            "0, [N/A], 1965, [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]",  # unreadable sample: skipped
            "0, 1965, 1965, 700.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"]
    c = bench.Clocks(0)
    c.proc = FakeSmi("\n".join(rows) + "\n")
    assert c.stop() == {"sm_mhz": 1740.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    c.proc = FakeSmi("0, 1200, 1965, 500, 0x8, Active, Not Active, Active, Not Active\n")
    assert c.stop()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    c.proc = FakeSmi("")
    assert c.stop() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    assert bench.Clocks(0).stop() is None  # the sampler never started (no nvidia-smi)


@pytest.mark.parametrize("q4", [False, True])
def test_decode_bytes_are_the_bytes_of_the_arrays_one_unit_reads(q4):
    """The roofline's algorithmic bytes per (sequence, layer, kv head), checked against the library's own cache
    layout: the codes and indices of T tokens and the reference rows of T / R blocks (deltakv_cache_bytes), one
    block-table entry per block, mu (fp32) and the basis of one kv head, and the group's queries and outputs."""
    from residual_kv_cache_delta_b200 import build as B
    from residual_kv_cache_delta_b200 import deltakv as D
    from residual_kv_cache_delta_b200 import synth
    B.build()
    w = synth.workload(2)
    T, nb = 32768, 32768 // w.ref_stride
    sh = D.Shape(w.num_q_heads, w.num_kv_heads, w.head_dim, w.rank, w.ref_stride, w.torch_dtype, q4=q4)
    codes, ref_idx, refs = D.cache_bytes(sh, nb)
    per_head = lambda x: x // w.num_kv_heads  # noqa: E731  (the arrays hold every kv head)
    es, d, r, G = w.elem_bytes, w.head_dim, w.rank, w.group
    split = per_head(codes) + per_head(ref_idx) + nb * 4
    assert bench.decode_split_bytes(w, T, q4) == split
    assert bench.decode_bytes(w, T, q4) == split + per_head(refs) + 2 * d * 4 + 2 * d * r * es + 2 * G * d * es


def test_search_work_closed_form_against_brute_force():
    """The search roofline's flops: causal (token, visible reference) pairs counted one by one on small cases
    (every non-reference position t sees the references j with j R < t), and the documented per-launch total
    of the single-layer 32768-token workload (8 kv heads)."""
    for T, R, start in ((1, 16, 0), (17, 16, 0), (100, 16, 0), (257, 32, 0), (300, 64, 40), (64, 16, 48)):
        brute = sum(len([j for j in range(T) if j * R < t]) for t in range(start, T) if t % R)
        assert bench.search_pairs(T, R, start) == brute, (T, R, start)
    from residual_kv_cache_delta_b200 import synth
    w = synth.workload(1)
    assert w.num_kv_heads * bench.search_flops(w, 32768) == pytest.approx(133.21e9, rel=1e-4)
