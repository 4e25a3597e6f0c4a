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

