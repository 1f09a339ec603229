"""Host-side logic of bench.py, without a GPU: the algorithmic bytes each
roofline fraction divides by, the shape of the committed DRAM-traffic records,
and the parsing of the clock samples that decides whether a run is kept."""
import glob
import os
import re
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _bytes(workload):
    return dict(bench.make_workload(workload)["kernels"])


def test_algorithmic_bytes_per_launch():
    """bf16 input (2 bytes per element), packed codes (half a byte), one scale
    byte per block, and for the dual format one fp32 group scale per 128."""
    M, K = 32768, 4096
    d = _bytes("dual")
    assert d["quantize"] == 2 * M * K + M * K // 2 + M * K // 16 + 4 * (M * K // 128) == 348_127_232
    assert d["dequantize"] == d["quantize"]
    M = K = 4096
    m = _bytes("mxfp4")
    assert m["quantize"] == m["dequantize"] == 2 * M * K + M * K // 2 + M * K // 32 == 42_467_328
    M, K = 8192, 4096
    assert _bytes("hadamard128")["quantize"] == 2 * M * K + M * K // 2 + M * K // 16
    # ARC writes the [K | S] operand: K + S code and scale columns per row
    KS = K + 256
    assert _bytes("arc")["arc"] == 2 * M * K + M * KS // 2 + M * KS // 16 == 87_162_880
    assert _bytes("arc_int4")["arc"] == _bytes("arc")["arc"]
    assert _bytes("arc_mxfp4")["arc"] == 2 * M * K + M * KS // 2 + M * KS // 32
    # the amax pre-pass reads the input a second time
    M, K = 256, 1024
    assert _bytes("nvfp4")["amax+quantize"] == 4 * M * K + M * K // 2 + M * K // 16


def test_rows_override_scales_the_workload():
    wl = bench.make_workload("arc", 2960)
    assert wl["M"] == 2960 and "[2960 rows]" in wl["desc"]
    assert dict(wl["kernels"])["arc"] == 2 * 2960 * 4096 + 2960 * 4352 // 2 + 2960 * 4352 // 16


def test_traffic_records_are_keyed_to_their_kernels_sources():
    """Each record names one timed kernel of one workload, holds a per-launch
    byte count and the hash of that kernel's own source files (so that an edit
    elsewhere leaves it valid, and an edit of the kernel voids it)."""
    paths = sorted(glob.glob(os.path.join(ROOT, "profiles", "traffic_*.txt")))
    assert paths
    for path in paths:
        name = os.path.basename(path)[len("traffic_"):-len(".txt")]
        workload, label = name.rsplit("_", 1)
        assert (workload, label) in bench.KERNEL_SOURCES, name
        txt = open(path).read()
        assert re.search(r"^source_sha: [0-9a-f]{16}$", txt, re.M), name
        val = re.search(r"^dram_bytes_per_launch: (\d+)$", txt, re.M)
        assert val and int(val.group(1)) > 0, name
        assert "--clock-control none" in txt, name
        for fn in bench.KERNEL_SOURCES[(workload, label)]:
            assert os.path.exists(os.path.join(ROOT, "fp4_micro_block_b200", "csrc", fn)), fn


def test_kernel_source_hash_depends_only_on_the_listed_files():
    files = bench.KERNEL_SOURCES[("mxfp4", "quantize")]
    assert bench.kernel_source_sha(files) == bench.kernel_source_sha(list(reversed(files)))
    assert bench.kernel_source_sha(files) != bench.kernel_source_sha(files + ["fp4q_arc.cuh"])


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _line(sm, smax, hw="Not Active", cap="Not Active"):
    return f"0, {sm}, {smax}, 640.5, 0x0000000000000000, {hw}, Not Active, Not Active, {cap}"


def test_clock_samples_inside_the_timed_region():
    cs = bench.ClockSampler(0)
    cs.proc = _FakeProc()
    cs.lines = [(0.0, _line(120, 1965)),                 # idle, before the region
                (10.0, _line(1965, 1965)), (10.2, _line(1950, 1965, cap="Active")),
                (10.4, _line(1965, 1965)),
                (20.0, _line(500, 1965, hw="Active"))]   # after the region
    c = cs.stop(9.9, 10.5)
    assert c["samples"] == 3
    assert c["sm_mhz"] == 1965.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]


def test_clock_samples_report_a_slowdown():
    cs = bench.ClockSampler(0)
    cs.proc = _FakeProc()
    cs.lines = [(1.0, _line(1100, 1965, hw="Active")), (1.1, _line(1100, 1965, hw="Active")),
                (1.2, "garbled")]
    c = cs.stop(0.9, 1.3)
    assert c["samples"] == 2 and c["sm_mhz"] == 1100.0
    assert c["reasons"] == ["hw_slowdown"]


def test_clock_sampler_without_nvidia_smi():
    cs = bench.ClockSampler(0)
    c = cs.stop(0.0, 1.0)
    assert c["sm_mhz"] is None and c["reasons"] == ["nvidia-smi unavailable"]
