"""Host-side logic of bench.py (CPU only): the peaks loader, the DRAM-traffic
record check, the algorithmic byte counts the rooflines divide by, and the
clock sampler's throttle-reason parsing."""
import hashlib
import json
import os

import pytest

import bench

FALLBACK = bench.PEAKS_FALLBACK


def _write(tmp_path, name, obj):
    p = tmp_path / name
    p.write_text(json.dumps(obj))
    return str(p)


def test_peaks_missing_file_uses_the_fallback(tmp_path):
    peaks, kind = bench.load_peaks(str(tmp_path / "absent.json"))
    assert peaks == FALLBACK and kind == "fallback"


@pytest.mark.parametrize("doc", [
    {"hbm_gbs": 6547.5, "bf16_tflops": 1645.2, "bf16_tflops_sustained": 1381.8},
    {"hbm": {"copy_gb/s": 6547.5}, "gemm": {"bf16_tflops_sustained": 1381.8, "bf16_tflops": 1645.2},
     "clocks": {"sm_mhz": 1965}},
    {"b200": {"HBM_GBs": 6547.5, "BF16_TFLOPS": 1645.2, "BF16_TFLOPS_SUSTAINED": 1381.8}},
])
def test_peaks_any_nesting(tmp_path, doc):
    peaks, kind = bench.load_peaks(_write(tmp_path, "p.json", doc))
    assert kind == "measured"
    assert peaks == {"hbm_gbs": 6547.5, "bf16_tflops": 1645.2, "bf16_tflops_sustained": 1381.8}


def test_peaks_partial_file_says_which_figures_are_fallback(tmp_path):
    peaks, kind = bench.load_peaks(_write(tmp_path, "p.json", {"hbm_gbs": 6000.0}))
    assert peaks["hbm_gbs"] == 6000.0 and peaks["bf16_tflops"] == FALLBACK["bf16_tflops"]
    assert kind == "measured hbm_gbs; fallback for the rest"


def test_traffic_record_is_used_only_for_its_own_source(tmp_path):
    src = tmp_path / "csrc"
    src.mkdir()
    (src / bench.KERNEL_SOURCES["attn_split_kernel"]).write_text("kernel v1\n")
    sha = hashlib.sha256(b"kernel v1\n").hexdigest()
    rec = {"attn_split_kernel": {"workload": "w", "dram_bytes_per_launch": 123, "source_sha256": sha, "command": "c"}}
    path = _write(tmp_path, "rec.json", rec)
    assert bench.captured_traffic("attn_split_kernel", "w", path, str(src)) == (123, "c")
    assert bench.captured_traffic("attn_split_kernel", "other", path, str(src))[0] is None
    (src / bench.KERNEL_SOURCES["attn_split_kernel"]).write_text("kernel v2\n")
    got = bench.captured_traffic("attn_split_kernel", "w", path, str(src))
    assert got == (None, "kernel source changed since the capture")
    assert bench.captured_traffic("attn_split_kernel", "w", str(tmp_path / "none.json"), str(src))[0] is None


def test_committed_traffic_record_names_the_bench_workload():
    with open(bench.TRAFFIC_RECORD) as f:
        rec = json.load(f)
    assert set(rec) == set(bench.KERNEL_SOURCES)
    for r in rec.values():
        assert r["workload"] == "decode_layer H4096 Hq32 Hkv8 D128 F11008 B128 kv2048"
        assert r["dram_bytes_per_launch"] > 0 and len(r["source_sha256"]) == 64


def test_layer_bytes_at_the_decode_workload():
    # hand counts for hidden 4096, 32 / 8 heads of 128, MLP 11008, B = 128, KV 2048:
    #   o:       4 B x 4096 x 4096 weights + 4 B x 128 x 4096 (A hi/lo) + 8 B x 128 x 4096 (y, residual)
    #   gate/up: 4 B x 4096 x 22016 + 4 B x 128 x 4096 + 4 B x 128 x 11008 (a hi/lo)
    #   down:    4 B x 11008 x 4096 + 4 B x 128 x 11008 + 8 B x 128 x 4096
    #   qkv:     4 B x 4096 x 6144 + 4 B x 128 x 4096 + q 4 B x 128 x 4096
    #            + K/V rows 128 x 16 x (256 + 4) B + rotary rows 128 x 512 B
    #   attention: 520 B per (row, kv head, key) + q 512 B per (row, head) + partials 520 B per (row, head, split)
    gemm, attn = bench.layer_bytes(128, 2048)
    assert gemm == {"gemm_o": 73_400_320, "gemm_gate_up_swiglu": 368_443_392, "gemm_down": 190_185_472,
                    "gemm_qkv_rope_quant": 105_455_616}
    assert attn == 1_109_655_552
    # the packed weights of the layer: 4 B x 177,209,344 parameters = 708.8 MB
    weights = 4 * (4096 * 6144 + 4096 * 4096 + 4096 * 22016 + 11008 * 4096)
    assert weights == 708_837_376
    assert sum(gemm.values()) > weights
    # one more split of 256 keys adds one partial per (row, head); one more key adds 520 B per (row, kv head)
    _, attn2 = bench.layer_bytes(128, 2049)
    assert attn2 - attn == 128 * 8 * 520 + 128 * 32 * 130 * 4


class _Proc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass


def _sampler_with(tmp_path, lines):
    p = tmp_path / "clocks.csv"
    p.write_text("\n".join(lines) + "\n")
    cs = bench.ClockSampler(0)
    cs.proc, cs.path = _Proc(), str(p)
    return cs


def test_clock_sampler_reports_power_cap_and_median_under_load(tmp_path):
    na, act = "Not Active", "Active"
    lines = [f"0, 1965, 1965, 120.5, 0x0, {na}, {na}, {na}, {na}, 0",      # idle: not counted
             f"0, 1850, 1965, 990.1, 0x4, {na}, {na}, {na}, {act}, 100",
             f"0, 1880, 1965, 995.0, 0x4, {na}, {na}, {na}, {act}, 100",
             f"0, 1900, 1965, 1001.0, 0x0, {na}, {na}, {na}, {na}, 99"]
    got = _sampler_with(tmp_path, lines).stop()
    assert got["sm_mhz"] == 1880 and got["sm_max_mhz"] == 1965
    assert got["reasons"] == ["sw_power_cap"] and got["samples"] == 3 and got["power_w_max"] == 1001.0


def test_clock_sampler_reports_thermal_and_hardware_slowdowns(tmp_path):
    na, act = "Not Active", "Active"
    lines = [f"0, 1400, 1965, 700, 0x48, {act}, {na}, {na}, {na}, 100",
             f"0, 1300, 1965, 650, 0x20, {na}, {na}, {act}, {na}, 100"]
    got = _sampler_with(tmp_path, lines).stop()
    assert got["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
