"""Host-side logic of bench.py (CPU only): the clock record that decides
whether a timed run is kept, the committed DRAM-traffic records and the
launch count it claims."""
import json
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _line(sm, mx=1965, reasons=("Not Active",) * 4):
    # index, clocks.sm, clocks.max.sm, power.draw, active mask, 4 reasons
    return ", ".join(["0", str(sm), str(mx), "812.5", "0x0000000000000000", *reasons])


def test_clock_summary_median_under_load_and_no_reasons():
    lines = [_line(345), _line(1965), _line(1950), _line(1965), _line(1965)]
    c = bench.ClockSampler.summarise(lines)
    # the idle sample (below half of max) is left out of the median
    assert c == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 5}


def test_clock_summary_reports_each_active_reason():
    act = ("Not Active", "Active", "Not Active", "Active")   # hw_thermal, sw_power_cap
    lines = [_line(1500), _line(1490, reasons=act), "garbled", _line("[N/A]")]
    c = bench.ClockSampler.summarise(lines)
    assert c["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert c["samples"] == 2 and c["sm_mhz"] == pytest.approx(1495.0)


def test_clock_summary_without_samples_is_none():
    assert bench.ClockSampler.summarise([]) is None
    assert bench.ClockSampler.summarise(["not, a, sample"]) is None


def test_traffic_records_name_existing_sources():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    assert rec, "no traffic records"
    for kernel, e in rec.items():
        assert kernel in bench.KERNEL_SOURCES, kernel
        for p in bench.KERNEL_SOURCES[kernel]:
            assert os.path.exists(os.path.join(ROOT, p)), p
        assert e["dram_bytes_per_launch"] > 0
        assert len(e["source_hash"]) == 16


def test_traffic_record_is_void_once_its_sources_change(monkeypatch, tmp_path):
    assert bench.profiled_traffic("no_such_kernel") is None
    kernel = "gemm_gate_up_large"
    stored = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))[kernel]
    if stored["source_hash"] != bench.kernel_source_hash(kernel):
        pytest.skip("record already void for the working tree's sources")
    assert bench.profiled_traffic(kernel) == stored["dram_bytes_per_launch"]
    extra = tmp_path / "changed.cu"
    extra.write_text("// one more source\n")
    monkeypatch.setitem(bench.KERNEL_SOURCES, kernel,
                        bench.KERNEL_SOURCES[kernel] + [str(extra)])
    assert bench.profiled_traffic(kernel) is None


@pytest.mark.parametrize("T,d,E,want", [
    (6144, 4096, 512, 10),   # tensor-core router, x copied to fp16 for the GEMM
    (512, 4096, 128, 10),
    (100, 4096, 128, 10),    # CUDA-core router without K split (T > 16)
    (16, 4096, 512, 11),     # K-split router + split reduction, tensor-core GEMM
    (8, 4096, 512, 10),      # K-split router, decode GEMM (no fp16 copy)
    (1, 32, 8, 9),           # one K split: no reduction kernel
    (4, 4096, 512, 1),       # verify batch: the whole layer in one launch
    (1, 4096, 512, 1),
    (5, 4096, 512, 10),      # five tokens: separate kernels again
])
def test_launch_count_follows_dispatch_rules(T, d, E, want):
    assert bench.launches_per_step(T, d, E) == want


def test_algorithmic_work_matches_the_workload_table():
    from moe_inputs import WORKLOADS
    large = WORKLOADS["large"]
    # packed int4 of gate, up, down (3 * 4096 * 1024 / 2) + fp16 scales per group of 64
    assert bench.expert_bytes(large) == 6_684_672
    assert bench.layer_flops(large, 6144) == pytest.approx(1.572e12, rel=1e-3)
    # 40 experts, the router matrix, x and y of four tokens
    assert bench.layer_hbm_bytes(large, 4, 40) == 40 * 6_684_672 + 4096 * 512 * 2 + 2 * 4 * 4096 * 2


def test_expert_load_counts_rows_per_expert():
    import numpy as np
    ids = np.array([[0, 3], [3, 5], [3, 0]])
    assert bench.expert_load(ids, 8) == {"experts_touched": 3, "rows_max": 3,
                                         "rows_mean_touched": 2.0, "rows_mean_all": 0.75}


def test_clock_line_parse_keeps_power_and_reasons():
    act = ("Not Active", "Not Active", "Not Active", "Active")
    sm, mx, pw, reasons = bench.ClockSampler.parse(_line(1800, reasons=act))
    assert (sm, mx, pw, reasons) == (1800.0, 1965.0, 812.5, {"sw_power_cap"})
    assert bench.ClockSampler.parse("garbled") is None


class _FakeNvml:
    """Stands in for pynvml: fixed clocks, 812.5 W, and the power-cap reason."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonSwPowerCap = 0x4

    def __init__(self, sm=1800, mask=0x4):
        self.sm, self.mask = sm, mask

    def nvmlDeviceGetClockInfo(self, h, kind):
        return self.sm

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetPowerUsage(self, h):
        return 812500

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.mask


def test_nvml_sample_reads_back_like_an_nvidia_smi_line():
    line = bench.ClockSampler.nvml_line(_FakeNvml(), None, 0)
    assert bench.ClockSampler.parse(line) == (1800.0, 1965.0, 812.5, {"sw_power_cap"})
    hot = bench.ClockSampler.nvml_line(_FakeNvml(sm=1500, mask=0x8 | 0x40), None, 0)
    assert bench.ClockSampler.parse(hot)[3] == {"hw_slowdown", "hw_thermal_slowdown"}
    c = bench.ClockSampler.summarise([line, line, hot])
    assert c["samples"] == 3 and c["sm_mhz"] == 1800.0
    assert c["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"]
