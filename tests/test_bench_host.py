"""Host-side logic of bench.py, on the CPU: the source spans that date the ncu traffic
figures, the traffic table itself, the FLOP counts the throughput divides, the clock
summary that decides whether a run is kept, and the JSON line of the reference arm."""
import json
import os

import pytest

import bench
import synth

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "exact_io_aware_44_b200", "csrc")


def test_kernel_source_spans_resolve_to_one_place_each():
    """Every span's markers occur once in its file, so a hash covers the kernel it names
    and an edit to that kernel changes it (a traffic figure then reads as stale)."""
    hashes = {}
    for name, (fname, spans) in bench.KERNEL_SOURCES.items():
        text = open(os.path.join(CSRC, fname)).read()
        for start, end in spans:
            if start:
                assert text.count(start) == 1, (name, start)
                a = text.index(start)
            else:
                a = 0
            if end:
                assert text.find(end, a) > a, (name, end)
        hashes[name] = bench.kernel_source_hash(name)
        assert len(hashes[name]) == 16
    # the d = 64/128 forward and the d = 256 forward are dated separately
    assert hashes["fwd"] != hashes["fwd256"]
    assert hashes["bwd_main"] != hashes["bwd_main_d64"]


def test_traffic_table_names_known_workloads_and_plausible_bytes():
    """Each recorded DRAM figure belongs to a workload the bench runs, and is at least
    the bytes that workload's kernel must read once (less would mean a wrong capture)."""
    for (kernel, wname), rec in bench.NCU_TRAFFIC.items():
        assert kernel in ("fwd", "bwd_main", "decode_split"), kernel
        assert len(rec["csrc_sha"]) == 16
        if kernel == "decode_split":
            w = synth.DECODE_WORKLOADS[wname]
            must_read = w.kv_bytes()
        else:
            w = synth.WORKLOADS[wname]
            tile = w.B * w.N * w.d * 2
            must_read = tile * (w.Hq + 2 * w.Hkv) + (tile * w.Hq if kernel == "bwd_main" else 0)
        assert must_read <= rec["bytes_per_launch"] <= 3 * must_read, (kernel, wname, rec, must_read)


def test_flop_counts_follow_the_stated_formula():
    """4 B Hq N^2 d for the forward, halved when causal; the backward 2.5 times that."""
    c3 = synth.WORKLOADS["c3"]
    assert c3.fwd_flops() == pytest.approx(4 * 2 * 32 * 8192 ** 2 * 128 / 2)
    assert c3.fwd_flops() == pytest.approx(1.0995e12, rel=1e-4)
    assert c3.bwd_flops() == pytest.approx(2.5 * c3.fwd_flops())
    c3n = synth.WORKLOADS["c3n"]
    assert c3n.fwd_flops() == pytest.approx(2 * c3.fwd_flops())
    assert bench.job_throughput(c3.fwd_flops(), 4, 1.0) == pytest.approx(4 * c3.fwd_flops() / 1e12)


def test_fp32_alu_peak_is_the_nominal_fma_rate():
    assert bench.FP32_ALU_TFLOPS == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)


def _sampler(samples, window):
    s = bench.ClockSampler(0)
    s.samples = list(samples)
    s.window = list(window)
    return s


def test_clock_summary_uses_the_timed_window_and_names_reasons():
    outside = [(0.0, 1965.0, 1965.0, 300.0, 0), (9.0, 1965.0, 1965.0, 300.0, 0)]
    inside = [(1.0, 1700.0, 1965.0, 900.0, 0x4), (2.0, 1650.0, 1965.0, 950.0, 0x4),
              (3.0, 1600.0, 1965.0, 990.0, 0x4 | 0x8 | 0x40)]
    summ = _sampler(outside + inside, (0.5, 3.5)).summary()
    assert summ["window"] == "timed region"
    assert summ["samples"] == 3
    assert summ["sm_mhz"] == 1650.0 and summ["sm_mhz_min"] == 1600.0 and summ["sm_max_mhz"] == 1965.0
    assert summ["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"]
    assert summ["power_w_max"] == 990.0


def test_clock_summary_falls_back_to_all_samples_for_short_regions():
    samples = [(0.0, 1965.0, 1965.0, 300.0, 0), (1.0, 1965.0, 1965.0, 310.0, 0x20),
               (2.0, 1900.0, 1965.0, 320.0, 0)]
    summ = _sampler(samples, (0.9, 1.1)).summary()  # one sample inside the region
    assert summ["window"].startswith("whole sampler run")
    assert summ["samples"] == 3
    assert summ["reasons"] == ["sw_thermal_slowdown"]
    assert _sampler([], (None, None)).summary()["reasons"] == ["no clock samples"]


def _reference_line(capsys, workload):
    assert bench.main(["--impl", "reference", "--workload", workload, "--steps", "1", "--warmup", "3"]) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


def test_reference_arm_prints_one_line_of_the_contract(capsys):
    """The reference arm is the float64 oracle on the host cores: one JSON line with the
    same metric and unit as the GPU arm, `impl` set, no host-device bytes."""
    line = _reference_line(capsys, "c1")
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s"
    assert line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 1 and line["warmup"] == 3
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["config"]["workload"].startswith("c1:")



def test_clock_marks_sample_the_region_edges():
    """With NVML up, each edge of the timed region takes a reading of its own, so a region
    shorter than the polling interval is never left without samples (a fake NVML here)."""
    class FakeNvml:
        NVML_CLOCK_SM = 0

        @staticmethod
        def nvmlDeviceGetClockInfo(h, kind):
            return 1800

        @staticmethod
        def nvmlDeviceGetPowerUsage(h):
            return 640_000  # mW

    s = bench.ClockSampler(0)
    s._nv = (FakeNvml, object(), lambda h: 0x4, 1965)
    s.mark(True)
    s.mark(False)
    summ = s.summary()
    assert summ["samples"] == 2
    assert summ["sm_mhz"] == 1800 and summ["sm_max_mhz"] == 1965
    assert summ["reasons"] == ["sw_power_cap"] and summ["power_w_max"] == 640.0
