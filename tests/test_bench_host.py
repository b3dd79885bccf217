"""Host arithmetic of bench.py that the JSON line's roofline rests on, on CPU: which FP4
ceiling a timed region is held against, where the peaks come from, when recorded DRAM
traffic is still valid, and the whole-job throughput formula."""
import json
import os

import pytest

import bench

PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1300.0,
         "source": "measured"}


@pytest.mark.parametrize("elapsed, bf16, word", [(0.04, 1600.0, "burst"),
                                                 (0.999, 1600.0, "burst"),
                                                 (1.0, 1300.0, "sustained"),
                                                 (6.5, 1300.0, "sustained")])
def test_fp4_ceiling_by_region_length(elapsed, bf16, word):
    peak, src = bench.fp4_ceiling(PEAKS, elapsed)
    assert peak == 4.0 * bf16  # dense FP4 : bf16 = 9 : 2.25 PFLOP/s
    assert f"bf16 {word} ({bf16} TFLOP/s)" in src and src.startswith("4 x measured")
    assert f"timed region {elapsed:.3f} s" in src


def test_peaks_file_or_fallback():
    p = bench.load_peaks()
    path = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        assert p["source"] == "measured"
        assert (p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"]) == \
            (m["hbm_gbs"], m["bf16_tflops"], m["bf16_tflops_sustained"])
    else:
        assert p == {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                     "source": "fallback"}


def test_traffic_only_for_the_source_it_was_taken_on():
    src = "bench.py"
    good = {"w": {"source": src, "sha256": bench.source_sha256(src), "bytes_per_launch": [7]}}
    stale = {"w": {"source": src, "sha256": "0" * 64, "bytes_per_launch": [7]}}
    assert bench.ncu_traffic("w", src, good)["bytes_per_launch"] == [7]
    assert bench.ncu_traffic("w", src, stale) is None
    assert bench.ncu_traffic("w", "oracle/__init__.py", good) is None  # another kernel's file
    assert bench.ncu_traffic("other", src, good) is None


def test_traffic_table_entries_are_well_formed():
    for table in (bench.NCU_TRAFFIC, bench.NCU_TRAFFIC_QUANTIZE):
        for name, e in table.items():
            wl = bench.synth.WORKLOADS[name]
            assert os.path.exists(os.path.join(bench.ROOT, e["source"]))
            assert len(e["sha256"]) == 64
            assert len(e["bytes_per_launch"]) == len(wl.linears)
            assert all(b > 0 for b in e["bytes_per_launch"])


def test_job_tflops():
    # 2 ranks x 10 steps x 1e12 FLOP over the slowest rank's 4 s
    assert bench.job_tflops(1e12, 10, 2, 4.0) == pytest.approx(5.0)


class _FakeNvml:
    """Stands in for pynvml: the clock and reasons it reports are those of the
    phase the test sets (before, inside or after the timed region)."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonSwPowerCap = 0x4
    PHASES = {"before": (700.0, 0x0), "inside": (1900.0, 0x4), "after": (600.0, 0x8)}

    def __init__(self):
        self.phase = "before"
        self.shut = False

    def nvmlInit(self):
        pass

    def nvmlShutdown(self):
        self.shut = True

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        raise RuntimeError("no such bus here")

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("gpu", i)

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        return self.PHASES[self.phase][0]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.PHASES[self.phase][1]



def test_clock_sampler_keeps_only_the_timed_region(monkeypatch):
    import sys
    import time
    fake = _FakeNvml()
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    c = bench.ClockSampler(0)
    c.start()
    time.sleep(0.05)
    fake.phase = "inside"
    time.sleep(0.01)  # let a sample of the old phase drain
    t0 = time.perf_counter()
    time.sleep(0.06)
    t1 = time.perf_counter()
    time.sleep(0.01)
    fake.phase = "after"
    time.sleep(0.05)
    clk = c.stop(t0, t1)
    assert fake.shut
    assert clk["sm_mhz"] == 1900.0 and clk["sm_max_mhz"] == 1965.0
    assert clk["reasons"] == ["sw_power_cap"]
    assert clk["samples"] >= 3 and clk["source"].startswith("nvml")


def test_clock_sampler_without_nvml_or_smi_reports_none(monkeypatch):
    import sys
    monkeypatch.setitem(sys.modules, "pynvml", None)  # import fails
    monkeypatch.setenv("PATH", "/nonexistent")          # and nvidia-smi cannot start
    c = bench.ClockSampler(0)
    c.start()
    assert c.stop() is None


def _profile_bench_commands():
    """Every `python bench.py ...` command quoted in the profile summaries, with shell line
    continuations joined; W in the few-row summary stands for each workload named there."""
    import glob
    import re
    import shlex
    cmds = []
    for path in sorted(glob.glob(os.path.join(bench.ROOT, "profiles", "*.md"))):
        text = open(path).read().replace("\\\n", " ")
        for line in text.splitlines():
            for m in re.finditer(r"python bench\.py([^`\n]*)", line):
                args = shlex.split(m.group(1).split(">")[0])
                subs = ["llm_small_m1", "llm_small_m16", "llm_small_m128"] if "W" in args else [None]
                for w in subs:
                    cmds.append((os.path.basename(path),
                                 [w if (a == "W" and w) else a for a in args]))
    return cmds


def test_profile_commands_parse_with_the_current_bench(monkeypatch):
    import sys
    cmds = _profile_bench_commands()
    assert len(cmds) >= 10
    for name, args in cmds:
        monkeypatch.setattr(sys, "argv", ["bench.py"] + args)
        try:
            a = bench.parse()
        except SystemExit:
            raise AssertionError(f"{name}: bench.py {' '.join(args)} no longer parses")
        assert a.workload in bench.synth.WORKLOADS
        # a summary named for one workload quotes commands that run that workload
        named = [w for w in bench.synth.WORKLOADS if w in name]
        if named:
            assert a.workload == max(named, key=len), f"{name}: runs {a.workload}"
