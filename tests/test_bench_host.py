"""Host-side pieces of bench.py, without a GPU: the clock sampler (against a stand-in NVML
module that only answers reads) and the comment-insensitive code digest that pins the
committed ncu traffic numbers to the kernel code they were captured on."""
import importlib.util
import os
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class FakeNVML:
    """Answers the read calls the sampler makes; records that nothing else is called."""
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, reasons, fail_init=False):
        self.clocks, self.reasons, self.fail_init = list(clocks), reasons, fail_init
        self.calls = []

    def nvmlInit(self):
        self.calls.append("init")
        if self.fail_init:
            raise RuntimeError("no driver")

    def nvmlDeviceGetHandleByUUID(self, uuid):
        self.calls.append("uuid")
        return "h"

    def nvmlDeviceGetHandleByIndex(self, i):
        self.calls.append("index")
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        assert kind == self.NVML_CLOCK_SM
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        assert kind == self.NVML_CLOCK_SM
        self.calls.append("clk")
        return self.clocks[self.calls.count("clk") % len(self.clocks)]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons


def test_clock_sampler_reads_nvml_and_maps_reason_bits(bench):
    nv = FakeNVML([1965, 1965, 1950], reasons=0x4 | 0x1)   # sw power cap (+ idle bit, not reported)
    with bench.ClockSampler(0, nvml=nv, use_smi=False) as clk:
        time.sleep(0.06)
    s = clk.summary()
    assert s["samples"] >= 3
    assert s["sm_max_mhz"] == 1965.0
    assert 1950 <= s["sm_mhz"] <= 1965
    assert s["reasons"] == ["sw_power_cap"]
    assert set(nv.calls) <= {"init", "uuid", "index", "clk"}


def test_clock_sampler_reports_throttling_reasons(bench):
    nv = FakeNVML([1200], reasons=0x8 | 0x40)
    with bench.ClockSampler(0, nvml=nv, use_smi=False) as clk:
        time.sleep(0.03)
    s = clk.summary()
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
    assert s["sm_mhz"] == 1200.0


def test_clock_sampler_without_nvml_says_so(bench):
    nv = FakeNVML([1965], reasons=0, fail_init=True)
    with bench.ClockSampler(0, nvml=nv, use_smi=False) as clk:
        pass
    s = clk.summary()
    assert s["sm_mhz"] is None and s["reasons"]


def test_code_digest_ignores_comments_and_layout_but_not_code(bench, tmp_path):
    a = tmp_path / "a.cuh"
    b = tmp_path / "b.cuh"
    c = tmp_path / "c.cuh"
    a.write_text('int f(int x) { return x + 1; }  // one\nconst char *s = "a // b";\n')
    b.write_text('/* header */\nint f(int x)\n{\n  return x + 1;   // one more comment\n}\nconst char *s = "a // b";\n')
    c.write_text('int f(int x) { return x + 2; }\nconst char *s = "a // b";\n')
    assert bench.code_digest(str(a)) == bench.code_digest(str(b))
    assert bench.code_digest(str(a)) != bench.code_digest(str(c))

