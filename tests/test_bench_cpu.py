"""bench.py host logic on CPU: the clock sampler against a fake NVML, and the
code fingerprint that ties the committed ncu traffic figures to kernel code."""

import sys
import time
import types

import bench


def _fake_nvml(clocks, powers_mw, reasons):
    """A stand-in for the pynvml module that replays fixed readings."""
    state = {"i": 0}
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1

    def nxt(seq):
        return seq[min(state["i"], len(seq) - 1)]

    def reason(h):  # the sampler reads clock, power, reasons: advance after the last
        v = nxt(reasons)
        state["i"] += 1
        return v

    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByPciBusId = lambda bus: (_ for _ in ()).throw(RuntimeError("no PCI match"))
    m.nvmlDeviceGetHandleByIndex = lambda i: ("handle", i)
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965
    m.nvmlDeviceGetClockInfo = lambda h, kind: nxt(clocks)
    m.nvmlDeviceGetPowerUsage = lambda h: nxt(powers_mw)
    m.nvmlDeviceGetCurrentClocksEventReasons = reason
    return m


def test_clock_sampler_reads_nvml(monkeypatch):
    fake = _fake_nvml([1965, 1600, 1580, 1580, 1580], [120_000, 990_000, 995_000, 993_000, 994_000],
                      [0x0, 0x4, 0x4, 0x4, 0x4])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    c = bench.ClockSampler(0)
    c.start()
    time.sleep(0.15)
    out = c.stop()
    assert out["source"] == "nvml, 10 ms"
    assert out["samples"] >= 5
    assert out["sm_max_mhz"] == 1965.0
    # samples under load (> 300 W) only: the idle 1965 MHz reading is left out
    assert out["sm_mhz"] == 1580.0
    assert out["reasons"] == ["sw_power_cap"]


def test_clock_sampler_flags_thermal_and_hw_slowdown(monkeypatch):
    fake = _fake_nvml([1200], [800_000], [0x8 | 0x40 | 0x20])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    c = bench.ClockSampler(0)
    c.start()
    time.sleep(0.05)
    out = c.stop()
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_sampler_without_nvml_or_smi(monkeypatch):
    broken = types.ModuleType("pynvml")

    def fail():
        raise RuntimeError("no driver")

    broken.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", broken)
    monkeypatch.setattr(bench.subprocess, "Popen", lambda *a, **k: (_ for _ in ()).throw(FileNotFoundError()))
    c = bench.ClockSampler(0)
    c.start()
    out = c.stop()
    assert out["sm_mhz"] is None


def test_clocks_rejected_rules():
    ok = {"sm_mhz": 1580.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert not bench.clocks_rejected(ok)
    assert not bench.clocks_rejected({"sm_mhz": 1960.0, "sm_max_mhz": 1965.0, "reasons": []})
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clocks_rejected({"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": [r]})
    # stuck low with no reason: a leftover clock lock
    assert bench.clocks_rejected({"sm_mhz": 1000.0, "sm_max_mhz": 1965.0, "reasons": []})
    # no samples at all is not a rejection
    assert not bench.clocks_rejected({"sm_mhz": None, "sm_max_mhz": None, "reasons": []})


def test_code_fingerprint_ignores_comments_only(tmp_path):
    src = tmp_path / "k.cu"
    base = 'int f(int x) {\n  // a comment\n  return x + 1;  /* another */\n}\nconst char* s = "a // b /* c";\n'
    src.write_text(base)
    ref = bench.code_fingerprint(str(src))
    # comments, blank lines and trailing blanks do not count
    src.write_text(base.replace("// a comment", "// reworded, longer comment").replace("/* another */", "") + "\n\n")
    assert bench.code_fingerprint(str(src)) == ref
    src.write_text("/* header\n   block */\n" + base.replace("return x + 1;", "return x + 1;   "))
    assert bench.code_fingerprint(str(src)) == ref
    # code does, including text inside a string literal that looks like a comment
    src.write_text(base.replace("x + 1", "x + 2"))
    assert bench.code_fingerprint(str(src)) != ref
    src.write_text(base.replace('"a // b /* c"', '"a // b /* d"'))
    assert bench.code_fingerprint(str(src)) != ref


def test_traffic_figures_match_the_kernel_code():
    """Every committed ncu traffic figure names the code it was taken on; the
    bench reports it only while that code is unchanged (null otherwise).  The
    committed figures are for the current kernel sources."""
    import os
    root = os.path.dirname(bench.__file__)
    for (kernel, _), entry in bench.NCU_TRAFFIC.items():
        src = os.path.join(root, "exact_blockwise_long_b200", "csrc", "bwd_tc.cu" if kernel.startswith("bwd") else "fwd_tc.cu")
        assert entry["code_sha256"] == bench.code_fingerprint(src), kernel

