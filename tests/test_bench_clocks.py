"""The benchmark's clock record, on synthetic samples: only samples inside the
timed region count, the median SM clock is reported, and every clock-event
reason bit seen there is named (hw_slowdown and the thermal reasons are the
ones that invalidate a run; sw_power_cap is kept and noted)."""

import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler(tmp_path, lines, t0, t1):
    s = object.__new__(bench.ClockSampler)
    s.path = str(tmp_path / "clocks_rank0.csv")
    s.raw = s.path + ".raw"
    with open(s.raw, "w") as f:
        f.write("\n".join(lines) + "\n")
    s.f = open(os.devnull, "w")
    s.proc = _FakeProc()
    s.t0, s.t1 = t0, t1
    return s


def test_window_median_and_reasons(tmp_path):
    lines = ["max 1965",
             "99.0000,1200,0x0,500.0",     # before the timed region: dropped
             "100.0000,1965,0x0,900.0",
             "100.0020,1950,0x4,1000.0",   # sw_power_cap
             "100.0040,1900,0x8,990.0",    # hw_slowdown
             "100.0060,1965,0x0,950.0",
             "100.0080,1965,0x60,950.0",   # both thermal reasons
             "101.0000,800,0x0,100.0",     # after it: dropped
             "garbage line"]
    rec = _sampler(tmp_path, lines, 100.0, 100.5).stop()
    assert rec["samples"] == 5
    assert rec["sm_mhz"] == 1965.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap",
                              "sw_thermal_slowdown"]
    kept = open(tmp_path / "clocks_rank0.csv").read().splitlines()
    assert kept[0].startswith("time,") and len(kept) == 6
    assert not os.path.exists(tmp_path / "clocks_rank0.csv.raw")


def test_clean_run_has_no_reasons(tmp_path):
    lines = ["max 1965"] + [f"{200 + 0.002 * i:.4f},1965,0x0,800.0" for i in range(50)]
    rec = _sampler(tmp_path, lines, 200.0, 201.0).stop()
    assert rec["samples"] == 50 and rec["reasons"] == [] and rec["sm_mhz"] == 1965.0


def test_sampler_unavailable():
    s = object.__new__(bench.ClockSampler)
    s.proc = None
    rec = s.stop()
    assert rec["samples"] == 0 and rec["reasons"] == ["sampler unavailable"]
