"""The bench's clock record keeps only the samples (NVML every 2 ms, or nvidia-smi) taken inside the
device-timed window (host logic, no GPU): idle samples before or after the region must not reach
the median or the reasons."""
import datetime
import os
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _DoneProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler(lines):
    s = object.__new__(bench.ClockSampler)
    s.thread = None
    s.source = "nvidia-smi, 20 ms"
    s.proc = _DoneProc()
    s.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
    s.file.write("\n".join(lines) + "\n")
    s.file.flush()
    return s


def _line(t, mhz, power_cap="Not Active", thermal="Not Active"):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return f"{ts}, 0, {mhz}, 1965, 900.0, 0x0, Not Active, Not Active, {thermal}, {power_cap}"


def test_only_samples_inside_the_window_count():
    t = 1_700_000_000.0
    lines = [_line(t - 0.5, 1965), _line(t + 0.02, 1800, power_cap="Active"),
             _line(t + 0.04, 1820), _line(t + 0.06, 1810), _line(t + 0.3, 1965, thermal="Active")]
    out = _sampler(lines).stop((t, t + 0.1))
    assert out["samples"] == 3
    assert out["sm_mhz"] == 1810.0
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]          # the thermal sample lies outside
    assert "window" not in out


def test_no_sample_inside_the_window_is_flagged():
    t = 1_700_000_000.0
    out = _sampler([_line(t - 1.0, 1965), _line(t + 1.0, 1900)]).stop((t, t + 0.05))
    assert out["samples"] == 2 and "window" in out


def test_without_a_window_every_sample_counts():
    t = 1_700_000_000.0
    out = _sampler([_line(t, 1900), _line(t + 0.02, 1700)]).stop()
    assert out["samples"] == 2 and out["sm_mhz"] == pytest.approx(1800.0)


class _DoneThread:
    def join(self):
        pass


def test_nvml_samples_inside_the_window_and_reason_bits():
    t = 1_700_000_000.0
    s = object.__new__(bench.ClockSampler)
    s.thread = _DoneThread()
    s.source = "nvml, 2 ms"
    s.samples = [(t - 0.01, 1965.0, 1965.0, set(), 300.0),
                 (t + 0.002, 1950.0, 1965.0, {"sw_power_cap"}, 990.0),
                 (t + 0.004, 1930.0, 1965.0, set(), 995.0),
                 (t + 0.2, 1965.0, 1965.0, {"hw_slowdown"}, 400.0)]
    out = s.stop((t, t + 0.01))
    assert out["samples"] == 2 and out["sm_mhz"] == pytest.approx(1940.0)
    assert out["reasons"] == ["sw_power_cap"] and out["power_w_max"] == 995.0
    assert out["source"] == "nvml, 2 ms"
    assert bench.ClockSampler.REASONS[0x4] == "sw_power_cap"
