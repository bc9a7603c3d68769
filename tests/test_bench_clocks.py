"""bench.py's clock record on CPU: parsing nvidia-smi's CSV samples (only
this GPU's rows, complete rows) and the summary the JSON line carries
(median SM clock under load, the maximum clock, the throttle reasons seen
under load)."""
import bench


def _row(sm, util, reasons=(), uuid="GPU-aaaa", smax=1965):
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    flags = ["Active" if n in reasons else "Not Active" for n in names]
    return ["2026/01/01 00:00:00.000", uuid, str(sm), str(smax), "700.0", str(util), *flags]


def test_summary_takes_the_loaded_samples():
    rows = [_row(1980, 0), _row(1965, 100), _row(1950, 98, ("sw_power_cap",)), _row(1900, 97),
            _row(345, 10, ("hw_slowdown",))]
    s = bench.ClockSampler.summarise(rows, 1965)
    assert s["sm_mhz"] == 1950.0                # median of 1965, 1950, 1900
    assert s["reasons"] == ["sw_power_cap"]     # the idle sample's reason is not counted
    assert s["sm_max_mhz"] == 1965.0
    assert s["samples"] == 5 and s["samples_under_load"] == 3


def test_summary_without_load_uses_every_sample():
    rows = [_row(1200, 0), _row(1300, 5, ("hw_thermal_slowdown",))]
    s = bench.ClockSampler.summarise(rows, 1965)
    assert s["sm_mhz"] == 1250.0
    assert s["reasons"] == ["hw_thermal_slowdown"]


def test_summary_of_no_samples():
    s = bench.ClockSampler.summarise([], 1965)
    assert s["sm_mhz"] is None and s["sm_max_mhz"] == 1965 and s["reasons"] == []


def test_stop_keeps_complete_rows_of_this_gpu():
    lines = [", ".join(_row(1965, 100)), ", ".join(_row(1965, 100, uuid="GPU-bbbb")),
             "2026/01/01 00:00:00.100, GPU-aaaa, 1965",  # cut short when the sampler stopped
             ", ".join(_row(1950, 99))]

    class Proc:
        def terminate(self):
            pass

        def communicate(self, timeout=None):
            return "\n".join(lines) + "\n", ""

    smp = bench.ClockSampler("GPU-aaaa")
    smp.proc = Proc()
    rows = smp.stop()
    assert len(rows) == 2 and all(r[1] == "GPU-aaaa" for r in rows)
    assert bench.ClockSampler.summarise(rows, 1965)["sm_mhz"] == 1957.5
