"""The clock record of bench.py's JSON line, from nvidia-smi samples taken
during the timed region: the median SM clock over the samples under load,
the maximum clock, and each throttle reason that was active in any sample
(a run that saw hw_slowdown, hw_thermal_slowdown or sw_thermal_slowdown is
rejected by whoever reads the line; sw_power_cap is kept and noted).  The
summary runs here on canned nvidia-smi output, with no GPU."""
import bench

# index, clocks.sm, clocks.max.sm, power.draw, reasons.active, hw_slowdown,
# hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
IDLE = "0, 345, 1965, 190.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"


def _load(mhz, cap=False, hw=False):
    return (f"0, {mhz}, 1965, 998.1, 0x4, {'Active' if hw else 'Not Active'}, Not Active, Not Active, "
            f"{'Active' if cap else 'Not Active'}\n")


def test_median_over_loaded_samples_and_power_cap_noted():
    lines = [IDLE, _load(1680, cap=True), _load(1700), _load(1710, cap=True), IDLE]
    r = bench.ClockSampler.summarize(lines)
    assert r["sm_mhz"] == 1700.0          # idle samples (below half the max) are left out
    assert r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]
    assert r["samples"] == 5


def test_hardware_slowdown_is_reported():
    r = bench.ClockSampler.summarize([_load(1500), _load(1490, hw=True)])
    assert r["reasons"] == ["hw_slowdown"]


def test_unparsable_and_short_lines_are_skipped():
    lines = ["", "garbage\n", "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active\n",
             _load(1600)]
    r = bench.ClockSampler.summarize(lines)
    assert r["samples"] == 1 and r["sm_mhz"] == 1600.0 and r["reasons"] == []


def test_no_samples():
    r = bench.ClockSampler.summarize([])
    assert r["sm_mhz"] is None and r["samples"] == 0 and r["reasons"] == []


def test_all_idle_samples_still_give_a_median():
    r = bench.ClockSampler.summarize([IDLE, IDLE])
    assert r["sm_mhz"] == 345.0
