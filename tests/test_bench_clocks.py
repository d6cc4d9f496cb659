"""bench.py's clock record: nvidia-smi CSV lines are summarised over the samples
taken inside the timed region (or over all of them, said so, when the region is
shorter than the sampling interval), with every throttle reason seen there."""
import datetime
import importlib.util
import os
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def line(t, mhz, power_cap=False):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    cap = "Active" if power_cap else "Not Active"
    return f"{ts}, {mhz}, 1965, 700.5, 0x0000000000000000, Not Active, Not Active, Not Active, {cap}"


def test_samples_inside_the_timed_region_are_kept():
    sampler = load_bench().ClockSampler
    t = time.time()
    lines = [line(t - 0.3, 1965), line(t + 0.005, 1850), line(t + 0.015, 1870, power_cap=True),
             line(t + 0.5, 1965)]
    s = sampler.parse(lines, (t, t + 0.02))
    assert s["window"] == "timed region" and s["samples"] == 2
    assert s["sm_mhz"] == 1860.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_a_region_without_samples_falls_back_to_the_whole_run():
    sampler = load_bench().ClockSampler
    t = time.time()
    s = sampler.parse([line(t, 1900), line(t + 0.02, 1950)], (t + 5, t + 6))
    assert s["window"] == "whole run" and s["samples"] == 2 and s["reasons"] == []


def test_unparsable_output_gives_no_clock():
    s = load_bench().ClockSampler.parse(["No devices were found", ""], None)
    assert s["sm_mhz"] is None and s["reasons"] == ["no samples"]
