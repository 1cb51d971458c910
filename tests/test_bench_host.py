"""Host logic of bench.py, on the CPU:
- the clock record that decides whether a timed run stands (median SM clock under load,
  throttle reasons);
- the source hash that keys the recorded DRAM traffic (blind to comments, not to code);
- the time-sized sample of the oracle's CPU baseline."""
import os
import shutil
import time

import bench


def _line(sm, watts, power_cap="Not Active", thermal="Not Active"):
    return (f"0, {sm} MHz, 1965 MHz, {watts:.2f} W, 0x0000000000000004, Not Active, Not Active, "
            f"{thermal}, {power_cap}\n")


def test_clock_summary_takes_the_loaded_median_and_the_active_reasons(tmp_path):
    path = tmp_path / "clocks.csv"
    lines = [_line(1965, 90.0)] * 5                                  # idle before the region
    lines += [_line(1590, 780.0, power_cap="Active")] * 7 + [_line(1620, 760.0)] * 4
    lines += ["garbage line\n", _line(1965, 95.0)]
    path.write_text("".join(lines))
    cs = bench.ClockSampler(0)
    cs.proc, cs.path = object(), str(path)
    s = cs.summary()
    assert s["sm_mhz"] == 1590.0            # median over the 11 loaded samples only
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 17 and s["power_w_max"] == 780.0
    path.write_text(_line(1500, 700.0, thermal="Active"))
    assert bench.ClockSampler.summary(cs)["reasons"] == ["sw_thermal_slowdown"]


def test_gemm_source_hash_ignores_comments_and_sees_code(tmp_path, monkeypatch):
    csrc = tmp_path / "epilogues_nvfp4_quantize_b200" / "csrc"
    shutil.copytree(os.path.join(bench.ROOT, "epilogues_nvfp4_quantize_b200", "csrc"), csrc)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.gemm_source_hash()
    monkeypatch.undo()
    assert base == bench.gemm_source_hash()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    gemm = csrc / "gemm.cuh"
    text = gemm.read_text()
    gemm.write_text("// a new comment line\n/* and a block\n comment */\n" + text.replace("\n", "\n\n", 3))
    assert bench.gemm_source_hash() == base
    gemm.write_text(text.replace("constexpr int STAGES = 5;", "constexpr int STAGES = 4;"))
    assert bench.gemm_source_hash() != base


class _SleepyLayer:
    """Stands in for the oracle: its step takes 0.1 ms per row."""
    pack_s = 0.0

    def __init__(self):
        self.calls = []

    def step(self, rows):
        self.calls.append(len(rows))
        time.sleep(1e-4 * len(rows))


def test_cpu_baseline_sizes_its_sample_by_time():
    layer = _SleepyLayer()
    out = bench.cpu_baseline(16384, target_s=0.6, layer=layer)
    n = int(out["sample"].split()[0])
    # 0.6 s at 0.1 ms a row is at most 6000 rows; sleeping overhead only lowers it
    assert 2000 <= n <= 6000 and n % 64 == 0
    assert sum(layer.calls) >= 256 + n                  # the probe, then the sized sample
    assert max(layer.calls) <= 1024                     # run in chunks of at most 1024 rows
    assert out["kind"] == "oracle" and out["value"] > 0
    assert "one_core" in out


def test_cpu_baseline_sample_is_capped_at_the_workload():
    layer = _SleepyLayer()
    out = bench.cpu_baseline(512, target_s=5.0, layer=layer)
    assert out["sample"].startswith("512 random rows")
    assert out["value"] > 0 and max(layer.calls) == 512
