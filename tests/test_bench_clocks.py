"""Host logic of the bench's clock record: which nvidia-smi lines count for
the timed region (no GPU and no nvidia-smi needed: lines are injected)."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _line(mhz, power_cap="Not Active", thermal="Not Active"):
    return f"0, {mhz}, 1965, 700.0, 0x0, Not Active, Not Active, {thermal}, {power_cap}"


def _sampler(stamped, t0, t1, interval_ms=50):
    cs = bench.ClockSampler(0, interval_ms=interval_ms)
    cs.lines = [(t, _line(*v) if isinstance(v, tuple) else _line(v)) for t, v in stamped]
    cs.t0, cs.t1 = t0, t1
    return cs


def test_lines_inside_the_region_and_the_nearest_outside():
    cs = _sampler([(0.00, 1000), (0.90, 1500), (1.00, 1965), (1.05, 1965), (1.10, 1950), (1.14, 1965),
                   (1.30, 1200)], t0=0.98, t1=1.12)
    s = cs.summary()
    # 0.90 is more than one interval before t0; 1.14 is the first after t1; 1.30 is too late
    assert s["samples"] == 4 and s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == []


def test_region_shorter_than_the_interval_uses_the_bracketing_samples():
    cs = _sampler([(0.50, 1965), (0.55, 1950), (0.60, 1965)], t0=0.56, t1=0.58)
    s = cs.summary()
    assert s["samples"] == 2 and s["sm_mhz"] == (1950 + 1965) / 2


def test_throttle_reasons_are_reported():
    cs = _sampler([(1.0, (1800, "Active")), (1.05, (1700, "Not Active", "Active"))], t0=0.99, t1=1.06)
    s = cs.summary()
    assert s["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]


def test_no_lines_is_reported_as_not_sampled():
    cs = _sampler([], t0=1.0, t1=2.0)
    assert cs.summary()["reasons"] == ["not sampled"]


def test_profile_records_are_read_only_for_the_profiled_sources(tmp_path, monkeypatch):
    # traffic and pipe utilisation come from a committed ncu summary only while
    # the kernel's sources hash to the value recorded with it
    import hashlib
    import bench
    src = tmp_path / "k.cu"
    src.write_text("kernel source\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "k.md").write_text(f"source_sha256: {sha}\ndram_bytes_per_launch: 1234\n"
                               "    pipe_fma_heavy_pct: 74.3\n    issue_active_pct: 65.2\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k.md", ["k.cu"]) == 1234
    pipes = bench.profiled_pipes("k.md", ["k.cu"])
    assert pipes["pipe_fma_heavy"] == 0.743 and pipes["issue_active"] == 0.652
    src.write_text("changed\n")
    assert bench.profiled_traffic("k.md", ["k.cu"]) is None
    assert bench.profiled_pipes("k.md", ["k.cu"]) is None
