"""Host logic of bench.py that decides what the measurement line reports:
the DRAM-traffic figure taken from the committed ncu summary only while its
recorded kernel-source digest matches the sources, the clock summary's
window and throttle reasons, the launch-count claim and the extra-path
record.  No GPU."""
import os

import pytest

import bench


def _profile(path, digest, dram="123456789"):
    path.write_text("# a summary\n"
                    f"kernel_source_digest: {digest}\n"
                    f"dram_bytes_per_launch: {dram}\n"
                    "algorithmic_bytes_per_launch: 1\n")
    return str(path)


def test_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PROFILE", _profile(tmp_path / "p.txt", bench.kernel_digest()))
    assert bench.profiled_traffic() == 123456789.0
    monkeypatch.setattr(bench, "PROFILE", _profile(tmp_path / "q.txt", "0" * 16))
    assert bench.profiled_traffic() is None
    monkeypatch.setattr(bench, "PROFILE", _profile(tmp_path / "r.txt", bench.kernel_digest(), dram="n/a"))
    assert bench.profiled_traffic() is None
    monkeypatch.setattr(bench, "PROFILE", str(tmp_path / "missing.txt"))
    assert bench.profiled_traffic() is None


def test_digest_follows_every_kernel_source(tmp_path, monkeypatch):
    copies = []
    for p in bench.KERNEL_SOURCES:
        q = tmp_path / os.path.basename(p)
        q.write_bytes(open(p, "rb").read())
        copies.append(str(q))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", copies)
    d0 = bench.kernel_digest()
    for q in copies:
        with open(q, "ab") as f:
            f.write(b"\n")
        d1 = bench.kernel_digest()
        assert d1 != d0
        d0 = d1


def test_the_committed_profile_names_a_digest_and_bytes():
    vals = {}
    with open(bench.PROFILE) as f:
        for line in f:
            if ":" in line:
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    assert len(vals["kernel_source_digest"]) == 16
    assert float(vals["dram_bytes_per_launch"]) > float(vals["algorithmic_bytes_per_launch"].split()[0]) * 0.99


def _sampler(samples, max_mhz=1965):
    s = bench.ClockSampler(0)
    s.ok = True
    s.max_mhz = max_mhz
    s.samples = samples
    return s


def test_clock_summary_inside_the_timed_region():
    samples = [(t, 1700 + t, 0x4 if t % 2 else 0x0) for t in range(10, 20)]
    out = _sampler(samples).summary(10, 19)
    assert out["window"] == "timed region" and out["samples_in_timed_region"] == 10
    assert out["sm_mhz"] == pytest.approx(1714.5)
    assert out["reasons"] == ["sw_power_cap"] and out["sm_max_mhz"] == 1965


def test_clock_summary_falls_back_to_the_load_window():
    samples = [(t, 1800, 0x0) for t in range(0, 10)] + [(10.5, 1600, 0x48)]
    out = _sampler(samples).summary(10, 11, t_load=5)
    assert out["samples_in_timed_region"] == 1
    assert out["window"] == "warm-up + timed region" and out["samples"] == 6
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]


def test_clock_summary_without_nvml():
    s = bench.ClockSampler(0)
    assert s.summary(0, 1)["reasons"] == ["nvml unavailable"]


def test_launch_count_claim():
    assert bench.launches_per_step(2047) == 3            # stream, merge, one-CTA reduction
    assert bench.launches_per_step(1_048_064) == 4       # the reduction clears, then one cooperative grid
    assert bench.launches_per_step(2047, world=8) == 16  # stream, merge, five shard steps


def test_extra_path_record_is_compact():
    rec = {"value": 1234.5678, "unit": "positions/s", "ms_per_step": 0.123456,
           "roofline": {"kernel_ms": 0.1111111, "bound": "hbm", "frac": 0.45678}}
    out = bench.compact_path(rec)
    assert out == {"value": 1234.6, "unit": "positions/s", "ms": 0.1235, "kernel_ms": 0.1111, "bound": "hbm",
                   "frac": 0.457}


def test_whole_job_rate_and_config():
    assert bench.whole_job_rate(2047, 4, 10, 2.0) == 2047 * 4 * 10 / 2.0
    c = bench.config_dict()
    assert c["n_rows"] == 2047 and c["vocab"] == 248_320 and "larger than L2" in c["l2"]
    assert "reduced profiling case" in bench.config_dict(rows=1024)["workload"]
    assert c["parallelism"].startswith("dp") and "dp8" in bench.config_dict(world=8)["parallelism"]
