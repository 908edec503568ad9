"""Host logic of bench.py that needs no GPU: which clock samples describe the
timed region, and when a recorded DRAM-traffic figure may be reported."""
import json
import os
import threading

import bench


def _sampler_with(samples, t_start, t_end):
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples = list(samples)
    s.t_open = min(t for t, *_ in samples) - 1.0
    s.t_start, s.t_end = t_start, t_end
    s._stop = threading.Event()
    s._thread = threading.Thread(target=lambda: None)
    s._thread.start()
    s._proc = None
    return s


def test_clock_samples_are_taken_from_the_timed_region():
    samples = [(0.0, 1200, 1965, {"sw_power_cap"}),   # warm-up, not reported
               (1.0, 1965, 1965, set()), (1.1, 1950, 1965, set()),
               (1.2, 1965, 1965, {"hw_slowdown"}), (1.3, 1965, 1965, set()),
               (5.0, 900, 1965, {"sw_thermal_slowdown"})]  # after the region
    out = _sampler_with(samples, 0.9, 1.35).stop()
    assert out["samples"] == 4 and out["window"] == "timed region"
    assert out["sm_mhz"] == 1965 and out["sm_min_mhz"] == 1950 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["hw_slowdown"]
    assert abs(out["timed_region_ms"] - 450.0) < 1e-6


def test_a_short_region_also_reports_the_warm_up_samples_and_says_so():
    samples = [(0.1, 1965, 1965, {"sw_power_cap"}), (0.2, 1960, 1965, set()),
               (1.0, 1965, 1965, set()), (9.0, 500, 1965, set())]
    out = _sampler_with(samples, 0.95, 1.05).stop()
    assert out["samples"] == 3  # everything up to the end of the region
    assert out["window"].startswith("warm-up and timed region")
    assert out["reasons"] == ["sw_power_cap"] and out["sm_min_mhz"] == 1960


def test_traffic_is_reported_only_for_the_kernel_source_it_was_taken_on(tmp_path, monkeypatch):
    root = tmp_path
    csrc = root / "logit_kl_divergence_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "kld_rows_kernel.cuh").write_text("int kernel = 1;  // kernel v1\n")
    (csrc / "kld_rows.cu").write_text("int launches = 1;\n")
    (csrc / "kld_internal.h").write_text("int header = 1;\n")
    (csrc / "kld_finish.cuh").write_text("int finishing = 1;\n")
    (root / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(root))
    h = bench.kernel_source_hash()
    rec = {"w": {"dram_bytes_per_launch": 123.0, "kernel_source_hash": h}}
    (root / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("w") == 123.0
    assert bench.recorded_traffic("other") is None
    # an edit of the comments alone keeps the record
    (csrc / "kld_rows_kernel.cuh").write_text("/* kernel */\nint kernel = 1;  // kernel v1, reworded\n\n")
    assert bench.kernel_source_hash() == h and bench.recorded_traffic("w") == 123.0
    (csrc / "kld_rows_kernel.cuh").write_text("int kernel = 2;  // kernel v2\n")   # the code changed since
    assert bench.kernel_source_hash() != h
    assert bench.recorded_traffic("w") is None
    h2 = bench.kernel_source_hash()
    (csrc / "kld_rows.cu").write_text("int launches = 2;\n")   # and so did its launch
    assert bench.kernel_source_hash() != h2

