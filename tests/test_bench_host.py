"""bench.py's host logic (no GPU): the reference arm's JSON line, and the roofline's
traffic figure being dropped once the kernel source no longer matches its ncu capture.

The reference arm runs on a two-matmul subset of the step with a shortened CPU budget, so that the
line's keys and their consistency are checked in seconds; the full arm differs only in
the matmuls it samples and the time it spends.
"""
import argparse
import hashlib
import json

import bench


def _args(steps=3, warmup=1, gpus=1):
    return argparse.Namespace(impl="reference", steps=steps, warmup=warmup, gpus=gpus)


def test_reference_line(monkeypatch, capsys):
    monkeypatch.setattr(bench, "STEP_ORDER", ["tiny", "gemv_m1"])
    monkeypatch.setattr(bench, "REFERENCE_SECONDS", 0.4)
    bench.reference_arm(_args(), world=1, rank=0)
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["steps"] == 3 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["ms_per_step"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert cb["unit"] == d["unit"] and cb["sample"] == d["config"]["sample"]
    e2e = d["e2e"]
    assert e2e == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}
    # the workload the line names is the one both arms report
    want = bench.step_config(1, 0.0, 0.0)
    for key in ("workload", "tokens", "encoder_tokens", "out_dtype", "parallelism"):
        assert d["config"][key] == want[key]


def test_reference_other_ranks_print_nothing(monkeypatch, capsys):
    monkeypatch.setattr(bench, "STEP_ORDER", ["tiny"])
    monkeypatch.setattr(bench, "REFERENCE_SECONDS", 0.2)
    bench.reference_arm(_args(gpus=2), world=2, rank=1)
    assert capsys.readouterr().out.strip() == ""


def test_traffic_follows_the_kernel_source(monkeypatch, tmp_path):
    src = tmp_path / "kernel.cuh"
    src.write_bytes(b"// a kernel\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    prof = tmp_path / "profile.md"
    prof.write_text(f"kernel_source_sha256: {sha}\ntraffic_bytes_per_launch_full: 1234\n")
    monkeypatch.setattr(bench, "TC_SOURCE", str(src))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(prof))
    assert bench.ncu_traffic() == (1234.0, None)
    src.write_bytes(b"// a kernel, changed\n")
    traffic, note = bench.ncu_traffic()
    assert traffic is None and note
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.md"))
    assert bench.ncu_traffic() == (None, None)


def test_peaks_come_from_the_measured_file():
    peaks = bench.load_peaks()
    assert peaks["hbm_gbs"] > 0 and peaks["tflops_burst"] >= peaks["tflops_sustained"] > 0
    assert peaks["source"] in ("measured", "fallback")
