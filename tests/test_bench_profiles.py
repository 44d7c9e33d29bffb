"""Host checks of the bench's bookkeeping: the committed ncu traffic summary
of the dominant kernel is found under the name the bench looks up, and its
DRAM bytes are reported only while the kernel source it was taken on is
unchanged; the --metric switch picks the plans' and the oracle's spatial
test together."""
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fields(path):
    kv = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    return kv


def test_traffic_summary_exists_under_the_bench_kernel_name():
    path = os.path.join(ROOT, "profiles", f"{bench.ROOFLINE_KERNEL}_wan720_traffic.txt")
    assert os.path.exists(path)
    kv = _fields(path)
    assert kv["kernel"] == bench.ROOFLINE_KERNEL and kv["workload"] == "wan720"
    # the per-launch figure is the captured one scaled by the units (heads): 40 of the capture's
    assert float(kv["dram_bytes_per_launch"]) == float(kv["captured_dram_bytes"]) * 40 / int(kv["captured_heads"])
    got = bench.recorded_traffic(bench.ROOFLINE_KERNEL, "wan720")
    if kv["source_sha256"] == bench.source_sha256():
        assert got == float(kv["dram_bytes_per_launch"])
    else:
        assert got is None


def test_stale_or_missing_summary_reports_no_traffic(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic(bench.ROOFLINE_KERNEL, "wan720") is None
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / f"{bench.ROOFLINE_KERNEL}_wan720_traffic.txt").write_text(
        "source_sha256: 0000\ndram_bytes_per_launch: 123\n")
    assert bench.recorded_traffic(bench.ROOFLINE_KERNEL, "wan720") is None
    (tmp_path / "profiles" / f"{bench.ROOFLINE_KERNEL}_wan720_traffic.txt").write_text(
        f"source_sha256: {bench.source_sha256()}\ndram_bytes_per_launch: 123\n")
    assert bench.recorded_traffic(bench.ROOFLINE_KERNEL, "wan720") == 123.0


def test_query_group_default_follows_the_plan():
    """--qsort auto turns radius-sorted query groups on where the plan accepts
    them (at most four tile rows per frame) and a tile-column strip holds more
    than one tile."""
    import dataclasses
    import pytest
    from sparse_attention_video_tra_b200 import TRA_FLAG_QSORT, TraError, synth
    W = synth.WORKLOADS
    assert bench.query_group_flags("auto", W["wan720"]) == TRA_FLAG_QSORT       # 3 tile rows of 16
    assert bench.query_group_flags("auto", W["hunyuan720"]) == TRA_FLAG_QSORT
    assert bench.query_group_flags("auto", W["len4x"]) == TRA_FLAG_QSORT
    assert bench.query_group_flags("auto", W["wan480"]) == 0                    # 1 tile row of 32
    assert bench.query_group_flags("on", W["wan480"]) == TRA_FLAG_QSORT
    assert bench.query_group_flags("off", W["wan720"]) == 0
    tall = dataclasses.replace(W["wan720"], H=200, W=200)                      # 13 tile rows
    assert bench.query_group_flags("auto", tall) == 0
    with pytest.raises(TraError):
        bench.query_group_flags("on", tall)


def test_metric_switch_selects_the_disk_plans_and_oracle_metric():
    """`--metric disk` adds TRA_FLAG_DISK to the plan flags and sends the
    oracle legs to the oracle's disk metric; the default stays the Chebyshev
    square.  The reference arm's line names the spatial test it ran."""
    import argparse
    import json
    import subprocess
    import sys
    import oracle
    from sparse_attention_video_tra_b200 import TRA_FLAG_DISK, synth
    wl = synth.WORKLOADS["tiny"]
    disk = argparse.Namespace(qsort="off", metric="disk")
    square = argparse.Namespace(qsort="off", metric="square")
    assert bench.plan_flags(disk, wl) == TRA_FLAG_DISK
    assert bench.plan_flags(square, wl) == 0
    assert bench.oracle_metric(disk) == oracle.DISK
    assert bench.oracle_metric(square) == oracle.CHEBYSHEV
    names = {}
    for m in ("square", "disk"):
        p = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--metric", m,
                            "--steps", "1", "--warmup", "0"], cwd=ROOT, capture_output=True, text=True, timeout=600)
        assert p.returncode == 0, p.stderr[-3000:]
        line = [json.loads(x) for x in p.stdout.splitlines() if x.startswith("{")][-1]
        assert line["impl"] == "reference" and line["value"] > 0
        names[m] = line["config"]["metric"]
    assert names == {"square": "Chebyshev square", "disk": "Euclidean disk (TRA_FLAG_DISK)"}


def test_peaks_are_labelled_by_their_source(tmp_path, monkeypatch):
    """Each roofline denominator is the measured file's number when the file
    holds one under that key, else the recipe's fallback, labelled as such."""
    import json
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.peak_value("bf16_tflops_sustained") == (1400.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6537.0, "bf16_tflops": "n/a"}))
    assert bench.peak_value("hbm_gbs") == (6537.0, "measured")
    assert bench.peak_value("bf16_tflops") == (1590.0, "fallback")
    assert bench.peak_value("bf16_tflops_sustained") == (1400.0, "fallback")
