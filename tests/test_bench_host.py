"""bench.py's host-side pieces without a GPU: the reference arm (the oracle timed on the host
cores) prints one JSON line with the contract's keys, and the per-launch traffic recorded
from ncu is reported only for the kernel source it was taken on."""
import io
import json
import os
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_arm_json_line():
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", "chunk480p", "--steps", "1",
                    "--warmup", "0"])
    lines = [ln for ln in buf.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC
    assert line["unit"] == "tokens/s" and line["value"] > 0
    assert line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] == 0
    assert line["higher_is_better"] is True and line["vs_baseline"] is None
    assert line["config"]["workload"].startswith("chunk480p")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert "tokens" in cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_print_nothing(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", "chunk480p", "--steps", "1",
                    "--warmup", "0"])
    assert buf.getvalue().strip() == ""


@pytest.mark.parametrize("matches", [True, False])
def test_recorded_traffic_follows_kernel_source(tmp_path, monkeypatch, matches):
    sha = bench.kernel_source_hash() if matches else "0" * 16
    rec = {"w/table": {"kernel_source_sha256_16": sha, "dram_bytes_per_launch": 12345}}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(path))
    assert bench.recorded_traffic("w", "table") == (12345 if matches else None)
    assert bench.recorded_traffic("other", "table") is None


def test_recorded_traffic_file_is_well_formed():
    with open(bench.PROFILE_TRAFFIC) as f:
        rec = json.load(f)
    assert rec
    for key, entry in rec.items():
        assert len(entry["kernel_source_sha256_16"]) == 16, key
        assert entry["dram_bytes_per_launch"] > 0, key


def test_cpu_baseline_reports_all_cores_and_one():
    w = bench.WORKLOADS["chunk480p"]()
    w.chunks = w.chunks[:1]
    host = bench.make_inputs(w, seed_offset=0)
    cb = bench.cpu_baseline(w, host, 0.6)
    assert cb["kind"] == "oracle" and cb["unit"] == "tokens/s"
    assert cb["value"] > 0 and cb["cores"] >= 1
    one = cb["single_thread"]
    assert one["value"] > 0 and one["unit"] == "tokens/s" and "one thread" in one["sample"]
