"""Host-side checks of bench.py (CPU only): the reference arm's JSON line
(it times the oracle, so it runs without a GPU) and the rule that a
recorded DRAM traffic figure is reported only for the sources it was
captured on."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                          "--warmup", "3", "--quiet"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["steps"] == 2 and d["warmup"] == 3 and d["higher_is_better"] is True and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == bench.WORKLOAD


def test_traffic_only_for_the_captured_sources(monkeypatch):
    sha = bench.sources_sha("decode")
    monkeypatch.setitem(bench.TRAFFIC, "probe_key", {"bytes": 1000, "alg": 800, "sha": sha, "how": "test"})
    b, note = bench.traffic_of("probe_key", "decode", 1600)
    assert b == 2000 and "scaled" in note  # the recorded ratio times the leg's algorithmic bytes
    b, _ = bench.traffic_of("probe_key", "decode")
    assert b == 1000
    monkeypatch.setitem(bench.TRAFFIC, "probe_key", {"bytes": 1000, "alg": 800, "sha": "0" * 16, "how": "test"})
    b, note = bench.traffic_of("probe_key", "decode", 1600)
    assert b is None and note.startswith("stale")
    b, note = bench.traffic_of("no_such_key", "decode", 1600)
    assert b is None and "not captured" in note


def test_throughput_and_peaks():
    assert bench.job_throughput(100, 4, 10.0) == 100 * 4 / 0.010
    peak, kind = bench.hbm_peak()
    assert peak > 1000 and kind in ("measured", "fallback")
    alu, akind = bench.alu_peak()
    assert abs(alu - 148 * 128 * 1965e6 / 1e12) < 1.0 and akind.startswith("derived")
