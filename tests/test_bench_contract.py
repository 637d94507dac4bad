"""The reference arm of bench.py on CPU: one JSON line with the contract's
keys, the repo arm's metric and config keys, and a measured (not
extrapolated) step time."""
import json
import os
import subprocess
import sys

from conftest import ROOT

REPO_CONFIG_KEYS = {"workload", "m", "layers", "trellis_bytes_per_step", "l2", "timing", "api", "launch",
                    "parallelism"}


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    sys.path.insert(0, ROOT)
    import bench

    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert REPO_CONFIG_KEYS <= set(d["config"])
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    # the step time is the sampled work's own time: steps x ms_per_step is the
    # measured total, and the bytes over that time give the value
    total_bytes = d["config"]["trellis_bytes_per_step"] * d["steps"]
    assert abs(total_bytes / (d["ms_per_step"] * d["steps"] * 1e-3) / 1e9 - d["value"]) <= 0.05 * d["value"]
