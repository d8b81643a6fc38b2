"""The reference arm of ``bench.py`` (the float64 oracle on the host cores) on CPU: one JSON line with the base
contract's keys, the same config object as the GPU arm, and the reference-specific keys (impl, cpu_baseline,
e2e without copies)."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny", "--steps", "3", "--warmup", "1"], capture_output=True, text=True, cwd=ROOT,
                         timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["steps"] == 3 and j["warmup"] == 1 and j["n_gpus"] == 1
    assert j["value"] > 0 and j["unit"] == "tokens/s" and j["higher_is_better"] is True
    assert j["config"]["workload"] == "tiny" and j["config"]["T"] == 256
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == j["value"]
    e = j["e2e"]
    assert e["value"] == j["value"] and e["unit"] == j["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0
    # the same config object as the GPU arm's
    sys.path.insert(0, ROOT)
    import bench
    import synth
    wl = synth.get_workload("tiny")
    assert j["config"] == bench.bench_config(wl, j["config"]["capacity"], 1)
