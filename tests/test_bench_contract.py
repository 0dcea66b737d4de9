"""The benchmark's reference arm on the host cores: its JSON line carries the keys
the benchmark contract asks for, and it times whole batches of the workload (never
more rows than the workload has)."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("extra", [[], ["--spherical"]])
def test_reference_arm_line_on_the_tiny_workload(extra):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                          "--steps", "2", "--warmup", "3", "--ref-seconds", "5"] + extra,
                         cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["config"]["workload"].startswith("tiny")
    assert d["config"]["method"] == ("spherical e-means" if extra else "e-means")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["unit"] == d["unit"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # a step is one batch of the tiny workload (1,024 rows of its 10,000), and the
    # rate counts the rows the oracle processed
    assert "2 oracle steps of 1024 rows each" in cb["sample"]
    assert abs(d["value"] - 2 * 1024 / (2 * d["ms_per_step"] / 1e3)) <= 1e-6 * d["value"]
