"""The bench's reference arm (the float64 oracle on host cores) prints one JSON line that
keeps the bench contract: metric, value, unit, steps, timing and the baseline blocks."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    out = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in out, key
    assert out["impl"] == "reference"
    assert out["steps"] == 1 and out["warmup"] == 3 and out["n_gpus"] == 1
    assert out["value"] > 0 and out["higher_is_better"] is True
    assert "workload" in out["config"]
    cb = out["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == out["value"]
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["e2e"]["d2h_bytes_per_step"] == 0


def test_warmup_below_three_is_refused():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "2"], cwd=ROOT, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode != 0


def test_config_block_describes_every_workload():
    """Every configuration's history kind (uniform, fixed, lognormal) and mode (scoring or
    training) is named in the bench line's workload description."""
    sys.path.insert(0, ROOT)
    import bench
    from gen import CONFIGS

    for name, cfg in CONFIGS.items():
        c = bench.config_block(cfg, 2)
        w = c["workload"]
        assert name in w and c["config"] == name
        assert ("training step" in w) == cfg.training
        assert ("inference scoring" in w) == (not cfg.training)
        kind = cfg.hist[0]
        assert {"uniform": "U[", "fixed": "every history at", "lognormal": "lognormal("}[kind] in w
        assert c["global_batch_users"] == 2 * cfg.B
        assert c["candidates_per_step"] == 2 * cfg.B * cfg.m
    assert bench.DEFAULT_CONFIG == "c2"
