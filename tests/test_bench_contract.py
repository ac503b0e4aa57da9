"""The JSON line contract of bench.py, checked on its CPU arm (no GPU needed).

`bench.py --impl reference` times the CPU fp64 oracle on a bounded sample of the
layer step and prints one line with the keys, units and `config` of the
tensor-core arm, so the two lines pair up; under a multi-rank launch only rank 0
prints.
"""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None, *args):
    env = dict(os.environ, **(extra_env or {}))
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    return [json.loads(l) for l in p.stdout.splitlines() if l.startswith("{")]


def test_reference_line_keys_and_config():
    lines = _run(None, "--steps", "1", "--warmup", "1")
    assert len(lines) == 1
    d = lines[0]
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["warmup"] >= 3, "at least three warm-up steps, whatever was asked"
    assert d["config"] == bench.layer_config(1)
    assert d["value"] > 0 and d["ms_per_step"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_prints_only_on_rank_0():
    assert _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, "--gpus", "2", "--steps", "1") == []
    lines = _run({"RANK": "0", "WORLD_SIZE": "2", "LOCAL_RANK": "0"}, "--gpus", "2", "--steps", "1")
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2 and lines[0]["config"] == bench.layer_config(2)


def test_layer_config_counts_the_whole_step():
    c = bench.layer_config(1)
    f = bench.layer_flops(4, 2048, 10, 128, 1280, 512)
    assert c["gflop_per_step"] == round(f["total"] / 1e9, 3)
    # attention fwd 18.80 + bwd 46.99, projection fwd 53.69 + bwd 107.37 GFLOP
    assert abs(f["attn_fwd"] / 1e9 - 18.797) < 0.01 and abs(f["proj_fwd"] / 1e9 - 53.687) < 0.01
    assert bench.layer_config(8)["global_batch"] == 32
