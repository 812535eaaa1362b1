"""The benchmark's reference arm (the oracle on the host cores) on CPU: one
JSON line with the contract's keys, the same `config` object the CUDA arm
builds for the workload, and zero host-device bytes.  Rank > 0 of a
multi-rank launch prints nothing."""
import json
import os
import subprocess
import sys

import bench
from speculative_decoding_verification_91_b200.inputs import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra, *args):
    env = dict(os.environ, **env_extra)
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", *args], cwd=ROOT,
                         env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    return [l for l in out.stdout.splitlines() if l.strip()]


def test_reference_line_on_the_tiny_workload():
    lines = _run({}, "--workload", "tiny", "--steps", "3", "--warmup", "3")
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3
    assert d["metric"] == bench.METRIC and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0
    wl = W.get_workload("tiny")
    cfg = d["config"]
    assert set(cfg) == set(bench.workload_config(wl, [1], 1, "").keys())
    assert cfg["workload"] == "tiny" and cfg["context"] == [int(x) for x in W.context_lengths(wl)]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_config_uses_the_stored_inputs():
    # the full-size workloads carry margin-guarded inputs; both arms name them
    wl = W.get_workload("b1_ctx8k")
    fx = bench.fixture_inputs(wl)
    assert fx is not None and "verify_b1_ctx8k.json" in fx["inputs"]
    assert len(fx["drafts"][0]) == wl.k
    if fx["draws"]:             # independent batch-1 draws of the acceptance recipe
        assert len(fx["drafts"]) == len(fx["draw_tokens"]) >= 16
        assert fx["tokens_per_step"] == round(sum(fx["draw_tokens"]) / len(fx["draw_tokens"]), 4)
        assert max(fx["draw_tokens"]) > 1
    else:
        assert len(fx["drafts"]) == wl.batch
        assert fx["tokens_per_step"] >= wl.batch


def test_reference_arm_other_ranks_print_nothing():
    assert _run({"RANK": "1", "WORLD_SIZE": "2"}, "--workload", "tiny", "--steps", "3",
                "--warmup", "3") == []
