"""Host-side checks of bench.py's output contract, on the CPU.

The reference arm (the oracle timed on the host cores) runs without a GPU, so its JSON line,
its rank handling under a multi-process launch and the algorithmic byte count can be checked
here; the GPU arm's line is checked on a B200 by the benchmark run itself.
"""
import json
import os
import subprocess
import sys

import pytest

import bench
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
             "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"}


def run_bench(args, env_extra=None):
    env = dict(os.environ, **(env_extra or {}))
    env.pop("CUDA_VISIBLE_DEVICES", None)
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    return r


def test_reference_arm_line():
    r = run_bench(["--impl", "reference", "--steps", "3", "--warmup", "3", "--ref-tokens", "64",
                   "--workload", "tiny", "--group", "64"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert BASE_KEYS <= set(d)
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["higher_is_better"] is True and d["steps"] == 3 and d["warmup"] == 3
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"] == "tiny"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    r = run_bench(["--impl", "reference", "--steps", "3", "--warmup", "3", "--ref-tokens", "64",
                   "--workload", "tiny", "--group", "64"], {"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_rejects_fewer_than_three_warmups():
    r = run_bench(["--impl", "reference", "--steps", "1", "--warmup", "1", "--ref-tokens", "64",
                   "--workload", "tiny", "--group", "64"])
    assert r.returncode != 0


@pytest.mark.parametrize("name,group,expected", [
    ("llama31_8b_128k", 128, 18960),   # 4*32*128 + 2*8*128 + 8*64 + 2*8*1
    ("llama32_3b", 128, 14864),
    ("llama32_3b", 32, 14912),
    ("llama32_1b", 64, 9488),
    ("tiny", 64, 1348),
])
def test_algorithmic_bytes_per_token(name, group, expected):
    """4 Hq d_h (Q in and out, bf16) + 2 Hkv d_h (K in) + Hkv d_h / 2 (codes) + 2 Hkv d_h / g
    (fp16 scales)."""
    assert bench.algorithmic_bytes_per_token(synth.WORKLOADS[name], group) == expected


def test_oracle_step_on_host_threads_matches_one_thread():
    """The reference arm's threaded oracle step (token chunks per thread, sums added) gives
    the single-threaded step's angles and statistics (the same per-token arithmetic; the
    sums in another order)."""
    import numpy as np
    w = synth.WORKLOADS["tiny"]
    inp = synth.make_inputs(w)
    tables = bench.oracle_tables(w, False)
    one = bench.oracle_step(inp, w, "pairwise_hadamard", 64, tables, False)
    many = bench.oracle_step_threads(inp, w, "pairwise_hadamard", 64, tables, False, 5)
    dphi = np.abs(one["phi"].astype(np.float64) - many["phi"]) % (np.pi / 2)
    assert np.minimum(dphi, np.pi / 2 - dphi).max() < 1e-6
    np.testing.assert_allclose(many["stats"], one["stats"], rtol=1e-12)
