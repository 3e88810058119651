"""The benchmark's reference arm on CPU: the oracle, timed on host cores on a
bounded sample of the GPU arm's workload.  Its JSON line carries the GPU arm's
metric, unit, direction and config (one builder serves both arms), a
cpu_baseline describing the run and an e2e with no host-device traffic; under
more than one rank only rank 0 runs it.  The GPU arm's cpu_baseline legs
sample whole requests (or lm_head rows) up to a CPU-time budget."""
import argparse
import json
import os
import subprocess
import sys

import numpy as np

import bench
from trie_constrained_beam_fr_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                          env=env, timeout=600, cwd=ROOT)


def test_reference_line_matches_the_gpu_arm_contract():
    r = _run(["--impl", "reference", "--config", "serving", "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 0 and d["data"] == "synthetic"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}

    w = synth.WORKLOADS["serving"]
    sids = synth.workload_catalog(w)
    levels = bench.catalog_level_sizes(sids)
    args = argparse.Namespace(norm="full", temperature=0.0)
    assert d["config"] == bench.logits_config(w, args, levels)
    # the level sizes the device build reports: root, then distinct prefixes
    C = w.codebook_sizes
    assert levels[0] == 1 and levels[-1] == np.unique(sids, axis=0).shape[0]
    for l in range(1, len(levels)):
        assert levels[l - 1] <= levels[l] <= levels[l - 1] * C[l - 1]


def test_level_sizes_of_a_hand_catalog():
    sids = np.array([[0, 1, 2], [0, 1, 3], [0, 2, 0], [5, 0, 0], [0, 1, 2]], np.int32)  # one duplicate
    assert bench.catalog_level_sizes(sids) == [1, 2, 3, 4]


def test_reference_arm_runs_on_rank_zero_only():
    r = _run(["--impl", "reference", "--config", "serving", "--steps", "1", "--warmup", "0"],
             {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_cpu_baseline_samples_whole_requests_up_to_the_time_budget():
    w = synth.scaled(synth.WORKLOADS["tiny"], B=3)
    sids = synth.workload_catalog(w)
    one = bench.cpu_baseline_logits(w, sids, "full", 0.0, min_s=0.0)  # at least one request
    assert one["kind"] == "oracle" and one["cores"] == 1 and one["value"] > 0
    assert "requests 0..0 of tiny (1 of B=3)" in one["sample"]
    every = bench.cpu_baseline_logits(w, sids, "full", 0.0, min_s=1e9)  # at most B requests
    assert "requests 0..2 of tiny (3 of B=3)" in every["sample"]


def test_cpu_baseline_lmhead_takes_rows_four_at_a_time():
    w = synth.WORKLOADS["tiny"]
    rng = np.random.default_rng(0)
    weight = rng.integers(-128, 128, size=(w.V, 16)).astype(np.float32) / 8192.0
    rows = rng.integers(-128, 128, size=(10, 16)).astype(np.float32) / 64.0
    cb = bench.cpu_baseline_lmhead(w, rows, weight, min_s=1e9)
    assert cb["kind"] == "oracle" and cb["value"] > 0
    assert "for 10 rows of request 0" in cb["sample"]
    assert "(%d rows: 1 at step 0" % (1 + (w.depth - 1) * w.K) in cb["sample"]
