"""The benchmark's reference arm (the CPU oracle timed on the host cores)
keeps the JSON-line contract of the GPU arm: one line from rank 0, the same
metric, unit and workload, its own cpu_baseline and an e2e object with no
host<->device bytes; other ranks print nothing and exit 0."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None):
    env = dict(os.environ)
    env.update(extra_env or {})
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                           "--warmup", "0"], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=600)


def test_reference_arm_json_line():
    p = _run()
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["unit"] == "pairs/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 0 and d["n_gpus"] == 1
    assert "L=16384" in d["config"]["workload"] and d["config"]["seq_len"] == 16384
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "pairs/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    # the step time is the stack's scored pairs at the measured rate, and the
    # line says it is extrapolated from bounded samples, with their seconds
    assert d["ms_per_step"] > 0
    assert d["extrapolated"] is True and d["measured_s"] > 0


def test_reference_arm_other_ranks_silent():
    p = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert p.returncode == 0, p.stderr[-2000:]
    assert not [l for l in p.stdout.splitlines() if l.startswith("{")]


def test_scored_pairs_counts_causal_rows_past_k():
    """The headline unit: an F layer scores the causal pairs (t, s <= t) of
    rows t >= k (rows t < k keep 0..t without a score), counted here by
    brute force."""
    sys.path.insert(0, ROOT)
    import bench
    for L, k, n_f in [(512, 64, 1), (100, 7, 3), (64, 64, 2), (50, 64, 1), (16384, 2048, 2)]:
        brute = n_f * sum(t + 1 for t in range(k, L))
        assert bench.scored_pairs(L, k, n_f) == brute
