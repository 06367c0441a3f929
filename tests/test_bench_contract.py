"""The parts of bench.py's output contract that need no GPU: the weight
replica schedule of the timed decode steps and the reference arm (the CPU
oracle timed on the same metric and workload) with its JSON line."""
from __future__ import annotations

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_replica_schedule_never_feeds_a_launch_from_l2():
    sys.path.insert(0, ROOT)
    import bench

    wbytes, _ = bench.step_bytes()
    R = 22
    assert R * wbytes > 3 * 126 * 2**20                      # the replicas exceed 3x the L2 size
    seq = [bench.replica_of(step, j, R) for step in range(3 * R) for j in range(len(bench.MS))]
    assert all(a != b for a, b in zip(seq, seq[1:]))         # consecutive launches, within and across steps
    last = {}
    for i, r in enumerate(seq):
        if r in last:
            assert i - last[r] == R                          # a replica returns only after R launches
        last[r] = i
    assert sorted(set(seq)) == list(range(R))


def test_reference_arm_json_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    env.pop("WORLD_SIZE", None)
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3",
                          "--ref-budget-s", "1"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["higher_is_better"] is True and d["value"] > 0 and d["steps"] == 2 and d["warmup"] >= 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 2
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("decode125m")
