"""The benchmark's reference arm (the CPU oracle) runs without a GPU and
prints one JSON line with the contract's keys; and the L2 rotation count
covers twice the L2 with the step's working set."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "0", "--steps", "2",
                        "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_rotation_count_covers_twice_the_l2():
    import math

    import bench
    import synth
    l2 = 126 * 2 ** 20
    for i in (1, 3):
        ws = bench.algorithmic_bytes(synth.workload(i), 2)["total"]
        r = math.ceil(2 * l2 / ws)
        assert r * ws >= 2 * l2 and r == 4
    for i in (2, 4):  # these working sets exceed twice the L2 by themselves
        assert bench.algorithmic_bytes(synth.workload(i), 2)["total"] >= 2 * l2
