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


def test_reference_arm_headline_rows_drawn_per_row():
    # the default headline (32-channel 4-bit layer) is far too large to draw
    # whole on the host: the reference arm draws only the rows it times
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
                        "--ref-rows", "2"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][0])
    assert d["config"]["seq_len"] == 16384 and d["config"]["label"] == "int4"
    assert d["cpu_baseline"]["cores"] >= 1 and "2 of 1024" in d["cpu_baseline"]["sample"]


def test_cpu_baseline_one_and_all_threads():
    import numpy as np
    import torch

    import bench
    import synth
    wl = synth.custom("bench-cpu", 91, b=2, hq=4, hkv=2, d=64, s=256, c=8, topk=16, kv_dtype="bf16",
                      label_dtype="int4", n_outlier=8, outlier_scale=6.0)
    di = synth.decode_inputs(wl)
    t = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    idx = torch.from_numpy(np.ascontiguousarray(synth.outlier_channels(wl), np.int32))
    rows = bench.DeviceRows(wl, t(di.q), t(di.k), t(di.v), idx)
    q, k, v, ir = rows.row(1, 1)
    assert q.shape == (1, 2, 64) and k.shape == (1, 1, 256, 64) and ir.shape == (1, 8)
    assert np.array_equal(k[0, 0], di.k[1, 1]) and np.array_equal(q[0], di.q[1, 2:4])
    cb = bench.cpu_baseline(wl, rows, 0.2)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["single_thread"]["value"] > 0
    assert 1 <= cb["cores"] <= (os.cpu_count() or 1) and cb["cpu_model"]
