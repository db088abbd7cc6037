"""The benchmark's multi-rank logic on CPU (gloo, world size 2): each rank
times its own independent layer, the job time is the max over ranks, and the
whole-job value counts every rank's tokens (weak scaling, no data-path
collective)."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (rank, rank, world)
        local = 1.0 + rank * 0.5          # rank 1 is slower
        m = bench.reduce_max(local)
        bench.barrier()
        q.put((rank, m, bench.job_value(8, world, 100, m)))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in res:
        assert m == pytest.approx(1.5)
        assert v == pytest.approx(8 * 2 * 100 / 1.5)


def test_single_rank_identity():
    import bench
    assert bench.reduce_max(3.25) == 3.25
    assert bench.job_value(8, 1, 10, 2.0) == 40.0


def test_algorithmic_bytes_match_hand_count():
    """Per-launch bytes of the Llama-2-7B-shaped layer: label 8*32*4096*32 B,
    selected K+V 8*32*256*256*2 B, q and bf16 out 8*32*128*2 B each."""
    import bench
    import synth
    ab = bench.algorithmic_bytes(synth.workload(1), out_esz=2)
    assert ab["label"] == 33554432 and ab["kv_selected"] == 33554432 and ab["q_out"] == 131072
    assert ab["append"] == 8 * 32 * (256 + 32)  # new token's key row read + label row written
    assert ab["total"] == 67239936 + 8 * 32 * 288
    ab2 = bench.algorithmic_bytes(synth.workload(2), out_esz=2)
    assert ab2["label"] == 32 * 32 * 16384 * 20  # 16 B payload + fp16 scale + fp16 zero
