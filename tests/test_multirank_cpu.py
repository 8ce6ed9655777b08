"""The multi-GPU plumbing of bench.py on the CPU: two `gloo` ranks.

The layer's shards are logical and live on one GPU, so `bench.py --gpus N`
runs N independent replicas; torch.distributed carries only the barriers
around the timed regions and the max over ranks of each timing, and the job
value is N x (work per rank) / (slowest rank's time).  These tests run that
plumbing with world size 2 on the gloo backend (no GPU).
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    ranks = bench.Ranks.from_env("gloo", timeout_s=60)
    try:
        ranks.barrier()
        local_ms = 100.0 + 50.0 * rank          # rank 1 is the slow one
        slowest = ranks.max(local_ms)
        none_stays = ranks.max(None)
        rate = bench.job_rate(1000.0, ranks.world, slowest, steps=10)
        ranks.barrier()
        q.put((rank, ranks.world, slowest, none_stays, rate))
    finally:
        ranks.close()


def test_two_gloo_ranks_time_as_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    assert codes == [0, 0], codes
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, world, slowest, none_stays, rate in got:
        assert world == 2
        assert slowest == 150.0          # both ranks see the slowest rank's time
        assert none_stays is None
        # 2 ranks x 1000 units over 10 steps of 15 ms each
        assert rate == pytest.approx(2 * 1000.0 / 0.015)


def test_single_process_needs_no_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    sys.path.insert(0, ROOT)
    import bench
    r = bench.Ranks.from_env("gloo")
    assert r.world == 1 and r.dist is None
    assert r.max(3.5) == 3.5
    r.barrier()
    r.close()


def test_reference_arm_runs_on_rank_zero_only():
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload, ref_sample_tokens, warmup, steps = 5, 8, 0, 1

    assert bench.run_reference(Args, rank=1, world=2) is None
