"""The benchmark's multi-rank logic on CPU: two gloo ranks, each a replica.

The work does not shard (independent problems per replica), so the only
cross-rank steps are the barrier and the max-over-ranks of the timed figures;
the reported value is the sum of the replicas' work over the slowest time.
The reference arm runs on rank 0 only; other ranks exit without work.
"""

import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (10 + r) ms per step
        ms = bench.max_over_ranks(10.0 + rank, world, "cpu")
        out[rank] = (ms, bench.aggregate_tflops(1e12, world, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_with_two_gloo_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        ms, tf = out[r]
        assert ms == 11.0                         # every rank sees the slowest replica
        assert tf == pytest.approx(world * 1e12 / 11e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate_tflops(2e12, 1, 2.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""                 # the non-zero rank prints nothing and does no work


@pytest.mark.parametrize("Sq,Sk,left,right,causal", [(9, 9, 3, 0, True), (7, 12, 2, 1, False), (12, 7, -1, 2, False),
                                                     (10, 10, -1, -1, True), (10, 10, -1, -1, False),
                                                     (8, 8, 2, -1, False), (5, 3, 0, 1, False)])
def test_window_pair_count_matches_oracle_mask(Sq, Sk, left, right, causal):
    import bench
    import oracle
    assert bench.window_pairs(Sq, Sk, left, right, causal) == oracle.allowed_mask(Sq, Sk, causal, (left, right)).sum()
