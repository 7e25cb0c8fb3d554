"""bench.py's multi-GPU path is replicas only: each rank runs the whole layer
on its own token batch, the job's time is the slowest rank's, and the rate is
every rank's tokens over that time.  The rank logic runs here on the CPU
with two gloo ranks."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world)
    try:
        # each rank times its own replica; the job takes the slowest per entry
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 5.0])
        dist.barrier()
        np.save(os.path.join(out_dir, "r%d.npy" % rank), np.array(got))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    for r in range(2):
        assert np.load(tmp_path / ("r%d.npy" % r)).tolist() == [2.0, 10.0, 5.0]


def test_single_process_is_unchanged():
    assert bench.max_over_ranks([3.5, 1.25]) == [3.5, 1.25]


def test_whole_job_rate_counts_every_replica():
    # 2 replicas x 10 steps x 512 tokens in 20 ms of the slowest replica
    assert bench.whole_job_rate(512, 10, 2, 20.0) == pytest.approx(512 * 10 * 2 / 0.020)
    assert bench.whole_job_rate(512, 10, 1, 20.0) * 2 == pytest.approx(bench.whole_job_rate(512, 10, 2, 20.0))


def test_replicas_get_their_own_tokens_and_the_same_weights():
    cfg = synth.CONFIGS[1]
    L = synth.make_layer(cfg)
    x0 = bench.replica_tokens(cfg, 0, L)
    x1 = bench.replica_tokens(cfg, 1, L)
    assert np.array_equal(x0, L.x)
    assert x1.shape == x0.shape and not np.array_equal(x1, x0)
    assert np.array_equal(x1, bench.replica_tokens(cfg, 1, L))  # seeded: the same on every call
