"""Host side of the peer-store expert-parallel layer (CPU, no kernel calls):
its sizes and refusals, the peer tables of ranks held by one process, and
the in-process counts all-gather against torch.distributed's all_gather on
two gloo ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import grouped_expert_gemm_router_b200 as moe
from grouped_expert_gemm_router_b200.ep_direct import DirectEP, connect_in_process, gather_counts_in_process

G = 2


def _shape(T=40, E=16, k=3):
    return moe.make_shape(T, 128, 128, E, k)


def test_local_rows_and_shape():
    s = _shape()
    for g in (1, 2, 4, 8, 16):
        Eg = 16 // g
        assert moe.moe_ep_direct_local_rows(s, g) == g * 40 * min(3, Eg)
        L = moe.moe_ep_direct_local_shape(s, g)
        assert (L.T, L.H, L.F, L.E, L.k, L.C, L.flags) == (g * 40 * min(3, Eg), 128, 128, Eg, 1, 0, 0)
        assert moe.moe_ep_direct_workspace_bytes(s, g) > 0


def test_unsupported_shapes():
    s = _shape()
    assert moe.moe_ep_direct_local_rows(s, 3) == -1                      # E % G != 0
    assert moe.moe_ep_direct_local_rows(s, 0) == -1
    capped = moe.make_shape(40, 128, 128, 16, 3, C=4, capacity=True)
    assert moe.moe_ep_direct_local_rows(capped, 2) == -1                 # uncapped layout only
    assert moe.moe_ep_direct_workspace_bytes(capped, 2) == 0
    big = moe.make_shape(40, 128, 128, 256, 3)
    assert moe.moe_ep_direct_local_rows(big, 16) > 0                     # G * E = 4096
    assert moe.moe_ep_direct_local_rows(big, 32) == -1                   # G * E > 4096
    with pytest.raises(moe.MoeError):
        moe.moe_ep_direct_local_shape(capped, 2)


def test_buffers_and_peer_tables():
    ranks = [DirectEP(_shape(), G, r, device="cpu") for r in range(G)]
    connect_in_process(ranks)
    for ep in ranks:
        assert ep.x_loc.shape == (ep.Tloc, 128) and ep.y_loc.shape == ep.x_loc.shape
        assert ep.b["y"].shape == (40 * 3, 128) and ep.cnt_all.shape == (G, 16)
        assert ep.peer_x_loc.tolist() == [r.x_loc.data_ptr() for r in ranks]
        assert ep.peer_y.tolist() == [r.b["y"].data_ptr() for r in ranks]
    with pytest.raises(moe.MoeError):
        DirectEP(_shape(), G, 0, device="cpu", x_loc=torch.empty((3, 128), dtype=torch.bfloat16))


def _fill_counts(ep, rank):
    ep.b["expert_counts"].copy_(torch.arange(16, dtype=torch.int32) * (rank + 1) + 100 * rank)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world)
    try:
        ep = DirectEP(_shape(), world, rank, device="cpu")
        _fill_counts(ep, rank)
        ep.gather_counts(lambda out, inp: dist.all_gather(list(out.unbind(0)), inp))
        dist.barrier()
        np.save(os.path.join(out_dir, "cnt_%d.npy" % rank), ep.cnt_all.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.slow
def test_in_process_counts_gather_equals_gloo_all_gather(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(G, port, str(tmp_path)), nprocs=G, join=True, start_method="spawn")
    ranks = [DirectEP(_shape(), G, r, device="cpu") for r in range(G)]
    for r, ep in enumerate(ranks):
        _fill_counts(ep, r)
    gather_counts_in_process(ranks)
    for r, ep in enumerate(ranks):
        assert np.array_equal(np.load(tmp_path / ("cnt_%d.npy" % r)), ep.cnt_all.numpy())
        for s in range(G):
            assert torch.equal(ep.cnt_all[s], ranks[s].b["expert_counts"])
