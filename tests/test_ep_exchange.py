"""Host side of the expert-parallel layer on two gloo ranks (CPU): the
buffers each rank exchanges, their sizes, and the in-process exchange that the
one-GPU tests use in place of the collective, against torch.distributed's
all_to_all_single and against the definition of the two passes."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import grouped_expert_gemm_router_b200 as moe
from grouped_expert_gemm_router_b200.ep import CapAndSpillEP, exchange_in_process

G = 2
# T tokens per rank, H, F, E, k, C: 16 experts, 8 per rank
SHAPE = dict(T=40, H=128, F=128, E=16, k=3, C=4)


def _shape():
    s = SHAPE
    return moe.make_shape(s["T"], s["H"], s["F"], s["E"], s["k"], C=s["C"], capacity=True)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _fill(ep, rank):
    """Seeded contents for every buffer the exchanges send."""
    g = torch.Generator().manual_seed(1000 + rank)

    def rnd(t):
        if t.dtype == torch.int32:
            t.copy_(torch.randint(0, 1 << 20, t.shape, generator=g, dtype=torch.int32))
        else:
            t.copy_(torch.randn(t.shape, generator=g).to(t.dtype))

    for t in (ep.b["x_perm"], ep.send_meta, ep.send_ovf, ep.back_cap, ep.back_ovf):
        rnd(t)



def _received(ep):
    return dict(recv_cap=ep.recv_cap, recv_meta=ep.recv_meta, recv_ovf=ep.recv_ovf,
                y_cap=ep.b["y"][:ep.cap_rows], recv_back_ovf=ep.recv_back_ovf)


def _as_np(t):
    return (t.view(torch.int16) if t.dtype == torch.bfloat16 else t).numpy().copy()


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world)
    try:
        ep = CapAndSpillEP(_shape(), world, device="cpu")
        _fill(ep, rank)

        def a2a(out, inp):
            # gloo has no 16-bit all-to-all: the bf16 rows go as their bytes
            if out.dtype == torch.bfloat16:
                out, inp = out.view(torch.uint8), inp.view(torch.uint8)
            dist.all_to_all_single(out, inp)

        ep.exchange_in(a2a)
        ep.exchange_out(a2a)
        dist.barrier()
        for k, t in _received(ep).items():
            np.save(os.path.join(out_dir, "%s_%d.npy" % (k, rank)), _as_np(t))
    finally:
        dist.destroy_process_group()


def test_buffer_sizes_follow_the_two_passes():
    s = _shape()
    ep = CapAndSpillEP(s, G, device="cpu")
    Eg, S = s.E // G, (min(s.k, s.E // G)) * (s.T - s.C)
    assert ep.S == S == moe.moe_ep_overflow_rows(s, G)
    assert ep.cap_rows == s.E * s.C
    assert ep.recv_cap.shape == (G * Eg * s.C, s.H) and ep.back_cap.shape == ep.recv_cap.shape
    for t in (ep.send_ovf, ep.recv_ovf, ep.back_ovf, ep.recv_back_ovf):
        assert t.shape == (G * S, s.H)
    assert ep.send_meta.shape == ep.recv_meta.shape == (G * 2 * Eg,)
    L = ep.local
    assert (L.T, L.H, L.F, L.E, L.k, L.C, L.flags) == (G * (Eg * s.C + S), s.H, s.F, Eg, 1, 0, 0)
    assert ep.x_loc.shape == ep.y_loc.shape == (L.T, s.H) and ep.h_loc.shape == (L.T, s.F)


def test_in_process_exchange_is_the_two_passes():
    """Block d of rank s's send buffer lands in block s of rank d's receive
    buffer, for every buffer of both directions."""
    ranks = [CapAndSpillEP(_shape(), G, device="cpu") for _ in range(G)]
    for r, ep in enumerate(ranks):
        _fill(ep, r)
    sent = [dict(cap=ep.b["x_perm"][:ep.cap_rows].clone(), meta=ep.send_meta.clone(), ovf=ep.send_ovf.clone(),
                 back_cap=ep.back_cap.clone(), back_ovf=ep.back_ovf.clone()) for ep in ranks]
    exchange_in_process(ranks, "exchange_in")
    exchange_in_process(ranks, "exchange_out")
    pairs = (("recv_cap", "cap"), ("recv_meta", "meta"), ("recv_ovf", "ovf"), ("y_cap", "back_cap"),
             ("recv_back_ovf", "back_ovf"))
    for d, ep in enumerate(ranks):
        got = _received(ep)
        for k_recv, k_sent in pairs:
            for s in range(G):
                assert torch.equal(got[k_recv].tensor_split(G)[s], sent[s][k_sent].tensor_split(G)[d]), (k_recv, d, s)


@pytest.mark.slow
def test_in_process_exchange_equals_gloo_all_to_all(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(G, port, str(tmp_path)), nprocs=G, join=True, start_method="spawn")
    ranks = [CapAndSpillEP(_shape(), G, device="cpu") for _ in range(G)]
    for r, ep in enumerate(ranks):
        _fill(ep, r)
    exchange_in_process(ranks, "exchange_in")
    exchange_in_process(ranks, "exchange_out")
    for r, ep in enumerate(ranks):
        for k, t in _received(ep).items():
            assert np.array_equal(np.load(tmp_path / ("%s_%d.npy" % (k, r))), _as_np(t)), (k, r)


def test_unsupported_expert_parallel_shapes():
    s = _shape()
    assert moe.moe_ep_overflow_rows(s, 3) == -1           # E % G != 0
    assert moe.moe_ep_overflow_rows(s, 0) == -1
    assert moe.moe_ep_workspace_bytes(s, 3) == 0
    uncapped = moe.make_shape(40, 128, 128, 16, 3)
    assert moe.moe_ep_overflow_rows(uncapped, 2) == -1
    with pytest.raises(moe.MoeError):
        moe.moe_ep_local_shape(uncapped, 2)
    # C >= T: no overflow rows at all
    assert moe.moe_ep_overflow_rows(moe.make_shape(40, 128, 128, 16, 3, C=40, capacity=True), 2) == 0
    # one rank per expert: at most one pair of a token per destination
    assert moe.moe_ep_overflow_rows(moe.make_shape(40, 128, 128, 16, 3, C=4, capacity=True), 16) == 36
