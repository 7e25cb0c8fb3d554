"""The expert-parallel forward() orchestrations on the host (CPU, no kernel
calls): the kernel phases are replaced by stand-ins, so what runs is the
sequence of phases and collectives each forward() issues.

Two-pass form: two gloo ranks run the real forward(); the stand-in "experts"
send every received row straight back, so after the two return passes each
rank's y capacity rows and overflow slots must hold exactly the rows it sent
(the exchange is its own inverse).  Peer-store form: a recorded run checks the
order of phases and collectives (counts all-gather, plan and dispatch, barrier,
experts with the fused return, barrier, combine)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import grouped_expert_gemm_router_b200 as moe
from grouped_expert_gemm_router_b200.ep import CapAndSpillEP
from grouped_expert_gemm_router_b200.ep_direct import DirectEP

G = 2


def _shape():
    return moe.make_shape(40, 128, 128, 16, 3, C=4, capacity=True)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _stub(ep, rank):
    g = torch.Generator().manual_seed(77 + rank)

    def route_and_pack(x, w_router, bias, stream=None):
        ep.b["x_perm"].copy_(torch.randn(ep.b["x_perm"].shape, generator=g).to(torch.bfloat16))
        ep.send_ovf.copy_(torch.randn(ep.send_ovf.shape, generator=g).to(torch.bfloat16))
        ep.send_meta.copy_(torch.arange(ep.send_meta.numel(), dtype=torch.int32) + 1000 * rank)

    def local_experts(w_gate, w_up, w_down, stream=None):
        ep.back_cap.copy_(ep.recv_cap)   # every received row goes straight back
        ep.back_ovf.copy_(ep.recv_ovf)

    ep.route_and_pack = route_and_pack
    ep.local_experts = local_experts
    ep.finish = lambda stream=None: ep.b["y"]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world)
    try:
        ep = CapAndSpillEP(_shape(), world, device="cpu")
        _stub(ep, rank)
        ep.forward(None, None, None, None, None, None)
        dist.barrier()
        ok = (torch.equal(ep.b["y"][:ep.cap_rows], ep.b["x_perm"][:ep.cap_rows])
              and torch.equal(ep.recv_back_ovf, ep.send_ovf))
        meta_ok = all(torch.equal(ep.recv_meta.tensor_split(world)[s],
                                  (torch.arange(ep.send_meta.numel(), dtype=torch.int32) + 1000 * s).tensor_split(world)[rank])
                      for s in range(world))
        np.save(os.path.join(out_dir, "ok_%d.npy" % rank), np.array([ok, meta_ok]))
    finally:
        dist.destroy_process_group()


@pytest.mark.slow
def test_two_pass_forward_round_trips_over_gloo(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(G, port, str(tmp_path)), nprocs=G, join=True, start_method="spawn")
    for r in range(G):
        assert np.load(tmp_path / ("ok_%d.npy" % r)).all(), r


def test_peer_store_forward_order(monkeypatch):
    import torch.distributed as dist
    ep = DirectEP(moe.make_shape(40, 128, 128, 16, 3), G, 1, device="cpu")
    calls = []
    for name in ("route", "plan_and_dispatch", "experts", "experts_and_return", "send_back", "finish"):
        monkeypatch.setattr(ep, name, (lambda n: (lambda *a, **k: calls.append(n)))(name))
    monkeypatch.setattr(dist, "all_gather_into_tensor", lambda out, inp, group=None: calls.append("all_gather"))
    monkeypatch.setattr(dist, "all_reduce", lambda t, group=None: calls.append("barrier"))
    ep._flag, ep._group = torch.zeros(1, dtype=torch.int32), None
    ep.forward(None, None, None, None, None, None)
    assert calls == ["route", "all_gather", "plan_and_dispatch", "barrier", "experts_and_return", "barrier", "finish"]
    calls.clear()
    ep.forward(None, None, None, None, None, None, fused_return=False)
    assert calls == ["route", "all_gather", "plan_and_dispatch", "barrier", "experts", "send_back", "barrier",
                     "finish"]


def test_peer_store_fp8_forward_order(monkeypatch):
    """The fp8 layer: the rows are quantized by the dispatch launch itself (no
    separate token quantization), then the fp8 experts with the fused return."""
    import torch.distributed as dist
    ep = DirectEP(moe.make_shape(40, 128, 128, 16, 3), G, 0, device="cpu", fp8=True)
    calls = []
    for name in ("route", "quantize_tokens", "plan_and_dispatch", "experts_fp8_and_return", "finish"):
        monkeypatch.setattr(ep, name, (lambda n: (lambda *a, **k: calls.append(n)))(name))
    monkeypatch.setattr(dist, "all_gather_into_tensor", lambda out, inp, group=None: calls.append("all_gather"))
    monkeypatch.setattr(dist, "all_reduce", lambda t, group=None: calls.append("barrier"))
    ep._flag, ep._group = torch.zeros(1, dtype=torch.int32), None
    ep.forward_fp8(None, None, None, None, None, None, None, None, None)
    assert calls == ["route", "all_gather", "plan_and_dispatch", "barrier", "experts_fp8_and_return", "barrier",
                     "finish"]

