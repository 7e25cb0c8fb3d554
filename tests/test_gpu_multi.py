"""The expert-parallel layers on real process groups, one process per GPU
(NCCL): each rank's out, bit for bit, against the single-GPU layer on its
own tokens.

The two-pass Cap-and-Spill form (its all-to-all passes through NCCL) runs on
one rank as well as on several; the peer-store form (symmetric memory, peer
stores over NVLink, bf16 and fp8) needs at least two GPUs and is skipped
otherwise.  NVLS is off in NCCL, the process group has a short timeout, and
the ranks leave only between layers."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

T_RANK = 64


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, direct):
    os.environ["NCCL_NVLS_ENABLE"] = "0"
    import torch.distributed as dist
    torch.cuda.set_device(rank)
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", rank))
    try:
        import grouped_expert_gemm_router_b200 as moe
        import synth
        from gpu_util import DeviceLayer, bf16_host
        from grouped_expert_gemm_router_b200.ep import CapAndSpillEP
        from grouped_expert_gemm_router_b200.ep_direct import DirectEP

        cfg = synth.LayerConfig("multi", T_RANK * world, 256, 256, 16, 4, C=12, alpha=1.0, seed=61)
        dl = DeviceLayer(synth.make_layer(cfg))  # the whole layer on this rank's GPU
        x = dl.x[rank * T_RANK:(rank + 1) * T_RANK]
        Eg = cfg.E // world
        sl = slice(rank * Eg, (rank + 1) * Eg)

        def single(shape, fp8=None):
            b = dl.bufs(shape)
            b["x"] = x
            if fp8 is None:
                moe.moe_forward(shape, b, b["ws"], args=moe.forward_args(b))
            else:
                b.update(fp8)
                f = moe.alloc_fp8_buffers(shape)
                b.update({k: f[k] for k in ("x_q", "x_scale", "h_q", "h_scale")})
                moe.moe_forward_fp8(shape, b, b["ws"])
            torch.cuda.synchronize()
            assert moe.moe_read_status(b["ws"]) == 0
            return bf16_host(b["out"])

        res = {}
        capped = moe.make_shape(T_RANK, cfg.H, cfg.F, cfg.E, cfg.k, C=cfg.C, capacity=True)
        ep = CapAndSpillEP(capped, world)
        for _ in range(2):  # a second layer reuses every buffer
            out = ep.forward(x, dl.w_router, dl.bias, dl.w_gate[sl], dl.w_up[sl], dl.w_down[sl])
        torch.cuda.synchronize()
        res["two_pass"] = np.array_equal(bf16_host(out), single(capped))
        if direct:
            shape = moe.make_shape(T_RANK, cfg.H, cfg.F, cfg.E, cfg.k)
            ref = single(shape)
            epd = DirectEP.on_process_group(shape)
            for fused in (True, False, True):
                out = epd.forward(x, dl.w_router, dl.bias, dl.w_gate[sl], dl.w_up[sl], dl.w_down[sl],
                                  fused_return=fused)
                torch.cuda.synchronize()
                res["direct_%d_%s" % (len(res), fused)] = np.array_equal(bf16_host(out), ref)
            wq = dl.bufs(shape)
            wq.update(moe.alloc_fp8_buffers(shape))
            moe.quantize_layer_weights_fp8(shape, wq)
            codes = {k: wq[k] for k in ("wg_q", "wg_scale", "wu_q", "wu_scale", "wd_q", "wd_scale")}
            ep8 = DirectEP.on_process_group(shape, fp8=True)
            out = ep8.forward_fp8(x, dl.w_router, dl.bias, *(codes[k][sl] for k in ("wg_q", "wg_scale", "wu_q",
                                                                                    "wu_scale", "wd_q", "wd_scale")))
            torch.cuda.synchronize()
            res["direct_fp8"] = np.array_equal(bf16_host(out), single(shape, codes))
        dist.barrier()
        np.save(os.path.join(out_dir, "ok_%d.npy" % rank), np.array([res[k] for k in sorted(res)]))
        with open(os.path.join(out_dir, "keys_%d.txt" % rank), "w") as f:
            f.write(",".join(sorted(res)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(600)
@pytest.mark.parametrize("world", [1, 2, 4])
def test_expert_parallel_on_nccl_process_groups(tmp_path, world):
    n = torch.cuda.device_count()
    if n < world:
        pytest.skip("needs %d GPUs" % world)
    direct = world >= 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), direct), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        ok = np.load(tmp_path / ("ok_%d.npy" % r))
        keys = (tmp_path / ("keys_%d.txt" % r)).read_text()
        assert ok.all(), "rank %d: %s -> %s" % (r, keys, ok.tolist())
