"""Randomised shapes through moe_forward, against the oracle: seeded draws of
T, H, F, E, k, the capacity C and the routing skew, each run with an x_perm
buffer (row copy + tiled SwiGLU) and without one (the SwiGLU GEMM gathers its
rows).  Routing indices, counts, offsets and the permutation are compared bit
for bit (the oracle's top-k on the GPU's fp32 logits), the output within the
output tolerance; both forms must agree bit for bit.  Random expert-parallel
layers (the two-pass form for capped shapes, the peer-store form otherwise,
G ranks emulated on the GPU) must give each rank's moe_forward bit for bit."""
import numpy as np
import pytest
import torch

import grouped_expert_gemm_router_b200 as moe
import synth
from gpu_util import (WEIGHT_TOL, DeviceLayer, assert_close_bf16, bf16_host, oracle_layer, run_cap_and_spill_ep,
                      run_direct_ep, shape_of)

pytestmark = pytest.mark.gpu


def _draw(i):
    rng = np.random.default_rng(1000 + i)
    E = int(rng.choice([1, 2, 3, 5, 8, 12, 16, 31, 64]))
    k = int(rng.integers(1, min(E, 8) + 1))
    T = int(rng.integers(1, 600))
    H = int(rng.choice([128, 256, 384]))
    F = int(rng.choice([128, 256, 512]))
    C = int(rng.choice([0, 0, int(rng.integers(0, max(1, T * k // E) + 4))]))
    alpha = float(rng.choice([0.0, 0.5, 1.5, 3.0]))
    return synth.LayerConfig("rand%d" % i, T, H, F, E, k, C=C, alpha=alpha, seed=2000 + i)


CASES = [_draw(i) for i in range(48)]


def _forward(dl, shape, gathered):
    b = dl.bufs(shape)
    moe.moe_forward(shape, b, b["ws"], args=moe.forward_args({**b, "x_perm": None} if gathered else b))
    torch.cuda.synchronize()
    return b


@pytest.mark.parametrize("cfg", CASES, ids=["%s-T%d-H%d-F%d-E%d-k%d-C%d" % (c.name, c.T, c.H, c.F, c.E, c.k, c.C)
                                            for c in CASES])
def test_random_shape_matches_oracle(orc, cfg):
    L = synth.make_layer(cfg)
    shape = shape_of(cfg)
    dl = DeviceLayer(L)
    b = _forward(dl, shape, gathered=False)
    g = _forward(dl, shape, gathered=True)
    assert moe.moe_read_status(b["ws"]) == 0 and moe.moe_read_status(g["ws"]) == 0
    logits = b["logits"].cpu().numpy()
    o = oracle_layer(orc, L, cfg, logits)
    assert np.array_equal(b["topk_idx"].cpu().numpy(), o["idx"])
    assert np.max(np.abs(b["topk_w"].cpu().numpy() - o["w"])) <= WEIGHT_TOL
    d = o["d"]
    assert np.array_equal(b["expert_counts"].cpu().numpy(), d["counts"])
    assert np.array_equal(b["expert_offsets"].cpu().numpy(), d["offsets"])
    assert np.array_equal(b["dest_row"].cpu().numpy(), d["dest_row"])
    assert_close_bf16(bf16_host(b["out"]), o["out"], "out")
    assert np.array_equal(bf16_host(b["out"]), bf16_host(g["out"])), "gathered form differs"


def _draw_ep(i):
    rng = np.random.default_rng(5000 + i)
    cfg = _draw(100 + i)
    divisors = [g for g in (2, 3, 4, 8) if cfg.E % g == 0]
    if not divisors:
        cfg = cfg.with_(E=8, k=min(cfg.k, 8))
        divisors = [2, 4, 8]
    return cfg, int(rng.choice(divisors))


EP_CASES = [_draw_ep(i) for i in range(16)]


@pytest.mark.parametrize("cfg,G", EP_CASES, ids=["%s-T%d-E%d-k%d-C%d-G%d" % (c.name, c.T, c.E, c.k, c.C, g)
                                                 for c, g in EP_CASES])
def test_random_expert_parallel_matches_single_gpu(cfg, G):
    L = synth.make_layer(cfg.with_(T=cfg.T * G))
    dl = DeviceLayer(L)
    if cfg.C > 0:
        shape = moe.make_shape(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k, C=cfg.C, capacity=True)
        ranks, xs = run_cap_and_spill_ep(dl, shape, G, fused_finish=bool(cfg.seed % 2),
                                              fused_pack=bool(cfg.T % 2))
    else:
        shape = moe.make_shape(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k)
        ranks, xs = run_direct_ep(dl, shape, G, fused_return=bool(cfg.seed % 2), fused_plan=bool(cfg.T % 2))
    for r, ep in enumerate(ranks):
        assert moe.moe_read_status(ep.ws) == 0 and moe.moe_read_status(ep.ws_loc) == 0
        b = dl.bufs(shape)
        b["x"] = xs[r]
        moe.moe_forward(shape, b, b["ws"], args=moe.forward_args(b))
        torch.cuda.synchronize()
        assert np.array_equal(bf16_host(ep.b["out"]), bf16_host(b["out"])), "rank %d" % r

