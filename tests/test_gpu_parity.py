"""CUDA path (through the C ABI) against the CPU oracle, element by element,
on seeded inputs small enough for the whole oracle, spanning several GEMM
tiles per expert with ragged tails, plus the edge cases."""
import numpy as np
import pytest
import torch

import grouped_expert_gemm_router_b200 as moe
import synth
from gpu_util import (LOGIT_TOL, WEIGHT_TOL, DeviceLayer, assert_close_bf16, bf16_host, check_tile_schedule, host,
                      run_steps, shape_of)
from gpu_util import oracle_layer as _oracle_full

pytestmark = pytest.mark.gpu

CASES = {
    # two row tiles per expert (about 350 routed rows each) and ragged tails
    "two_tiles_E4_k2": synth.LayerConfig("t", 700, 256, 384, 4, 2, seed=1),
    # H = 384: the down projection ends on a single 128-feature accumulator
    "skew_E8_k3_H384": synth.LayerConfig("t", 300, 384, 256, 8, 3, alpha=1.5, seed=2),
    "capacity_E16_k4_C24": synth.LayerConfig("t", 200, 256, 256, 16, 4, C=24, alpha=1.0, seed=3),
    "tiny_config": synth.CONFIGS[1],
    "single_token": synth.LayerConfig("t", 1, 128, 128, 1, 1, seed=4),
    "k_equals_E": synth.LayerConfig("t", 40, 128, 128, 4, 4, seed=5),
    "E1_dense": synth.LayerConfig("t", 300, 128, 256, 1, 1, seed=6),
    "many_experts_E256_k8": synth.LayerConfig("t", 96, 128, 128, 256, 8, alpha=0.5, seed=7),
}


@pytest.mark.parametrize("name", list(CASES))
def test_layer_parity(orc, name):
    cfg = CASES[name]
    L = synth.make_layer(cfg)
    shape = shape_of(cfg)
    dl = DeviceLayer(L)
    r = host(run_steps(dl, shape), shape)
    assert r["status"] == 0, hex(r["status"])

    # step 1: logits against the oracle's, then indices/weights given the GPU's logits
    ref_logits = orc.router_logits(L.x, L.w_router, L.bias)
    assert np.all(np.abs(r["logits"] - ref_logits) <= LOGIT_TOL * np.maximum(1.0, np.abs(ref_logits)))
    o = _oracle_full(orc, L, cfg, r["logits"])
    assert np.array_equal(r["topk_idx"], o["idx"])
    assert np.max(np.abs(r["topk_w"] - o["w"])) <= WEIGHT_TOL

    # steps 2-3: bit-exact counts, offsets, permutation, gathered rows, schedule
    d = o["d"]
    assert np.array_equal(r["expert_counts"], d["counts"])
    assert np.array_equal(r["expert_offsets"], d["offsets"])
    assert np.array_equal(r["dest_row"], d["dest_row"])
    filled = d["src_token"] >= 0
    assert np.array_equal(r["src_token"][filled], d["src_token"][filled])
    if cfg.C > 0:
        assert np.all(r["src_token"][~filled] == -1)
        assert np.array_equal(r["cap_cnt"], d["cap_cnt"]) and np.array_equal(r["spill_cnt"], d["spill_cnt"])
        assert np.array_equal(r["spill_off"], d["spill_off"])
        assert r["total_spill"] == int(d["spill_cnt"].sum())
    assert np.array_equal(r["x_perm"][filled], o["x_perm"][filled])
    check_tile_schedule(r, shape, d["counts"], d["offsets"], d["spill_off"])

    # step 4: GEMMs within the output tolerance, on every filled row
    assert_close_bf16(r["h"][filled], o["h"][filled], "h")
    assert_close_bf16(r["y"][filled], o["y"][filled], "y")
    # step 5: combine is bit-exact given the same y; the layer within tolerance
    same_y_out = orc.combine(r["y"], r["dest_row"], r["topk_w"])
    assert np.array_equal(r["out"], same_y_out)
    assert_close_bf16(r["out"], o["out"], "out")


# moe_forward builds the dispatch inside the router for up to 4096 routed
# pairs and with the separate dispatch kernels above that; both must give the
# step-by-step results bit for bit.
FORWARD_CASES = {
    "skew_E8_k3_H384": CASES["skew_E8_k3_H384"],
    "capped_C7": synth.LayerConfig("t", 150, 128, 256, 12, 3, C=7, alpha=1.2, seed=10),
    "pairs_at_fused_limit": synth.LayerConfig("t", 1024, 128, 128, 16, 4, alpha=0.7, seed=31),
    "pairs_above_fused_limit": synth.LayerConfig("t", 1366, 128, 128, 16, 3, alpha=0.7, seed=32),
}
SAME_KEYS = ("logits", "topk_idx", "topk_w", "expert_counts", "expert_offsets", "dest_row", "num_tiles",
             "total_spill", "cap_cnt", "spill_cnt", "spill_off", "order", "grp_tile_start", "tile_map", "row_cap",
             "h", "y", "out", "status")


@pytest.mark.parametrize("with_x_perm", [True, False], ids=["x_perm", "gathered"])
@pytest.mark.parametrize("name", list(FORWARD_CASES))
def test_forward_entry_point_matches_steps(orc, name, with_x_perm):
    """moe_forward against the five entry points called one by one; without
    an x_perm buffer the SwiGLU GEMM gathers its rows from x itself."""
    cfg = FORWARD_CASES[name]
    L = synth.make_layer(cfg)
    shape = shape_of(cfg)
    dl = DeviceLayer(L)
    a = host(run_steps(dl, shape), shape)
    b = dl.bufs(shape)
    b["x_perm"].fill_(0)
    moe.moe_forward(shape, b, b["ws"], args=moe.forward_args(b if with_x_perm else {**b, "x_perm": None}))
    torch.cuda.synchronize()
    f = host(b, shape)
    for key in SAME_KEYS:
        assert np.array_equal(a[key], f[key]), key
    assert a["status"] == 0
    filled = a["src_token"] >= 0
    assert np.array_equal(a["src_token"], f["src_token"]) if cfg.C > 0 else np.array_equal(a["src_token"][filled],
                                                                                           f["src_token"][filled])
    if with_x_perm:
        assert np.array_equal(a["x_perm"][filled], f["x_perm"][filled])
    else:
        assert not f["x_perm"].any(), "x_perm must stay untouched"


@pytest.mark.parametrize("name", list(CASES))
def test_swiglu_gather_equals_permuted_copy(orc, name):
    """The SwiGLU GEMM reading rows x[src_token[r]] with TMA gathers gives
    the h of the GEMM on the permuted copy x_perm, bit for bit, on every
    filled row (several tiles, ragged tails, capacity layout, E = 256)."""
    cfg = CASES[name]
    L = synth.make_layer(cfg)
    shape = shape_of(cfg)
    dl = DeviceLayer(L)
    b = run_steps(dl, shape)
    h2 = torch.zeros_like(b["h"])
    moe.moe_grouped_swiglu_gather(shape, b["x"], b["src_token"], b["w_gate"], b["w_up"], h2, b["ws"])
    torch.cuda.synchronize()
    r = host(b, shape)
    assert r["status"] == 0
    filled = r["src_token"] >= 0
    g = bf16_host(h2)
    assert np.array_equal(g[filled], r["h"][filled])
    assert not g[~filled].any(), "rows no tile covers stay unwritten"


def test_logits_in_ties(orc):
    """Integer-valued logits with many ties, given to the router directly:
    indices must follow the lowest-index tie-break exactly."""
    cfg = synth.LayerConfig("t", 257, 128, 128, 16, 5, seed=8)
    L = synth.make_layer(cfg)
    rng = np.random.default_rng(0)
    logits = rng.integers(-2, 3, size=(cfg.T, cfg.E)).astype(np.float32)
    logits[3, :] = np.nan
    logits[4, 7] = np.nan
    shape = shape_of(cfg, logits_in=True)
    dl = DeviceLayer(L)
    r = host(run_steps(dl, shape, logits=logits), shape)
    idx, w, _ = orc.topk_softmax(logits, cfg.k)
    assert np.array_equal(r["topk_idx"], idx)
    ok = np.isfinite(w).all(axis=1)
    assert np.max(np.abs(r["topk_w"][ok] - w[ok])) <= WEIGHT_TOL
    assert r["status"] & moe.MOE_DEV_NAN_LOGIT


@pytest.mark.parametrize("T,E,k", [(257, 64, 7), (120, 100, 33), (257, 128, 8), (100, 200, 40), (300, 128, 8),
                                   (40, 256, 256)])
def test_logits_in_ties_wide(orc, T, E, k):
    """Ties among each lane's several candidates (E > 32), zeros of both
    signs, NaNs, and k past one warp's width: the step-by-step router and
    moe_forward (which builds the dispatch inside the router for small
    batches) both follow the lowest-index tie-break exactly."""
    cfg = synth.LayerConfig("t", T, 128, 128, E, k, seed=9)
    L = synth.make_layer(cfg)
    rng = np.random.default_rng(E + k)
    logits = rng.integers(-2, 3, size=(T, E)).astype(np.float32)
    logits[(logits == 0) & (rng.random((T, E)) < 0.5)] = -0.0
    logits[1, :] = np.nan
    logits[2, ::3] = np.nan
    shape = shape_of(cfg, logits_in=True)
    dl = DeviceLayer(L)
    idx, w, _ = orc.topk_softmax(logits, k)
    ok = np.isfinite(w).all(axis=1)
    r = host(run_steps(dl, shape, logits=logits), shape)
    b = dl.bufs(shape)
    b["logits"].copy_(torch.from_numpy(logits))
    moe.moe_forward(shape, b, b["ws"], args=moe.forward_args(b))
    torch.cuda.synchronize()
    f = host(b, shape)
    for got in (r, f):
        assert np.array_equal(got["topk_idx"], idx)
        assert np.max(np.abs(got["topk_w"][ok] - w[ok])) <= WEIGHT_TOL
        assert got["status"] & moe.MOE_DEV_NAN_LOGIT
    assert np.array_equal(r["out"], f["out"])


def test_all_tokens_to_one_expert(orc):
    """A dominant bias sends every token to expert 0 (n_0 = T, 3 row tiles)."""
    cfg = synth.LayerConfig("t", 600, 128, 256, 8, 2, seed=9)
    L = synth.make_layer(cfg)
    L.bias = np.zeros(cfg.E, np.float32)
    L.bias[0] = 1000.0
    shape = shape_of(cfg)
    r = host(run_steps(DeviceLayer(L), shape), shape)
    assert r["expert_counts"][0] == cfg.T
    o = _oracle_full(orc, L, cfg, r["logits"])
    assert np.array_equal(r["dest_row"], o["d"]["dest_row"])
    assert_close_bf16(r["out"], o["out"], "out")


@pytest.mark.parametrize("C", [0, 1, 7, 10_000])
def test_capacity_equals_uncapped(orc, C):
    """Capacity layout (C = 0: everything in the overflow; C >= max n_e:
    nothing spills) gives the uncapped output bit for bit, with no drops."""
    cfg = synth.LayerConfig("t", 150, 128, 256, 12, 3, alpha=1.2, seed=10)
    L = synth.make_layer(cfg)
    dl = DeviceLayer(L)
    su = shape_of(cfg)
    sc = moe.make_shape(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k, C=C, capacity=True)
    u = host(run_steps(dl, su), su)
    c = host(run_steps(dl, sc), sc)
    assert u["status"] == 0 and c["status"] == 0
    assert np.array_equal(u["out"], c["out"])
    assert len(set(c["dest_row"].tolist())) == cfg.T * cfg.k
    if C == 0:
        assert np.array_equal(c["dest_row"], u["dest_row"])
    if C >= cfg.T:
        assert c["total_spill"] == 0


def test_cuda_graph_replay_with_new_routing(orc):
    """Capture the whole layer once; replay it on new tokens (new routing):
    no routing-dependent host shape exists, so the replay stays exact."""
    cfg = CASES["skew_E8_k3_H384"]
    L = synth.make_layer(cfg)
    shape = shape_of(cfg)
    dl = DeviceLayer(L)
    b = dl.bufs(shape)
    args = moe.forward_args(b)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        moe.moe_forward(shape, b, b["ws"], stream=s, args=args)  # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_forward(shape, b, b["ws"], args=args)
    for seed_offset in (11, 12):
        x2 = synth.x_tokens(cfg, seed_offset)
        b["x"].copy_(torch.from_numpy(x2.view(np.int16)).view(torch.bfloat16))
        g.replay()
        torch.cuda.synchronize()
        r = host(b, shape)
        L2 = synth.Layer(cfg, x2, L.w_router, L.bias, L.w_gate, L.w_up, L.w_down)
        o = _oracle_full(orc, L2, cfg, r["logits"])
        assert np.array_equal(r["topk_idx"], o["idx"])
        assert np.array_equal(r["dest_row"], o["d"]["dest_row"])
        assert_close_bf16(r["out"], o["out"], "out after replay")
    del g


def test_scan_wait_expires_and_reports(orc):
    """A histogram block that never publishes makes its successor's bounded
    wait run out: the kernel returns, the status word says so, and the
    context stays usable."""
    cfg = synth.LayerConfig("t", 2048, 128, 128, 8, 2, seed=13)  # 4096 pairs = 2 scan blocks
    L = synth.make_layer(cfg)
    dl = DeviceLayer(L)
    shape = shape_of(cfg, flags=moe.MOE_FLAG_TEST_STALL_SCAN)
    b = dl.bufs(shape)
    moe.moe_set_wait_timeout_ns(200_000_000)
    try:
        moe.moe_route(shape, b["x"], b["w_router"], b["bias"], b["logits"], b["topk_idx"], b["topk_w"], b["ws"])
        moe.moe_permute(shape, b["x"], b["topk_idx"], b["expert_counts"], b["expert_offsets"], b["src_token"],
                        b["dest_row"], b["x_perm"], b["ws"])
        st = moe.moe_read_status(b["ws"], clear=True)
    finally:
        moe.moe_set_wait_timeout_ns(1_000_000_000)
    assert st & moe.MOE_DEV_SCAN_TIMEOUT
    ok = shape_of(cfg)
    r = host(run_steps(dl, ok), ok)
    assert r["status"] == 0
    o = _oracle_full(orc, L, cfg, r["logits"])
    assert np.array_equal(r["dest_row"], o["d"]["dest_row"])


@pytest.mark.parametrize("name", ["two_tiles_E4_k2", "skew_E8_k3_H384", "capacity_E16_k4_C24", "tiny_config",
                                  "single_token", "k_equals_E", "E1_dense", "many_experts_E256_k8"])
def test_down_with_fused_combine(orc, name):
    """The combine of step 5 inside the down GEMM's epilogue: the same y, and
    out bit-identical to the separate combine kernel's, on two calls in a row
    (the arrival counts must return to zero after each call)."""
    cfg = CASES[name]
    L = synth.make_layer(cfg)
    dl = DeviceLayer(L)
    shape = shape_of(cfg)
    b = run_steps(dl, shape)  # route, permute, swiglu, down, combine
    y_ref = bf16_host(b["y"])
    out_ref = bf16_host(b["out"])
    for _ in range(2):
        b["y"].fill_(0)
        b["out"].fill_(0)
        moe.moe_grouped_down_combine(shape, b["h"], b["w_down"], b["src_token"], b["dest_row"], b["topk_w"], b["y"],
                                     b["out"], b["ws"])
        torch.cuda.synchronize()
        assert moe.moe_read_status(b["ws"], clear=True) == 0
        filled = b["src_token"].cpu().numpy() >= 0
        assert np.array_equal(bf16_host(b["y"])[filled], y_ref[filled])
        assert np.array_equal(bf16_host(b["out"]), out_ref)
    # and the whole layer with the flag, against the oracle
    sf = shape_of(cfg, flags=moe.MOE_FLAG_FUSED_COMBINE)
    bf = dl.bufs(sf)
    moe.moe_forward(sf, bf, bf["ws"])
    torch.cuda.synchronize()
    r = host(bf, sf)
    assert r["status"] == 0
    o = _oracle_full(orc, L, cfg, r["logits"])
    assert np.array_equal(r["out"], orc.combine(r["y"], r["dest_row"], r["topk_w"]))
    assert_close_bf16(r["out"], o["out"], "out (fused combine)")


def test_gemm_wait_expires_and_reports(orc):
    """The SwiGLU GEMM's token producer in CTA 0 never loads its first stage:
    the MMA issuer's bounded wait runs out, the kernel records the timeout,
    lets the copies it issued land, frees its tensor memory and returns; the
    context stays usable and a clean layer in it matches the oracle."""
    cfg = CASES["two_tiles_E4_k2"]
    L = synth.make_layer(cfg)
    dl = DeviceLayer(L)
    shape = shape_of(cfg, flags=moe.MOE_FLAG_TEST_STALL_GEMM)
    b = dl.bufs(shape)
    moe.moe_set_wait_timeout_ns(50_000_000)
    try:
        moe.moe_route(shape, b["x"], b["w_router"], b["bias"], b["logits"], b["topk_idx"], b["topk_w"], b["ws"])
        moe.moe_permute(shape, b["x"], b["topk_idx"], b["expert_counts"], b["expert_offsets"], b["src_token"],
                        b["dest_row"], b["x_perm"], b["ws"])
        assert moe.moe_read_status(b["ws"], clear=True) == 0
        moe.moe_grouped_swiglu(shape, b["x_perm"], b["w_gate"], b["w_up"], b["h"], b["ws"])
        st = moe.moe_read_status(b["ws"], clear=True)
    finally:
        moe.moe_set_wait_timeout_ns(1_000_000_000)
    assert st == moe.MOE_DEV_GEMM_TIMEOUT, hex(st)
    ok = shape_of(cfg)
    r = host(run_steps(dl, ok), ok)
    assert r["status"] == 0
    o = _oracle_full(orc, L, cfg, r["logits"])
    filled = o["d"]["src_token"] >= 0
    assert_close_bf16(r["h"][filled], o["h"][filled], "h after a GEMM timeout")
    assert_close_bf16(r["out"], o["out"], "out after a GEMM timeout")




def test_forward_graph_replays_with_new_inputs(orc):
    """moe.ForwardGraph: moe_forward captured once; replays on new tokens
    written into the same buffers give the eager moe_forward's results bit
    for bit (the launch grid depends only on the shape)."""
    cfg = FORWARD_CASES["capped_C7"]
    L = synth.make_layer(cfg.with_(T=cfg.T * 3))
    shape = shape_of(cfg)
    dl = DeviceLayer(L)
    b = dl.bufs(shape)
    b["x"] = dl.x[:cfg.T].clone()
    g = moe.ForwardGraph(shape, b, b["ws"])
    ref = dl.bufs(shape)
    for part in (1, 2):
        xs = dl.x[part * cfg.T:(part + 1) * cfg.T]
        b["x"].copy_(xs)
        g.replay()
        ref["x"] = xs
        moe.moe_forward(shape, ref, ref["ws"], args=moe.forward_args(ref))
        torch.cuda.synchronize()
        assert np.array_equal(bf16_host(b["out"]), bf16_host(ref["out"])), part
        assert torch.equal(b["topk_idx"], ref["topk_idx"])
    assert moe.moe_read_status(b["ws"]) == 0
