"""Expert-parallel layer with device-initiated peer stores, G ranks held by one
process on one GPU: each rank's peer tables point at the other ranks' own
x_loc and y (connect_in_process) and the counts all-gather is done by copies.
The put kernels store into other ranks' buffers and never wait on another
rank, so running the ranks one after another on one GPU is safe.

Each rank's output must equal, bit for bit, the single-GPU moe_forward of its
own tokens, and match the oracle within the output tolerance; the rows each
rank receives are checked bit-exactly against the routing (per local expert,
every source's tokens in (source, token) order)."""
import types

import numpy as np
import pytest
import torch

import grouped_expert_gemm_router_b200 as moe
import synth
from gpu_util import DeviceLayer, assert_close_bf16, bf16_host, oracle_layer, run_direct_ep, run_direct_ep_fp8
from grouped_expert_gemm_router_b200.ep_direct import DirectEP, connect_in_process, gather_counts_in_process

pytestmark = pytest.mark.gpu

CASES = {
    "decode_E64_k6": (synth.LayerConfig("epd", 128, 256, 256, 64, 6, alpha=1.2, seed=51), (1, 2, 4, 8)),
    "E16_k4_F384": (synth.LayerConfig("epd", 200, 256, 384, 16, 4, alpha=1.0, seed=52), (2, 4)),
    "E8_k2_skew": (synth.LayerConfig("epd", 96, 128, 256, 8, 2, alpha=3.0, seed=53), (2, 8)),
    "k_equals_E": (synth.LayerConfig("epd", 40, 128, 128, 4, 4, seed=54), (2, 4)),
    "several_tiles_E4_k2": (synth.LayerConfig("epd", 700, 256, 256, 4, 2, alpha=0.3, seed=55), (2,)),
    # the most experts a layer may have: 256, 128 or 32 per rank
    "E256_k8": (synth.LayerConfig("epd", 48, 128, 128, 256, 8, alpha=0.8, seed=56), (1, 2, 8)),
}


def _cases():
    return [(name, G) for name, (_, gs) in CASES.items() for G in gs]


def _shape(cfg):
    return moe.make_shape(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k)


def _single_gpu(dl, shape, x):
    b = dl.bufs(shape)
    b["x"] = x
    moe.moe_forward(shape, b, b["ws"], args=moe.forward_args(b))
    torch.cuda.synchronize()
    assert moe.moe_read_status(b["ws"]) == 0
    return b


def _check_received_rows(ranks, xs, G, E, H):
    Eg = E // G
    idx = [ep.b["topk_idx"].cpu().numpy() for ep in ranks]
    xh = [bf16_host(x) for x in xs]
    for d, ep in enumerate(ranks):
        x_loc = bf16_host(ep.x_loc)
        row = 0
        for el in range(Eg):
            e = d * Eg + el
            want = np.concatenate([xh[s][np.nonzero((idx[s] == e).any(axis=1))[0]] for s in range(G)]).reshape(-1, H)
            assert np.array_equal(x_loc[row:row + len(want)], want), (d, el)
            row += len(want)


FUSED = [("decode_E64_k6", 8), ("E16_k4_F384", 4), ("E8_k2_skew", 2), ("several_tiles_E4_k2", 2)]


@pytest.mark.parametrize("fused_return", [False, True], ids=["return_kernel", "fused_return"])
@pytest.mark.parametrize("name,G", _cases(), ids=["%s-G%d" % c for c in _cases()])
def test_direct_ep_matches_single_gpu_and_oracle(orc, name, G, fused_return):
    if fused_return and (name, G) not in FUSED:
        pytest.skip("fused return checked on a subset")
    cfg, _ = CASES[name]
    L = synth.make_layer(cfg.with_(T=cfg.T * G))
    dl = DeviceLayer(L)
    shape = _shape(cfg)
    ranks, xs = run_direct_ep(dl, shape, G, fused_return, fused_plan=fused_return)
    for ep in ranks:
        assert moe.moe_read_status(ep.ws) == 0
        assert moe.moe_read_status(ep.ws_loc) == 0
    _check_received_rows(ranks, xs, G, cfg.E, cfg.H)
    for r, ep in enumerate(ranks):
        ref = _single_gpu(dl, shape, xs[r])
        assert torch.equal(ep.b["topk_idx"], ref["topk_idx"])
        assert np.array_equal(bf16_host(ep.b["out"]), bf16_host(ref["out"])), "rank %d" % r
        view = types.SimpleNamespace(x=L.x[r * cfg.T:(r + 1) * cfg.T], w_gate=L.w_gate, w_up=L.w_up,
                                     w_down=L.w_down)
        o = oracle_layer(orc, view, cfg, ep.b["logits"].cpu().numpy())
        assert_close_bf16(bf16_host(ep.b["out"]), o["out"], "out rank %d" % r)


# Full size: the Mixtral-8x7B-shaped layer (T = 512 per rank, H = 4096,
# F = 14336, E = 8, k = 2) on 2 and 8 ranks, bit for bit against each rank's
# single-GPU layer (which the full-size parity tests pin to the oracle).
@pytest.mark.parametrize("G,fused_return", [(2, False), (8, False), (8, True)])
def test_direct_ep_full_size_mixtral_matches_single_gpu(G, fused_return):
    cfg = synth.CONFIGS[2]
    L = synth.make_layer(cfg.with_(T=cfg.T * G))
    dl = DeviceLayer(L)
    shape = _shape(cfg)
    ranks, xs = run_direct_ep(dl, shape, G, fused_return, fused_plan=fused_return)
    for r, ep in enumerate(ranks):
        assert moe.moe_read_status(ep.ws) == 0 and moe.moe_read_status(ep.ws_loc) == 0
        ref = _single_gpu(dl, shape, xs[r])
        assert np.array_equal(bf16_host(ep.b["out"]), bf16_host(ref["out"])), "rank %d" % r


@pytest.mark.parametrize("fused_plan", [False, True], ids=["plan_then_dispatch", "plan_dispatch"])
def test_direct_ep_clamps_counts_beyond_the_buffers(fused_plan):
    """Gathered counts past what the buffers hold (a source claiming more
    rows than it can send) are clamped the same way on every rank: nothing
    is stored outside a buffer, MOE_DEV_BAD_ROW is raised, and a clean layer
    in the same context still matches the single-GPU one."""
    cfg = CASES["E16_k4_F384"][0]
    G = 2
    L = synth.make_layer(cfg.with_(T=cfg.T * G))
    dl = DeviceLayer(L)
    shape = _shape(cfg)
    ranks = [DirectEP(shape, G, r) for r in range(G)]
    connect_in_process(ranks)
    for r, ep in enumerate(ranks):
        ep.route(dl.x[r * cfg.T:(r + 1) * cfg.T], dl.w_router, dl.bias)
    gather_counts_in_process(ranks)
    for ep in ranks:
        ep.cnt_all[0, 3] = 1 << 24  # more than T pairs for one expert
        ep.cnt_all[1, :] = cfg.T    # more rows than one source can send a rank
    for r, ep in enumerate(ranks):
        if fused_plan:
            ep.plan_and_dispatch(dl.x[r * cfg.T:(r + 1) * cfg.T])
        else:
            ep.plan()
    torch.cuda.synchronize()
    if not fused_plan:
        for r, ep in enumerate(ranks):
            ep.dispatch(dl.x[r * cfg.T:(r + 1) * cfg.T])
    torch.cuda.synchronize()
    assert all(moe.moe_read_status(ep.ws_loc) & moe.MOE_DEV_BAD_ROW for ep in ranks)
    for ep in ranks:
        moe.moe_read_status(ep.ws)  # clear
    ranks2, xs = run_direct_ep(dl, shape, G, fused_plan=fused_plan)
    for r, ep in enumerate(ranks2):
        assert moe.moe_read_status(ep.ws_loc) == 0
        ref = _single_gpu(dl, shape, xs[r])
        assert np.array_equal(bf16_host(ep.b["out"]), bf16_host(ref["out"]))


def test_direct_ep_rejects_unsupported_shapes():
    cfg = CASES["E16_k4_F384"][0]
    with pytest.raises(moe.MoeError):
        DirectEP(moe.make_shape(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k, C=8, capacity=True), 2, 0)
    with pytest.raises(moe.MoeError):
        DirectEP(_shape(cfg), 3, 0)  # E % G != 0
    with pytest.raises(moe.MoeError):
        DirectEP(_shape(cfg), 2, 2)  # rank out of range


@pytest.mark.parametrize("mode", ["quantize", "codes", "separate"])
@pytest.mark.parametrize("name,G", [("decode_E64_k6", 8), ("E16_k4_F384", 4), ("E8_k2_skew", 2),
                                    ("several_tiles_E4_k2", 2)], ids=lambda v: str(v))
def test_direct_ep_fp8_matches_single_gpu_fp8(name, G, mode):
    """e4m3 rows on the links: each rank's out equals moe_forward_fp8 on its
    tokens bit for bit (per-row token codes and scales are the same whichever
    rank quantizes them; the same fp8 GEMM arithmetic on the same rows)."""
    cfg, _ = CASES[name]
    L = synth.make_layer(cfg.with_(T=cfg.T * G))
    dl = DeviceLayer(L)
    shape = _shape(cfg)
    wq = dl.bufs(shape)
    wq.update(moe.alloc_fp8_buffers(shape))
    moe.quantize_layer_weights_fp8(shape, wq)
    ranks, xs = run_direct_ep_fp8(dl, shape, G, wq, mode)
    for r, ep in enumerate(ranks):
        assert moe.moe_read_status(ep.ws) == 0 and moe.moe_read_status(ep.ws_loc) == 0
        b = dl.bufs(shape)
        b["x"] = xs[r]
        b.update({k: wq[k] for k in ("wg_q", "wg_scale", "wu_q", "wu_scale", "wd_q", "wd_scale")})
        f = moe.alloc_fp8_buffers(shape)
        b.update({k: f[k] for k in ("x_q", "x_scale", "h_q", "h_scale")})
        moe.moe_forward_fp8(shape, b, b["ws"])
        torch.cuda.synchronize()
        assert moe.moe_read_status(b["ws"]) == 0
        assert np.array_equal(bf16_host(ep.b["out"]), bf16_host(b["out"])), "rank %d" % r


@pytest.mark.parametrize("name,G", [("decode_E64_k6", 8), ("E8_k2_skew", 2)], ids=lambda v: str(v))
def test_direct_ep_quantizing_dispatch_stores_the_row_quantizer_codes(name, G):
    """The dispatch that quantizes the rows it sends leaves in every owner's
    x_loc_q and scale_loc exactly the codes and scales of the rows
    moe_quantize_rows_fp8 makes before a plain dispatch of codes."""
    cfg, _ = CASES[name]
    L = synth.make_layer(cfg.with_(T=cfg.T * G))
    dl = DeviceLayer(L)
    shape = _shape(cfg)
    wq = dl.bufs(shape)
    wq.update(moe.alloc_fp8_buffers(shape))
    moe.quantize_layer_weights_fp8(shape, wq)
    got, _ = run_direct_ep_fp8(dl, shape, G, wq, "quantize")
    ref, _ = run_direct_ep_fp8(dl, shape, G, wq, "codes")
    Eg = cfg.E // G
    for r in range(G):
        n = int(ref[r].cnt_all[:, r * Eg:(r + 1) * Eg].sum())
        assert n == int(got[r].cnt_all[:, r * Eg:(r + 1) * Eg].sum()) and n > 0
        assert torch.equal(got[r].x_loc_q[:n], ref[r].x_loc_q[:n]), "rank %d codes" % r
        assert torch.equal(got[r].scale_loc[:n], ref[r].scale_loc[:n]), "rank %d scales" % r


def test_direct_ep_fp8_full_size_decode():
    """The DeepSeek-V2-Lite-shaped layer (uncapped) on 8 ranks in fp8, bit
    for bit against each rank's moe_forward_fp8."""
    cfg = synth.CONFIGS[4].with_(C=0)
    G = 8
    L = synth.make_layer(cfg.with_(T=cfg.T * G))
    dl = DeviceLayer(L)
    shape = _shape(cfg)
    wq = dl.bufs(shape)
    wq.update(moe.alloc_fp8_buffers(shape))
    moe.quantize_layer_weights_fp8(shape, wq)
    ranks, xs = run_direct_ep_fp8(dl, shape, G, wq)
    for r, ep in enumerate(ranks):
        b = dl.bufs(shape)
        b["x"] = xs[r]
        b.update({k: wq[k] for k in ("wg_q", "wg_scale", "wu_q", "wu_scale", "wd_q", "wd_scale")})
        f = moe.alloc_fp8_buffers(shape)
        b.update({k: f[k] for k in ("x_q", "x_scale", "h_q", "h_scale")})
        moe.moe_forward_fp8(shape, b, b["ws"])
        torch.cuda.synchronize()
        assert np.array_equal(bf16_host(ep.b["out"]), bf16_host(b["out"])), "rank %d" % r

