"""Expert-parallel Cap-and-Spill layer (two equal-split all-to-all passes)
with G ranks held by one process on one GPU: each rank's phases run on its
own buffers and the all-to-alls are carried out as buffer copies
(exchange_in_process, checked against torch.distributed's all_to_all_single
on gloo ranks in test_ep_exchange.py).  Nothing waits on another rank, so
emulating several ranks on one GPU is safe.

Each rank's output must equal, bit for bit, the single-GPU moe_forward of its
own tokens (same routing, same capacity layout, the same rows through the same
GEMM arithmetic), and match the oracle within the output tolerance.  The rows
each rank receives are checked bit-exactly against the tokens the routing
sends it, in the local order (expert, then source rank, capacity rows before
overflow rows)."""
import types

import numpy as np
import pytest
import torch

import grouped_expert_gemm_router_b200 as moe
import synth
from gpu_util import DeviceLayer, assert_close_bf16, bf16_host, oracle_layer, run_cap_and_spill_ep
from grouped_expert_gemm_router_b200.ep import CapAndSpillEP

pytestmark = pytest.mark.gpu

CASES = {
    # decode-like: 64 experts, C = 16, skewed, heavy overflow
    "decode_E64_k6_C16": (synth.LayerConfig("ep", 128, 256, 256, 64, 6, C=16, alpha=1.2, seed=41), (1, 2, 4, 8)),
    "E16_k4_C24_F384": (synth.LayerConfig("ep", 200, 256, 384, 16, 4, C=24, alpha=1.0, seed=42), (2, 4)),
    # C = 0: every pair goes through the overflow pass
    "C0_all_overflow": (synth.LayerConfig("ep", 96, 128, 256, 8, 2, C=0, alpha=0.5, seed=43), (2,)),
    # C >= T: no overflow, zero-row overflow slots
    "C_ge_T_no_overflow": (synth.LayerConfig("ep", 64, 128, 128, 8, 2, C=64, seed=44), (2, 8)),
    # local experts of several row tiles with ragged tails
    "several_tiles_E4_k2": (synth.LayerConfig("ep", 700, 256, 256, 4, 2, C=200, alpha=0.3, seed=45), (2,)),
    # the most experts a layer may have: 256, 128 or 32 per rank
    "E256_k8_C2": (synth.LayerConfig("ep", 48, 128, 128, 256, 8, C=2, alpha=0.8, seed=46), (1, 2, 8)),
}


def _cases():
    return [(name, G) for name, (_, gs) in CASES.items() for G in gs]


def _shape(cfg):
    return moe.make_shape(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k, C=cfg.C, capacity=True)


def _single_gpu(dl, shape, x):
    b = dl.bufs(shape)
    b["x"] = x
    moe.moe_forward(shape, b, b["ws"], args=moe.forward_args(b))
    torch.cuda.synchronize()
    assert moe.moe_read_status(b["ws"]) == 0
    return b


def _check_received_rows(ranks, xs, G, E, H):
    """x_loc of rank d: for each local expert, every source's tokens routed
    to it in token order (the capacity rows are the first C of them)."""
    Eg = E // G
    idx = [ep.b["topk_idx"].cpu().numpy() for ep in ranks]
    xh = [bf16_host(x) for x in xs]
    for d, ep in enumerate(ranks):
        lay = moe.moe_workspace_layout(ep.local)
        ws = ep.ws_loc.cpu().numpy()
        counts = ws[lay.cap_cnt:lay.cap_cnt + 4 * Eg].view(np.int32)
        x_loc = bf16_host(ep.x_loc)
        row = 0
        for el in range(Eg):
            e = d * Eg + el
            want = np.concatenate([xh[s][np.nonzero((idx[s] == e).any(axis=1))[0]] for s in range(G)]).reshape(-1, H)
            assert counts[el] == len(want), (d, el)
            assert np.array_equal(x_loc[row:row + len(want)], want), (d, el)
            row += len(want)


@pytest.mark.parametrize("name,G", _cases(), ids=["%s-G%d" % c for c in _cases()])
def test_ep_layer_matches_single_gpu_and_oracle(orc, name, G):
    cfg, _ = CASES[name]
    L = synth.make_layer(cfg.with_(T=cfg.T * G))
    dl = DeviceLayer(L)
    shape = _shape(cfg)
    ranks, xs = run_cap_and_spill_ep(dl, shape, G)
    for ep in ranks:
        assert moe.moe_read_status(ep.ws) == 0
        assert moe.moe_read_status(ep.ws_loc) == 0
    _check_received_rows(ranks, xs, G, cfg.E, cfg.H)
    for r, ep in enumerate(ranks):
        ref = _single_gpu(dl, shape, xs[r])
        assert torch.equal(ep.b["topk_idx"], ref["topk_idx"])
        assert torch.equal(ep.b["dest_row"], ref["dest_row"])
        assert np.array_equal(bf16_host(ep.b["out"]), bf16_host(ref["out"])), "rank %d" % r
        view = types.SimpleNamespace(x=L.x[r * cfg.T:(r + 1) * cfg.T], w_gate=L.w_gate, w_up=L.w_up,
                                     w_down=L.w_down)
        o = oracle_layer(orc, view, cfg, ep.b["logits"].cpu().numpy())
        assert_close_bf16(bf16_host(ep.b["out"]), o["out"], "out rank %d" % r)


# Full size: the DeepSeek-V2-Lite-shaped decode layer (T = 128 per rank,
# H = 2048, F = 1408, E = 64, k = 6, C = 16) on 2 and 8 ranks, bit for bit
# against each rank's single-GPU layer (which the full-size parity tests pin
# to the oracle).
@pytest.mark.parametrize("G", [2, 8])
def test_ep_full_size_decode_matches_single_gpu(G):
    cfg = synth.CONFIGS[4]
    L = synth.make_layer(cfg.with_(T=cfg.T * G))
    dl = DeviceLayer(L)
    shape = _shape(cfg)
    ranks, xs = run_cap_and_spill_ep(dl, shape, G)
    for r, ep in enumerate(ranks):
        assert moe.moe_read_status(ep.ws) == 0 and moe.moe_read_status(ep.ws_loc) == 0
        ref = _single_gpu(dl, shape, xs[r])
        assert np.array_equal(bf16_host(ep.b["out"]), bf16_host(ref["out"])), "rank %d" % r


@pytest.mark.parametrize("name,G", [("decode_E64_k6_C16", 8), ("E16_k4_C24_F384", 4), ("C0_all_overflow", 2)],
                         ids=lambda v: str(v))
def test_ep_unpack_combine_equals_unpack_then_combine(name, G):
    """The combine that reads the overflow results from the return slots
    gives the out of the unpack followed by the combine, bit for bit."""
    cfg, _ = CASES[name]
    L = synth.make_layer(cfg.with_(T=cfg.T * G))
    dl = DeviceLayer(L)
    shape = _shape(cfg)
    ranks, _ = run_cap_and_spill_ep(dl, shape, G, fused_finish=True)
    fused = [ep.b["out"].clone() for ep in ranks]
    assert any(int(ep.send_meta.view(G, 2, -1)[:, 1].sum()) > 0 for ep in ranks), "no overflow rows"
    for r, ep in enumerate(ranks):
        ep.b["out"].zero_()
        ep.finish(fused=False)
        torch.cuda.synchronize()
        assert torch.equal(ep.b["out"], fused[r]), "rank %d" % r


@pytest.mark.parametrize("name,G", [("decode_E64_k6_C16", 8), ("C0_all_overflow", 2), ("C_ge_T_no_overflow", 2)],
                         ids=lambda v: str(v))
def test_ep_gather_pack_equals_gather_then_pack(name, G):
    """The row copy that writes overflow rows straight into the send slots
    leaves the capacity rows, the slots and the counts sent ahead exactly as
    the row copy followed by the pack does."""
    from grouped_expert_gemm_router_b200.ep import CapAndSpillEP
    cfg, _ = CASES[name]
    L = synth.make_layer(cfg.with_(T=cfg.T * G))
    dl = DeviceLayer(L)
    shape = _shape(cfg)
    for r in range(G):
        x = dl.x[r * cfg.T:(r + 1) * cfg.T]
        got, ref = CapAndSpillEP(shape, G), CapAndSpillEP(shape, G)
        for ep, fused in ((got, True), (ref, False)):
            ep.send_ovf.zero_()
            ep.route_and_pack(x, dl.w_router, dl.bias, fused=fused)
        torch.cuda.synchronize()
        assert moe.moe_read_status(got.ws) == 0
        assert torch.equal(got.send_meta, ref.send_meta), r
        assert torch.equal(got.send_ovf, ref.send_ovf), r
        assert torch.equal(got.b["x_perm"][:got.cap_rows], ref.b["x_perm"][:ref.cap_rows]), r


def test_ep_rejects_uncapped_layout():
    cfg = CASES["E16_k4_C24_F384"][0]
    with pytest.raises(moe.MoeError):
        CapAndSpillEP(moe.make_shape(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k), 2)
    with pytest.raises(moe.MoeError):
        CapAndSpillEP(_shape(cfg), 3)  # E % G != 0
