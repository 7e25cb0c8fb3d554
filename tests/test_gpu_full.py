"""Parity at the full sizes of the five workload configs (config 5 at each skew
alpha), through moe_forward as the benchmark runs it.  Everything integer
(routing indices, counts, offsets, permutation, schedule) is
checked in full; the GEMM outputs on sampled rows and the layer output on
sampled tokens, which the oracle computes one by one."""
import numpy as np
import pytest
import torch

import grouped_expert_gemm_router_b200 as moe
import synth
from gpu_util import (LOGIT_TOL, WEIGHT_TOL, DeviceLayer, assert_close_bf16, check_tile_schedule, host, shape_of)

pytestmark = pytest.mark.gpu

FULL = [(1, None), (2, None), (3, None), (4, None), (5, 0.0), (5, 1.0), (5, 2.0)]


def _sample_rows(rng, d, counts, cfg, n=6):
    """Rows to check: the first and last row of the busiest expert, a row of
    the least busy non-empty expert, and random filled rows."""
    filled = np.flatnonzero(d["src_token"] >= 0)
    order = np.argsort(-counts, kind="stable")
    picks = []
    for e in (order[0], order[np.count_nonzero(counts) - 1]):
        rows = np.flatnonzero(d["dest_row_expert"] == e)
        picks += [rows[0], rows[-1]]
    picks += list(rng.choice(filled, size=min(n, len(filled)), replace=False))
    return sorted(set(int(r) for r in picks))


@pytest.mark.parametrize("cid,alpha", FULL, ids=["cfg%d%s" % (c, "" if a is None else "-a%g" % a) for c, a in FULL])
def test_full_config(orc, cid, alpha):
    cfg = synth.CONFIGS[cid] if alpha is None else synth.CONFIGS[cid].with_(alpha=alpha)
    L = synth.make_layer(cfg)
    shape = shape_of(cfg)
    dl = DeviceLayer(L)
    b = dl.bufs(shape)
    # as the benchmark runs it: no x_perm, the SwiGLU GEMM gathers its rows
    moe.moe_forward(shape, b, b["ws"], args=moe.forward_args({**b, "x_perm": None}))
    torch.cuda.synchronize()
    r = host(b, shape)
    assert r["status"] == 0, hex(r["status"])
    rng = np.random.default_rng(cid * 10 + int(alpha or 0))

    toks = np.sort(rng.choice(cfg.T, size=min(cfg.T, 48), replace=False))
    ref_logits = orc.router_logits(L.x[toks], L.w_router, L.bias)
    assert np.all(np.abs(r["logits"][toks] - ref_logits) <= LOGIT_TOL * np.maximum(1.0, np.abs(ref_logits)))

    idx, w, _ = orc.topk_softmax(r["logits"], cfg.k)
    assert np.array_equal(r["topk_idx"], idx)
    assert np.max(np.abs(r["topk_w"] - w)) <= WEIGHT_TOL

    capped = cfg.C > 0
    d = orc.dispatch(idx, cfg.E, C=cfg.C, capped=capped)
    assert np.array_equal(r["expert_counts"], d["counts"])
    assert np.array_equal(r["expert_offsets"], d["offsets"])
    assert np.array_equal(r["dest_row"], d["dest_row"])
    filled = d["src_token"] >= 0
    assert np.array_equal(r["src_token"][filled], d["src_token"][filled])
    check_tile_schedule(r, shape, d["counts"], d["offsets"], d["spill_off"])

    d["dest_row_expert"] = np.full(d["P"], -1)
    d["dest_row_expert"][d["dest_row"]] = idx.reshape(-1)
    rows = _sample_rows(rng, d, d["counts"], cfg)
    h_ref, y_ref = [], []
    for row in rows:
        t, e = d["src_token"][row], d["dest_row_expert"][row]
        hr = orc.swiglu_row(L.x[t], L.w_gate[e], L.w_up[e])
        h_ref.append(hr)
        y_ref.append(orc.down_row(hr, L.w_down[e]))
    assert_close_bf16(r["h"][rows], np.stack(h_ref), "h (sampled rows)")
    assert_close_bf16(r["y"][rows], np.stack(y_ref), "y (sampled rows)")

    tk = np.sort(rng.choice(cfg.T, size=min(cfg.T, 4), replace=False)).astype(np.int32)
    out_ref = orc.token_outputs(tk, L.x, idx, w, L.w_gate, L.w_up, L.w_down)
    assert_close_bf16(r["out"][tk], out_ref, "out (sampled tokens)")
    # combine is bit-exact given the GPU's own y, on every token
    assert np.array_equal(r["out"], orc.combine(r["y"], r["dest_row"], r["topk_w"]))

    if capped:
        # the capacity layout must give the uncapped result exactly, with no drop
        su = moe.make_shape(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k)
        bu = dl.bufs(su)
        moe.moe_forward(su, bu, bu["ws"])
        torch.cuda.synchronize()
        assert np.array_equal(bu["out"].cpu().view(torch.int16).numpy(), b["out"].cpu().view(torch.int16).numpy())
        assert r["total_spill"] == int(d["spill_cnt"].sum()) > 0
