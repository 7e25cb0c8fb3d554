"""Parity at the full sizes of the five workload configs (config 5 at each skew
alpha), through moe_forward in both of its forms: with an x_perm buffer (the
row copy, then the tiled SwiGLU GEMM: what the benchmark runs when a batch
has more than 32 routed rows per expert) and without one (the SwiGLU GEMM
gathers its rows from x); and with the combine fused into the down GEMM,
whose output must equal the separate combine's bit for bit.

Everything integer (routing indices, counts, offsets, permutation, schedule)
is checked in full.  The GEMM outputs are checked on rows the oracle computes
one by one, chosen from the device's own tile map: one filled row of every
tile (so every expert, row tile and, since a whole row is compared, every
feature block the persistent schedule ran), plus the first and last row of
every expert.  The layer output is checked on at least 64 tokens, among them
every token routed to the busiest expert's last row tile.  The oracle is the
only reference; its single-threaded calls run side by side in threads (the
C calls release the interpreter lock)."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import grouped_expert_gemm_router_b200 as moe
import synth
from gpu_util import (LOGIT_TOL, WEIGHT_TOL, DeviceLayer, assert_close_bf16, check_tile_schedule, host, shape_of)

pytestmark = pytest.mark.gpu

FULL = [(1, None), (2, None), (3, None), (4, None), (5, 0.0), (5, 1.0), (5, 2.0)]
THREADS = max(1, min(32, os.cpu_count() or 1))


def _tile_rows(tile_map, rng):
    """One filled row of every tile (random within the tile) and, per tile,
    its expert."""
    rows, experts = [], []
    for e, s0, lens, s1 in tile_map:
        l0, l1 = lens & 0xFFFF, (lens >> 16) & 0xFFFF
        c = int(rng.integers(l0 + l1))
        rows.append(int(s0 + c) if c < l0 else int(s1 + c - l0))
        experts.append(int(e))
    return rows, experts


def _expert_rows(d, idx, E):
    """Permuted rows of each expert in stable order (their pairs' flat order)."""
    flat_e = idx.reshape(-1)
    out = []
    for e in range(E):
        out.append(d["dest_row"][np.flatnonzero(flat_e == e)])
    return out


def _busiest_last_tile_tokens(r, d, counts):
    """Tokens of the rows of the busiest expert's last tile in the schedule."""
    g = 0  # the schedule's expert groups run in descending-count order
    e = int(r["order"][g])
    assert counts[e] == counts.max()
    last = r["grp_tile_start"][g + 1] - 1
    te, s0, lens, s1 = (int(v) for v in r["tile_map"][last])
    assert te == e
    l0, l1 = lens & 0xFFFF, (lens >> 16) & 0xFFFF
    rows = list(range(s0, s0 + l0)) + list(range(s1, s1 + l1))
    return np.unique(d["src_token"][rows])


def _oracle_rows(orc, L, pool, rows, row_token, row_expert):
    def one(row):
        t, e = int(row_token[row]), int(row_expert[row])
        hr = orc.swiglu_row(L.x[t], L.w_gate[e], L.w_up[e])
        return hr, orc.down_row(hr, L.w_down[e])

    res = list(pool.map(one, rows))
    return np.stack([a for a, _ in res]), np.stack([b for _, b in res])


def _oracle_tokens(orc, L, pool, toks, idx, w):
    chunks = [toks[i::THREADS] for i in range(THREADS) if len(toks[i::THREADS])]
    res = list(pool.map(lambda c: orc.token_outputs(c, L.x, idx, w, L.w_gate, L.w_up, L.w_down), chunks))
    out = np.empty((len(toks), L.x.shape[1]), np.uint16)
    for i, r in enumerate(res):
        out[i::THREADS][:len(r)] = r
    return out


@pytest.mark.parametrize("cid,alpha", FULL, ids=["cfg%d%s" % (c, "" if a is None else "-a%g" % a) for c, a in FULL])
def test_full_config(orc, cid, alpha):
    cfg = synth.CONFIGS[cid] if alpha is None else synth.CONFIGS[cid].with_(alpha=alpha)
    L = synth.make_layer(cfg)
    shape = shape_of(cfg)
    dl = DeviceLayer(L)
    runs = {}
    fused = shape_of(cfg, flags=moe.MOE_FLAG_FUSED_COMBINE)
    for form in ("tiled", "gather", "fused_combine"):
        b = dl.bufs(shape)
        if form == "tiled":
            moe.moe_forward(shape, b, b["ws"])  # row copy into x_perm, tiled SwiGLU GEMM
        elif form == "gather":
            moe.moe_forward(shape, b, b["ws"], args=moe.forward_args({**b, "x_perm": None}))
        else:  # the combine inside the down GEMM's epilogue
            moe.moe_forward(fused, b, b["ws"])
        torch.cuda.synchronize()
        r = host(b, shape)
        assert r["status"] == 0, "%s: device status %#x" % (form, r["status"])
        runs[form] = (b, r)
    b, r = runs["tiled"]
    rg = runs["gather"][1]
    # the fused combine: out bit-identical to the separate combine's
    assert np.array_equal(runs.pop("fused_combine")[1]["out"], r["out"])
    rng = np.random.default_rng(cid * 10 + int(alpha or 0))

    # routing and dispatch: in full, and identical in both forms
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
    for key in ("logits", "topk_idx", "topk_w", "expert_counts", "expert_offsets", "dest_row", "num_tiles"):
        assert np.array_equal(np.asarray(rg[key]), np.asarray(r[key])), "gather form differs in " + key
    assert np.array_equal(rg["tile_map"], r["tile_map"])
    # the tiled form's row copy, on every filled row
    frows = np.flatnonzero(filled)
    assert np.array_equal(r["x_perm"][frows], L.x[d["src_token"][frows]])

    # GEMM outputs: one row of every tile, first and last row of every expert
    row_expert = np.full(d["P"], -1, np.int64)
    row_expert[d["dest_row"]] = idx.reshape(-1)
    rows, texp = _tile_rows(r["tile_map"], rng)
    assert all(row_expert[rw] == e for rw, e in zip(rows, texp)), "a tile row outside its expert"
    for er in _expert_rows(d, idx, cfg.E):
        if len(er):
            rows += [int(er[0]), int(er[-1])]
    rows = sorted(set(rows))
    # the layer output: every token of the busiest expert's last row tile, and
    # random tokens up to 64 (all of them for a small batch)
    need = _busiest_last_tile_tokens(r, d, d["counts"])
    rest = np.setdiff1d(np.arange(cfg.T), need)
    extra = rng.choice(rest, size=min(len(rest), max(0, 64 - len(need))), replace=False)
    tk = np.sort(np.concatenate([need, extra])).astype(np.int32)
    assert len(tk) >= min(64, cfg.T)

    with ThreadPoolExecutor(THREADS) as pool:
        h_ref, y_ref = _oracle_rows(orc, L, pool, rows, d["src_token"], row_expert)
        out_ref = _oracle_tokens(orc, L, pool, tk, idx, w)
    for form, (_, rr) in runs.items():
        assert_close_bf16(rr["h"][rows], h_ref, "%s: h (one row per tile, %d rows)" % (form, len(rows)))
        assert_close_bf16(rr["y"][rows], y_ref, "%s: y (one row per tile, %d rows)" % (form, len(rows)))
        assert_close_bf16(rr["out"][tk], out_ref, "%s: out (%d tokens)" % (form, len(tk)))
        # the combine is bit-exact given the GPU's own y, on every token
        assert np.array_equal(rr["out"], orc.combine(rr["y"], rr["dest_row"], rr["topk_w"])), form

    if capped:
        # the capacity layout must give the uncapped result exactly, with no drop
        su = moe.make_shape(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k)
        bu = dl.bufs(su)
        moe.moe_forward(su, bu, bu["ws"])
        torch.cuda.synchronize()
        assert np.array_equal(bu["out"].cpu().view(torch.int16).numpy(), b["out"].cpu().view(torch.int16).numpy())
        assert r["total_spill"] == int(d["spill_cnt"].sum()) > 0
