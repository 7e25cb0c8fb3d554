"""Helpers of the GPU parity tests: move seeded layers to the device, run the
C-ABI path step by step, read results back, and check a result against the
oracle's with the tolerances of the spec definition.

Tolerances (written here once, used by every GPU test):
  logits          |gpu - oracle| <= 1e-5 * max(1, |oracle|)
  indices, counts, offsets, permutation, tile schedule: bit-exact
  gate weights    |gpu - oracle| <= 1e-6 (oracle top-k run on the GPU logits)
  bf16 tensors    max|gpu - ref| <= 2e-2 * max|ref| over the compared set
"""
from __future__ import annotations

import numpy as np
import torch

import grouped_expert_gemm_router_b200 as moe
import synth

REL_TOL = 2e-2
LOGIT_TOL = 1e-5
WEIGHT_TOL = 1e-6


def bf16_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f32(a_bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(a_bits)


def shape_of(cfg, logits_in=False, flags=0):
    return moe.make_shape(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k, C=cfg.C, capacity=cfg.C > 0 or bool(flags & 1),
                          logits_in=logits_in, flags=flags & ~1)


class DeviceLayer:
    def __init__(self, L: synth.Layer, device="cuda"):
        self.L = L
        self.x = bf16_dev(L.x, device)
        self.w_router = torch.from_numpy(L.w_router).to(device)
        self.bias = None if L.bias is None else torch.from_numpy(L.bias).to(device)
        self.w_gate = bf16_dev(L.w_gate, device)
        self.w_up = bf16_dev(L.w_up, device)
        self.w_down = bf16_dev(L.w_down, device)

    def bufs(self, shape):
        b = moe.alloc_buffers(shape)
        b.update(x=self.x, w_router=self.w_router, bias=self.bias, w_gate=self.w_gate, w_up=self.w_up,
                 w_down=self.w_down)
        return b


def run_steps(dl: DeviceLayer, shape, b=None, logits=None):
    """Run the five entry points one by one; returns the buffer dict."""
    if b is None:
        b = dl.bufs(shape)
    if logits is not None:
        b["logits"].copy_(torch.from_numpy(logits))
    moe.moe_route(shape, b["x"], b["w_router"], b["bias"], b["logits"], b["topk_idx"], b["topk_w"], b["ws"])
    moe.moe_permute(shape, b["x"], b["topk_idx"], b["expert_counts"], b["expert_offsets"], b["src_token"],
                    b["dest_row"], b["x_perm"], b["ws"])
    moe.moe_grouped_swiglu(shape, b["x_perm"], b["w_gate"], b["w_up"], b["h"], b["ws"])
    moe.moe_grouped_down(shape, b["h"], b["w_down"], b["y"], b["ws"])
    moe.moe_combine(shape, b["y"], b["dest_row"], b["topk_w"], b["out"])
    torch.cuda.synchronize()
    return b


def host(b, shape):
    """Copy every buffer (and the inspectable workspace sections) to numpy."""
    r = {}
    for k in ("logits", "topk_w"):
        r[k] = b[k].cpu().numpy()
    for k in ("topk_idx", "expert_counts", "expert_offsets", "src_token", "dest_row"):
        r[k] = b[k].cpu().numpy()
    for k in ("x_perm", "h", "y", "out"):
        r[k] = bf16_host(b[k])
    L = moe.moe_workspace_layout(shape)
    ws = b["ws"].cpu().numpy()
    E = shape.E

    def i32(off, n):
        return ws[off:off + 4 * n].view(np.int32).copy()

    r["num_tiles"] = int(i32(L.num_tiles, 1)[0])
    r["total_spill"] = int(i32(L.total_spill, 1)[0])
    r["cap_cnt"] = i32(L.cap_cnt, E)
    r["spill_cnt"] = i32(L.spill_cnt, E)
    r["spill_off"] = i32(L.spill_off, E + 1)
    r["order"] = i32(L.order, E)
    r["grp_tile_start"] = i32(L.grp_tile_start, E + 1)
    r["tile_map"] = i32(L.tile_map, 4 * L.max_tiles).reshape(-1, 4)[:max(r["num_tiles"], 0)]
    r["max_tiles"] = L.max_tiles
    r["row_cap"] = int(i32(L.row_cap, 1)[0])
    r["status"] = moe.moe_read_status(b["ws"], clear=True)
    return r


def assert_close_bf16(gpu_bits, ref_bits, what):
    g = f32(gpu_bits).astype(np.float64)
    ref = f32(ref_bits).astype(np.float64)
    assert np.all(np.isfinite(g)), "%s: non-finite GPU values" % what
    scale = np.max(np.abs(ref))
    err = np.max(np.abs(g - ref)) if g.size else 0.0
    assert err <= REL_TOL * scale, "%s: max|gpu-ref| = %g > %g * %g" % (what, err, REL_TOL, scale)
    return err / scale if scale > 0 else 0.0


def expert_of_rows(n_counts, offsets, E, C, capped, spill_off, P):
    """Expert owning each permuted row (-1 for rows no expert owns)."""
    own = np.full(P, -1, np.int64)
    for e in range(E):
        n = int(n_counts[e])
        if not capped:
            own[offsets[e]:offsets[e] + n] = e
        else:
            cap = min(n, C)
            own[e * C:e * C + cap] = e
            own[E * C + spill_off[e]:E * C + spill_off[e] + (n - cap)] = e
    return own


def check_tile_schedule(r, shape, counts, offsets, spill_off):
    """The tile map is one of many valid schedules: check it is valid, and
    that the parts fixed by its definition (order, tile count per expert) are
    exactly as defined."""
    E, C = shape.E, shape.C
    capped = bool(shape.flags & moe.MOE_FLAG_CAPACITY)
    order = sorted(range(E), key=lambda e: (-int(counts[e]), e))
    assert r["order"].tolist() == order
    nt = r["num_tiles"]
    assert 0 <= nt <= r["max_tiles"]
    P = moe.moe_permuted_rows(shape)
    own = expert_of_rows(counts, offsets, E, C, capped, spill_off, P)
    covered = np.zeros(P, np.int64)
    gts = r["grp_tile_start"]
    assert gts[0] == 0 and gts[E] == nt and np.all(np.diff(gts) >= 0)
    for g, e in enumerate(order):
        for ti in range(gts[g], gts[g + 1]):
            te, s0, lens, s1 = (int(v) for v in r["tile_map"][ti])
            l0, l1 = lens & 0xFFFF, (lens >> 16) & 0xFFFF
            assert te == e
            assert l0 >= 1
            assert (l0 + 15) // 16 * 16 + (l1 + 15) // 16 * 16 <= r["row_cap"] <= 256
            for s, l in ((s0, l0), (s1, l1)):
                if l:
                    assert np.all(own[s:s + l] == e), "tile rows outside expert %d" % e
                    covered[s:s + l] += 1
        if counts[e] == 0:
            assert gts[g + 1] == gts[g]
    assert np.array_equal(covered, (own >= 0).astype(np.int64)), "every filled row in exactly one tile"
    # the row cap is the largest padded per-expert row count, capped at 256
    req = []
    for e in range(E):
        n = int(counts[e])
        cap = min(n, C) if capped else n
        req.append(min(256, (cap + 15) // 16 * 16 + (n - cap + 15) // 16 * 16))
    assert r["row_cap"] == max(16, max(req))
    if r["row_cap"] < 256:
        assert all(gts[g + 1] - gts[g] == (1 if counts[e] else 0) for g, e in enumerate(order))


def oracle_layer(orc, L, cfg, logits_gpu):
    """Oracle routing from the GPU logits (same fp32 logits on both sides),
    then the oracle's own dispatch, experts and combine."""
    idx, w, _ = orc.topk_softmax(logits_gpu, cfg.k)
    capped = cfg.C > 0
    d = orc.dispatch(idx, cfg.E, C=cfg.C, capped=capped)
    P = d["P"]
    x_perm = np.zeros((P, cfg.H), np.uint16)
    h = np.zeros((P, cfg.F), np.uint16)
    y = np.zeros((P, cfg.H), np.uint16)
    flat = idx.reshape(-1)
    for i, r in enumerate(d["dest_row"]):
        t, e = i // cfg.k, flat[i]
        x_perm[r] = L.x[t]
        h[r] = orc.swiglu_row(L.x[t], L.w_gate[e], L.w_up[e])
        y[r] = orc.down_row(h[r], L.w_down[e])
    out = orc.combine(y, d["dest_row"], w)
    return dict(idx=idx, w=w, d=d, x_perm=x_perm, h=h, y=y, out=out)


def run_cap_and_spill_ep(dl, shape, G, fused_finish=True, fused_pack=True):
    """The two-pass expert-parallel layer on G ranks held by this process;
    rank r holds tokens [r T, (r+1) T) of the layer dl (fused_finish: the
    unpack folded into the combine; fused_pack: the row copy writing the
    overflow rows straight into the send slots)."""
    from grouped_expert_gemm_router_b200.ep import CapAndSpillEP, exchange_in_process
    T, Eg = shape.T, shape.E // G
    ranks = [CapAndSpillEP(shape, G) for _ in range(G)]
    xs = [dl.x[r * T:(r + 1) * T] for r in range(G)]
    for r, ep in enumerate(ranks):
        ep.route_and_pack(xs[r], dl.w_router, dl.bias, fused=fused_pack)
    exchange_in_process(ranks, "exchange_in")
    for r, ep in enumerate(ranks):
        sl = slice(r * Eg, (r + 1) * Eg)
        ep.local_experts(dl.w_gate[sl], dl.w_up[sl], dl.w_down[sl])
    exchange_in_process(ranks, "exchange_out")
    for ep in ranks:
        ep.finish(fused=fused_finish)
    torch.cuda.synchronize()
    return ranks, xs


def run_direct_ep(dl, shape, G, fused_return=False, fused_plan=False):
    """The peer-store expert-parallel layer on G ranks held by this process
    (fused_return: the down GEMM stores its results into the owners' y;
    fused_plan: plan and dispatch in one launch)."""
    from grouped_expert_gemm_router_b200.ep_direct import DirectEP, connect_in_process, gather_counts_in_process
    T, Eg = shape.T, shape.E // G
    ranks = [DirectEP(shape, G, r) for r in range(G)]
    connect_in_process(ranks)
    xs = [dl.x[r * T:(r + 1) * T] for r in range(G)]
    for r, ep in enumerate(ranks):
        ep.route(xs[r], dl.w_router, dl.bias)
    gather_counts_in_process(ranks)
    if fused_plan:
        for r, ep in enumerate(ranks):
            ep.plan_and_dispatch(xs[r])
    else:
        for ep in ranks:
            ep.plan()
        for r, ep in enumerate(ranks):
            ep.dispatch(xs[r])
    for r, ep in enumerate(ranks):
        sl = slice(r * Eg, (r + 1) * Eg)
        if fused_return:
            ep.experts_and_return(dl.w_gate[sl], dl.w_up[sl], dl.w_down[sl])
        else:
            ep.experts(dl.w_gate[sl], dl.w_up[sl], dl.w_down[sl])
    if not fused_return:
        for ep in ranks:
            ep.send_back()
    for ep in ranks:
        ep.finish()
    torch.cuda.synchronize()
    return ranks, xs


def run_direct_ep_fp8(dl, shape, G, wq, mode="quantize"):
    """The fp8 peer-store layer on G ranks held by this process: each rank's
    token rows become e4m3 code rows and scales in the owners' buffers, the
    owners run the fp8 GEMMs on their experts (wq: the layer's weight codes
    and scales from moe_quantize_weights_fp8, sliced per rank here) and the
    down GEMM stores the results into the tokens' owners' y.  mode
    "quantize": plan and dispatch in one launch that quantizes the rows it
    sends; "codes": the tokens quantized first, then plan and dispatch in one
    launch; "separate": quantize, plan, dispatch as three launches."""
    from grouped_expert_gemm_router_b200.ep_direct import DirectEP, connect_in_process, gather_counts_in_process
    T, Eg = shape.T, shape.E // G
    ranks = [DirectEP(shape, G, r, fp8=True) for r in range(G)]
    connect_in_process(ranks)
    xs = [dl.x[r * T:(r + 1) * T] for r in range(G)]
    for r, ep in enumerate(ranks):
        ep.route(xs[r], dl.w_router, dl.bias)
        if mode != "quantize":
            ep.quantize_tokens(xs[r])
    gather_counts_in_process(ranks)
    if mode != "separate":
        for r, ep in enumerate(ranks):
            ep.plan_and_dispatch(xs[r] if mode == "quantize" else None)
    else:
        for ep in ranks:
            ep.plan()
        for ep in ranks:
            ep.dispatch_fp8()
    for r, ep in enumerate(ranks):
        sl = slice(r * Eg, (r + 1) * Eg)
        ep.experts_fp8_and_return(wq["wg_q"][sl], wq["wg_scale"][sl], wq["wu_q"][sl], wq["wu_scale"][sl],
                                  wq["wd_q"][sl], wq["wd_scale"][sl])
    for ep in ranks:
        ep.finish()
    torch.cuda.synchronize()
    return ranks, xs
