"""Two-regime cost model of the grouped expert GEMMs and its measurement.

The TEMPO verdict page (arXiv 2608.13057, key machinery and core discovery)
models the MoE-block time of one GPU as a max-affine function of the number of
activated experts G and the number of routed tokens N,

    t = max(a + b*G, c + beta*N)                      (two-regime law)
    t = max(a + b*G + b2*(Tt - G), c + beta*N)        (tile-aware form)

where b is the per-expert cost of streaming its weights from HBM (the flat
regime), beta the per-token compute cost (the linear regime), and
Tt = sum_e ceil(n_e / tile) the number of row tiles; an expert whose tokens
fill more than one tile pays b2 for each extra tile.  The per-expert
inflection n* = b / beta is the token count at which an expert moves from the
flat to the linear regime (the page reports 156-168 tokens for its fp8
kernel on its hardware).

`fit_max_affine` fits the parameters to measured (G, N, Tt, t) points;
`sweep` measures them with this library's grouped GEMMs on the current GPU
(routing exactly n tokens to each of G experts through caller-given logits);
`python -m grouped_expert_gemm_router_b200.cost_model` runs a sweep and the
fit and prints one JSON line.
"""
from __future__ import annotations

import json
import math

import numpy as np


def _lstsq(X, y):
    coef, *_ = np.linalg.lstsq(X, y, rcond=None)
    return coef


def _fit_from(flat, X1, X2, t, iters):
    """Alternating assignment from one initial split; returns (sse, p1, p2, flat)."""
    p1 = p2 = None
    for _ in range(iters):
        if flat.sum() < X1.shape[1] or (~flat).sum() < X2.shape[1]:
            return None
        p1 = _lstsq(X1[flat], t[flat])
        p2 = _lstsq(X2[~flat], t[~flat])
        new = (X1 @ p1) >= (X2 @ p2)
        if np.array_equal(new, flat):
            break
        flat = new
    pred = np.maximum(X1 @ p1, X2 @ p2)
    return float(np.sum(((pred - t) / t) ** 2)), p1, p2, (X1 @ p1) >= (X2 @ p2)


def fit_max_affine(G, N, t, Tt=None, iters=100):
    """Least-squares fit (relative error) of t ~ max(a + b*G [+ b2*(Tt - G)], c + beta*N).

    The max of two planes is fitted by alternating assignment: split the
    points by tokens per expert N/G (the few-token points in the flat
    regime), fit each plane to its points by linear least squares, give every
    point to the plane that predicts the larger time, and repeat until no
    point changes side.  This is run from every threshold split of N/G, and
    the one-plane fits (all flat, all linear) are candidates too; the
    candidate with the smallest squared relative error is returned, with the
    inflection n* = b / beta, the sides and the error."""
    G = np.asarray(G, np.float64)
    N = np.asarray(N, np.float64)
    t = np.asarray(t, np.float64)
    tile = Tt is not None
    cols1 = [np.ones_like(G), G] + ([np.asarray(Tt, np.float64) - G] if tile else [])
    X1 = np.stack(cols1, axis=1)
    X2 = np.stack([np.ones_like(N), N], axis=1)
    if len(t) < X1.shape[1] + X2.shape[1]:
        raise ValueError("too few points for the fit")
    # relative least squares: scale each row by 1/t
    w = 1.0 / t
    cands = []
    p1 = _lstsq(X1 * w[:, None], np.ones_like(t))
    cands.append((float(np.sum(((X1 @ p1) - t) ** 2 * w ** 2)), p1, np.array([-np.inf, 0.0]), np.ones(len(t), bool)))
    p2 = _lstsq(X2 * w[:, None], np.ones_like(t))
    cands.append((float(np.sum(((X2 @ p2) - t) ** 2 * w ** 2)), np.array([-np.inf] + [0.0] * (X1.shape[1] - 1)), p2,
                  np.zeros(len(t), bool)))
    ratio = N / G
    for thr in np.unique(ratio)[:-1]:
        r = _fit_from(ratio <= thr, X1 * w[:, None], X2 * w[:, None], np.ones_like(t), iters)
        if r is not None:
            cands.append(r)
    sse, p1, p2, flat = min(cands, key=lambda c: c[0])
    pred = np.maximum(X1 @ p1, X2 @ p2)
    rel = (pred - t) / t
    a, b = float(p1[0]), float(p1[1])
    b2 = float(p1[2]) if tile else 0.0
    c, beta = float(p2[0]), float(p2[1])
    return {
        "a": a, "b": b, "b2": b2, "c": c, "beta": beta,
        "n_star": b / beta if beta > 0 else math.inf,
        "flat": [bool(v) for v in flat],
        "rel_rms": float(np.sqrt(np.mean(rel ** 2))),
        "rel_max": float(np.max(np.abs(rel))),
    }


def predict(p, G, N, Tt=None):
    G = np.asarray(G, np.float64)
    N = np.asarray(N, np.float64)
    flat = p["a"] + p["b"] * G + (p["b2"] * (np.asarray(Tt, np.float64) - G) if Tt is not None else 0.0)
    return np.maximum(flat, p["c"] + p["beta"] * N)


def routing_logits(G, n, E):
    """fp32 logits [G*n, E] that send tokens g*n .. g*n+n-1 to expert g (k = 1)."""
    T = G * n
    lg = np.zeros((T, E), np.float32)
    lg[np.arange(T), np.repeat(np.arange(G), n)] = 1.0
    return lg


def row_tiles(n, row_cap=256):
    """Row tiles the schedule builder gives an expert of n rows (uncapped)."""
    return max(1, -(-n // row_cap))


def sweep(H, F, E, Gs, ns, reps=20, seed=0, device="cuda"):
    """Time the two grouped GEMMs for every (G, n): G experts with n tokens
    each (k = 1), weights N(0, 0.02^2) bf16, tokens N(0, 1).  Inputs stay
    resident; L2 is cleaned (256 MiB written, then 256 MiB read) before every
    timed repetition.  Returns one record per point (median of reps, in us)."""
    import torch

    from . import (alloc_buffers, make_shape, moe_gather, moe_grouped_down, moe_grouped_swiglu, moe_read_status,
                   moe_route_dispatch)

    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed)
    wg = (torch.randn((E, H, F), generator=gen, device=dev) * 0.02).to(torch.bfloat16)
    wu = (torch.randn((E, H, F), generator=gen, device=dev) * 0.02).to(torch.bfloat16)
    wd = (torch.randn((E, F, H), generator=gen, device=dev) * 0.02).to(torch.bfloat16)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(64 << 20, dtype=torch.float32, device=dev)
    out = []
    for G in Gs:
        for n in ns:
            T = G * n
            shape = make_shape(T, H, F, E, 1, logits_in=True)
            b = alloc_buffers(shape, device=dev)
            x = torch.randn((T, H), generator=gen, device=dev).to(torch.bfloat16)
            b["logits"].copy_(torch.from_numpy(routing_logits(G, n, E)))
            moe_route_dispatch(shape, x, None, None, b["logits"], b["topk_idx"], b["topk_w"], b["expert_counts"],
                               b["expert_offsets"], b["src_token"], b["dest_row"], b["ws"])
            moe_gather(shape, x, b["src_token"], b["x_perm"], b["ws"])
            counts = b["expert_counts"].cpu().numpy()
            assert counts[:G].tolist() == [n] * G and not counts[G:].any(), "routing did not give n rows per expert"

            def gemms():
                moe_grouped_swiglu(shape, b["x_perm"], wg, wu, b["h"], b["ws"])
                moe_grouped_down(shape, b["h"], wd, b["y"], b["ws"])

            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
            for i in range(-3, reps):
                flush_w.zero_()
                flush_r.sum()
                if i >= 0:
                    ev[i][0].record()
                gemms()
                if i >= 0:
                    ev[i][1].record()
            torch.cuda.synchronize()
            if moe_read_status(b["ws"]):
                raise RuntimeError("device status set during the sweep")
            us = float(np.median([s.elapsed_time(e) for s, e in ev])) * 1e3
            out.append({"G": G, "n": n, "N": G * n, "Tt": G * row_tiles(n), "t_us": us})
            del b, x
    return out


def main(argv=None):
    import argparse

    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--H", type=int, default=4096)
    ap.add_argument("--F", type=int, default=14336)
    ap.add_argument("--E", type=int, default=8)
    ap.add_argument("--G", type=str, default="1,2,4,8")
    ap.add_argument("--n", type=str, default="1,8,16,32,64,96,128,160,192,256,320,384,512,768,1024")
    ap.add_argument("--reps", type=int, default=20)
    a = ap.parse_args(argv)
    Gs = [int(v) for v in a.G.split(",")]
    ns = [int(v) for v in a.n.split(",")]
    pts = sweep(a.H, a.F, a.E, Gs, ns, reps=a.reps)
    G = [p["G"] for p in pts]
    N = [p["N"] for p in pts]
    t = [p["t_us"] for p in pts]
    fit2 = fit_max_affine(G, N, t)
    fit3 = fit_max_affine(G, N, t, Tt=[p["Tt"] for p in pts])
    for f in (fit2, fit3):
        f.pop("flat")
    print(json.dumps({"shape": {"H": a.H, "F": a.F, "E": a.E}, "points": pts, "fit": fit2, "fit_tiles": fit3}))


if __name__ == "__main__":
    main()
