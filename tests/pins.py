"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each ``check_*`` function takes an ``oracle.Oracle`` and raises
AssertionError on a mismatch.  The oracle tests call them on the real oracle;
the mutation test calls them on modified copies of it, to show that each
plausible mistake is caught by at least one pin.

What pins what (nothing here re-types the oracle's own loops):
  top-k      brute force over all k-subsets + Python's sorted() for the order
  weights    scipy.special.softmax on the selected logits; k=2 closed form
  logits     numpy float64 matmul
  dispatch   numpy stable argsort, numpy bincount/cumsum, O(n^2) rank count
  capacity   zero drops, C >= max n_e and C = 0 reductions, overflow bound
  experts    torch float64 matmul for the dense E=1, k=1 layer
  layer      identity experts with unit weights give bf16(k*x) exactly;
             capacity layout output bit-identical to the uncapped output
  fp8        torch.float8_e4m3fn for every code's value and for rounding
             (ties to even, subnormals, saturation); the power-of-two scale
             against its closed-form bounds; row and weight quantizers
             against a torch restatement (frexp + float8 cast); dequantized
             values exactly decode(q) * s
"""
from __future__ import annotations

import itertools
import math

import numpy as np
import scipy.special
import torch

import synth


def _beats(a, i, b, j):
    """The selection key of the routing definition: larger logit first, equal
    logits to the lower expert index, NaN below every number."""
    an, bn = math.isnan(a), math.isnan(b)
    if an or bn:
        return (i < j) if (an and bn) else bn
    if a != b:
        return a > b
    return i < j


def _order_key(l, e):
    return (1 if math.isnan(l) else 0, 0.0 if math.isnan(l) else -l, e)


def check_topk_bruteforce(orc, trials=300, seed=1):
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        E = int(rng.integers(1, 11))
        k = int(rng.integers(1, min(4, E) + 1))
        T = 3
        logits = rng.integers(-3, 4, size=(T, E)).astype(np.float32)  # integer-valued: many ties
        idx, w, _ = orc.topk_softmax(logits, k)
        for t in range(T):
            l = [float(v) for v in logits[t]]
            winners = [S for S in itertools.combinations(range(E), k)
                       if all(_beats(l[i], i, l[j], j) for i in S for j in range(E) if j not in S)]
            assert len(winners) == 1, "definition must single out one subset"
            assert set(idx[t].tolist()) == set(winners[0]), (l, idx[t], winners[0])
            best_sum = max(sum(l[i] for i in S) for S in itertools.combinations(range(E), k))
            assert sum(l[i] for i in idx[t]) == best_sum
            assert idx[t].tolist() == sorted(winners[0], key=lambda e: _order_key(l[e], e))


def check_topk_nan(orc):
    nan = float("nan")
    logits = np.array([[nan, 1.0, nan, -np.inf, 0.5],
                       [nan, nan, nan, nan, nan],
                       [-0.0, 0.0, -0.0, 1.0, nan]], dtype=np.float32)
    idx, w, nseen = orc.topk_softmax(logits, 3)
    assert idx[0].tolist() == [1, 4, 3]   # -inf still beats NaN
    assert idx[1].tolist() == [0, 1, 2]   # all NaN: index order
    assert idx[2].tolist() == [3, 0, 1]   # -0 == +0: lower index first
    assert nseen == 2 + 5 + 1


def check_softmax_weights(orc, seed=2):
    rng = np.random.default_rng(seed)
    for E, k in [(8, 2), (64, 8), (64, 6), (128, 8), (5, 5), (3, 1)]:
        logits = (rng.standard_normal((40, E)) * 2).astype(np.float32)
        idx, w, _ = orc.topk_softmax(logits, k)
        sel = np.take_along_axis(logits, idx, axis=1).astype(np.float64)
        ref = scipy.special.softmax(sel, axis=1)
        assert np.max(np.abs(w - ref)) <= 1e-7
        assert np.all(np.abs(w.astype(np.float64).sum(1) - 1.0) <= 1e-6)
        assert np.all(np.diff(w, axis=1) <= 0)
    # k = 2 closed form: w0 = 1 / (1 + exp(l1 - l0))
    logits = np.array([[0.25, 2.0, -1.0]], dtype=np.float32)
    idx, w, _ = orc.topk_softmax(logits, 2)
    assert idx[0].tolist() == [1, 0]
    w0 = 1.0 / (1.0 + math.exp(0.25 - 2.0))
    assert abs(float(w[0, 0]) - w0) <= 6e-8 and abs(float(w[0, 1]) - (1 - w0)) <= 6e-8


def check_router_logits(orc, seed=3):
    for (T, H, E, alpha) in [(17, 96, 8, 0.0), (9, 256, 64, 2.0), (5, 64, 3, 1.0)]:
        cfg = synth.LayerConfig("t", T, H, 64, E, 1, alpha=alpha, seed=seed)
        L = synth.make_layer(cfg, with_experts=False)
        logits = orc.router_logits(L.x, L.w_router, L.bias)
        ref = (synth.bf16_bits_to_f32(L.x).astype(np.float64) @ L.w_router.astype(np.float64)).astype(np.float32)
        if L.bias is not None:
            ref = ref + L.bias  # fp32 add, as the definition states
        d = np.abs(logits.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
        assert d.max() <= 1 and (d == 0).mean() >= 0.98, (d.max(), (d == 0).mean())


def check_dispatch_uncapped(orc, seed=4):
    rng = np.random.default_rng(seed)
    for (T, E, k) in [(1, 1, 1), (7, 4, 2), (50, 8, 3), (200, 64, 8), (33, 5, 5)]:
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        d = orc.dispatch(idx, E)
        flat = idx.reshape(-1)
        assert np.array_equal(d["counts"], np.bincount(flat, minlength=E))
        assert np.array_equal(d["offsets"], np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
        order = np.argsort(flat, kind="stable")          # row r holds pair order[r]
        assert np.array_equal(d["dest_row"][order], np.arange(T * k))
        assert np.array_equal(d["src_token"], order // k)
        assert d["counts"].sum() == T * k and d["counts"].max() <= T


def check_dispatch_bruteforce(orc, seed=5):
    rng = np.random.default_rng(seed)
    T, E, k = 12, 5, 3
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    flat = idx.reshape(-1).tolist()
    d = orc.dispatch(idx, E)
    for i, e in enumerate(flat):
        before_experts = sum(1 for x in flat if x < e)
        same_before = sum(1 for x in flat[:i] if x == e)
        assert d["dest_row"][i] == before_experts + same_before


def check_capacity_layout(orc, seed=6):
    rng = np.random.default_rng(seed)
    for (T, E, k, C) in [(40, 8, 2, 3), (128, 64, 6, 16), (10, 4, 4, 0), (9, 6, 2, 20), (30, 5, 3, 7)]:
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        # skew: push most tokens to expert 0 on half the trials
        if rng.random() < 0.5:
            idx[:, 0] = 0
            for t in range(T):
                rest = [e for e in rng.permutation(E) if e != 0][:k - 1]
                idx[t, 1:] = rest
        u = orc.dispatch(idx, E)
        c = orc.dispatch(idx, E, C=C, capped=True)
        R = T * k
        P = E * C + k * max(0, T - C)
        assert c["P"] == P
        rows = c["dest_row"]
        assert len(set(rows.tolist())) == R, "every routed pair has its own row (no drop)"
        assert rows.min() >= 0 and rows.max() < P
        assert np.array_equal(c["counts"], u["counts"])
        assert np.array_equal(c["cap_cnt"], np.minimum(u["counts"], C))
        assert np.array_equal(c["spill_cnt"], u["counts"] - np.minimum(u["counts"], C))
        assert (c["cap_cnt"].sum() + c["spill_cnt"].sum()) == R
        assert c["spill_cnt"].sum() <= P - E * C
        src = c["src_token"]
        for i in range(R):
            assert src[rows[i]] == i // k
        assert (src >= 0).sum() == R
        # rank within the expert (uncapped) decides capacity vs overflow
        for i in range(R):
            e = idx.reshape(-1)[i]
            r = u["dest_row"][i] - u["offsets"][e]
            if r < C:
                assert rows[i] == e * C + r
            else:
                assert rows[i] == E * C + c["spill_off"][e] + r - C
        if C == 0:
            assert np.array_equal(rows, u["dest_row"])
        if C >= u["counts"].max():
            assert c["spill_cnt"].sum() == 0
    # worst case: k experts hold every token, the overflow fills its buffer exactly
    T, E, k, C = 20, 6, 3, 4
    idx = np.tile(np.arange(k, dtype=np.int32), (T, 1))
    c = orc.dispatch(idx, E, C=C, capped=True)
    assert c["spill_cnt"].sum() == c["P"] - E * C == k * (T - C)


def check_identity_layer(orc, seed=7):
    for (T, H, E, k, C, capped, alpha) in [(37, 64, 8, 2, 0, False, 0.0), (20, 32, 6, 6, 2, True, 1.0),
                                          (64, 128, 8, 8, 0, False, 2.0), (5, 16, 3, 1, 1, True, 0.0)]:
        cfg = synth.LayerConfig("t", T, H, 16, E, k, C=C, alpha=alpha, seed=seed)
        L = synth.make_layer(cfg, with_experts=False)
        r = orc.forward(L.x, L.w_router, L.bias, None, None, None, k, C=C, capped=capped,
                        expert=1, w_in=np.ones((T, k), np.float32))
        ref = synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(L.x) * np.float32(k))
        assert np.array_equal(r["out"], ref)


def check_identity_softmax_weights(orc, seed=11):
    """Identity experts and the routing's own weights: sum_j w_j = 1, so the
    layer returns x up to the fp32 rounding of the weighted sum."""
    for (T, H, E, k, alpha) in [(33, 64, 8, 2, 0.0), (16, 32, 64, 8, 2.0)]:
        cfg = synth.LayerConfig("t", T, H, 16, E, k, alpha=alpha, seed=seed)
        L = synth.make_layer(cfg, with_experts=False)
        r = orc.forward(L.x, L.w_router, L.bias, None, None, None, k, expert=1)
        assert _bf16_ulps(r["out"], L.x).max() <= 1


def check_combine_vs_torch(orc, seed=12):
    rng = np.random.default_rng(seed)
    T, H, k, P = 23, 40, 3, 80
    y = synth.f32_to_bf16_bits(rng.standard_normal((P, H)).astype(np.float32))
    dest = rng.permutation(P)[:T * k].astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    out = orc.combine(y, dest, w)
    yt = torch.from_numpy(synth.bf16_bits_to_f32(y)).double()[torch.from_numpy(dest.astype(np.int64))]
    ref = (yt.view(T, k, H) * torch.from_numpy(w).double()[:, :, None]).sum(1).float().to(torch.bfloat16)
    ref_bits = ref.view(torch.int16).numpy().view(np.uint16)
    d = _bf16_ulps(out, ref_bits)
    assert d.max() <= 1 and (d == 0).mean() >= 0.98


def _bf16_ulps(a_bits, b_bits):
    a = a_bits.astype(np.int32)
    b = b_bits.astype(np.int32)
    a = np.where(a & 0x8000, 0x8000 - a, a)  # sign-magnitude -> ordered integers
    b = np.where(b & 0x8000, 0x8000 - b, b)
    return np.abs(a - b)


def check_dense_swiglu_vs_torch(orc, seed=8):
    for (T, H, F) in [(12, 64, 96), (5, 128, 256)]:
        cfg = synth.LayerConfig("t", T, H, F, 1, 1, seed=seed)
        L = synth.make_layer(cfg)
        r = orc.forward(L.x, L.w_router, None, L.w_gate, L.w_up, L.w_down, 1)
        assert np.all(r["w"] == 1.0)
        x = torch.from_numpy(synth.bf16_bits_to_f32(L.x)).double()
        wg = torch.from_numpy(synth.bf16_bits_to_f32(L.w_gate[0])).double()
        wu = torch.from_numpy(synth.bf16_bits_to_f32(L.w_up[0])).double()
        wd = torch.from_numpy(synth.bf16_bits_to_f32(L.w_down[0])).double()
        g = x @ wg
        h = (torch.nn.functional.silu(g) * (x @ wu)).float().to(torch.bfloat16)
        y = (h.double() @ wd).float().to(torch.bfloat16)
        h_bits = h.view(torch.int16).numpy().view(np.uint16)
        y_bits = y.view(torch.int16).numpy().view(np.uint16)
        dh = _bf16_ulps(r["h"], h_bits)
        dy = _bf16_ulps(r["out"], y_bits)
        assert dh.max() <= 1 and (dh == 0).mean() >= 0.99, (dh.max(), (dh == 0).mean())
        assert dy.max() <= 2 and (dy == 0).mean() >= 0.97, (dy.max(), (dy == 0).mean())


def check_capped_equals_uncapped(orc, seed=9):
    cfg = synth.LayerConfig("t", 48, 64, 128, 8, 3, C=4, alpha=1.5, seed=seed)
    L = synth.make_layer(cfg)
    u = orc.forward(L.x, L.w_router, L.bias, L.w_gate, L.w_up, L.w_down, 3)
    c = orc.forward(L.x, L.w_router, L.bias, L.w_gate, L.w_up, L.w_down, 3, C=4, capped=True)
    assert np.array_equal(u["out"], c["out"])
    assert c["spill_cnt"].sum() > 0  # the case really spills


def check_token_outputs(orc, seed=10):
    cfg = synth.LayerConfig("t", 30, 64, 128, 6, 2, alpha=0.5, seed=seed)
    L = synth.make_layer(cfg)
    r = orc.forward(L.x, L.w_router, L.bias, L.w_gate, L.w_up, L.w_down, 2)
    toks = np.array([0, 7, 29], np.int32)
    o = orc.token_outputs(toks, L.x, r["idx"], r["w"], L.w_gate, L.w_up, L.w_down)
    assert np.array_equal(o, r["out"][toks])


def _torch_e4m3(v):
    """float32 -> e4m3 codes by torch's cast (round to nearest even)."""
    t = torch.as_tensor(np.asarray(v, np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def check_e4m3_decode_all_codes(orc):
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([orc.e4m3_decode(q) for q in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.nanmax(got) == 448.0 and got[1] == 2.0 ** -9


def check_e4m3_encode_rounding(orc, seed=13):
    vals = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    fin = np.unique(vals[np.isfinite(vals) & (vals >= 0)])
    mids = (fin[1:] + fin[:-1]) / 2  # ties: round to the even code
    rng = np.random.default_rng(seed)
    rand = np.concatenate([rng.uniform(-448, 448, 3000), rng.uniform(-2 ** -5, 2 ** -5, 3000),
                           rng.standard_normal(3000) * 40, np.linspace(448, 464, 17)])
    v = np.concatenate([fin, -fin, mids, -mids, rand]).astype(np.float32)
    got = np.array([orc.e4m3_encode(x) for x in v], np.uint8)
    assert np.array_equal(got, _torch_e4m3(v))
    # beyond 464 torch gives NaN; the oracle saturates (never reached with its scales)
    assert orc.e4m3_encode(1000.0) == 0x7E and orc.e4m3_encode(-1000.0) == 0xFE


def check_fp8_scale(orc, seed=14):
    rng = np.random.default_rng(seed)
    for a in np.concatenate([rng.lognormal(0, 8, 2000), 2.0 ** np.arange(-60, 60)]).astype(np.float32):
        s = orc.fp8_scale(float(a))
        m, e = math.frexp(s)
        assert m == 0.5, "scale must be a power of two"
        assert 128 * s < a <= 256 * s, (a, s)
    for j in range(-40, 40):
        assert orc.fp8_scale(2.0 ** j) == 2.0 ** (j - 8)
    assert orc.fp8_scale(0.0) == 1.0


def _torch_quant_rows(v_f32):
    """Rows -> (codes, scales) restated with torch: scale 2^(ceil(log2 amax) - 8)."""
    t = torch.as_tensor(v_f32, dtype=torch.float32)
    amax = t.abs().amax(dim=-1)
    m, e = torch.frexp(amax)
    c = torch.where(m == 0.5, e - 1, e)
    s = torch.where(amax > 0, torch.ldexp(torch.ones_like(amax), (c - 8).float()), torch.ones_like(amax))
    q = (t / s[..., None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return q.numpy(), s.numpy()


def check_quantize_rows_and_weights(orc, seed=15):
    rng = np.random.default_rng(seed)
    rows = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(
        (rng.standard_normal((33, 160)) * rng.lognormal(0, 3, (33, 1))).astype(np.float32)))
    rows[3] = 0.0
    bits = synth.f32_to_bf16_bits(rows)
    q, s = orc.quantize_rows(bits)
    tq, ts = _torch_quant_rows(rows)
    assert np.array_equal(s, ts) and np.array_equal(q, tq)
    # weights [E, K, N] -> codes [E, N, K], one scale per (e, n) over K
    w = synth.f32_to_bf16_bits((rng.standard_normal((3, 96, 40)) * 0.02).astype(np.float32))
    wq, ws = orc.quantize_weights(w)
    tq, ts = _torch_quant_rows(synth.bf16_bits_to_f32(w).transpose(0, 2, 1))
    assert wq.shape == (3, 40, 96) and np.array_equal(wq, tq) and np.array_equal(ws, ts)
    # dequantized values are exactly decode(q) * s, and within 2^-4 relative of the input
    deq = synth.bf16_bits_to_f32(orc.dequantize(q, s)).astype(np.float64)
    ref = torch.as_tensor(q).view(torch.float8_e4m3fn).double().numpy() * s[:, None].astype(np.float64)
    assert np.array_equal(deq, ref)
    err = np.abs(deq - rows)
    assert np.all(err <= 2.0 ** -4 * np.abs(rows) + 2.0 ** -10 * s[:, None])
    back = orc.dequantize_weights(wq, ws)
    assert back.shape == w.shape
    assert np.all(np.abs(synth.bf16_bits_to_f32(back) - synth.bf16_bits_to_f32(w)) <=
                  2.0 ** -4 * np.abs(synth.bf16_bits_to_f32(w)) + 2.0 ** -10 * ws[:, None, :])


ALL_CHECKS = [check_topk_bruteforce, check_topk_nan, check_softmax_weights, check_router_logits,
              check_dispatch_uncapped, check_dispatch_bruteforce, check_capacity_layout, check_identity_layer,
              check_identity_softmax_weights, check_combine_vs_torch, check_dense_swiglu_vs_torch,
              check_capped_equals_uncapped, check_token_outputs, check_e4m3_decode_all_codes,
              check_e4m3_encode_rounding, check_fp8_scale, check_quantize_rows_and_weights]
