"""The oracle against hand-worked fixtures in tests/golden (each cites its passage)."""
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    rows = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        key, *vals = line.split()
        rows.setdefault(key, []).append(vals)
    return rows


def _ints(rows, key):
    return np.array([int(v) for v in rows[key][0]], dtype=np.int64)


def test_routing_ties(orc):
    g = _read("routing_ties.txt")
    k = int(g["k"][0][0])
    logits = np.array([[float(v) for v in r] for r in g["logits"]], dtype=np.float32)
    idx, w, _ = orc.topk_softmax(logits, k)
    assert idx.tolist() == [[int(v) for v in r] for r in g["idx"]]
    ref = np.array([[float(v) for v in r] for r in g["w"]])
    assert np.max(np.abs(w - ref)) <= 1e-7


def test_dispatch_small(orc):
    g = _read("dispatch_small.txt")
    E = int(g["E"][0][0])
    idx = np.array([[int(v) for v in r] for r in g["idx"]], dtype=np.int32)
    d = orc.dispatch(idx, E)
    for key in ("counts", "offsets", "dest_row", "src_token"):
        assert np.array_equal(d[key], _ints(g, key)), key
    C = int(g["C"][0][0])
    c = orc.dispatch(idx, E, C=C, capped=True)
    assert c["P"] == int(g["P_capped"][0][0])
    for key in ("cap_cnt", "spill_cnt", "spill_off"):
        assert np.array_equal(c[key], _ints(g, key)), key
    assert np.array_equal(c["dest_row"], _ints(g, "dest_row_capped"))
    assert np.array_equal(c["src_token"], _ints(g, "src_token_capped"))


def test_cap_and_spill_43(orc):
    g = _read("cap_and_spill_43.txt")
    T, E = int(g["T"][0][0]), int(g["E"][0][0])
    idx = np.zeros((T, 1), dtype=np.int32)
    c = orc.dispatch(idx, E, C=int(g["C"][0][0]), capped=True)
    assert c["cap_cnt"][0] == int(g["cap_cnt0"][0][0])
    assert c["spill_cnt"][0] == int(g["spill_cnt0"][0][0])
    assert c["spill_cnt"][0] == T - 16 == 27
    p = orc.dispatch(idx, E, C=int(g["C_padded"][0][0]), capped=True)
    assert p["spill_cnt"].sum() == int(g["spill_padded"][0][0])
