"""The two-regime cost model fit (TEMPO verdict page, arXiv 2608.13057, key
machinery: t = max(a + b*G, c + beta*N), tile-aware + b2*(Tt - G)) on the
CPU: exact recovery of known parameters, recovery under noise, and the
routing the measurement sweep feeds the library."""
import math

import numpy as np
import pytest

from grouped_expert_gemm_router_b200 import cost_model as cm

GS = [1, 2, 4, 8]
NS = [1, 8, 16, 32, 64, 96, 128, 160, 192, 256, 320, 384, 512, 768, 1024]


def _grid(tiles=False):
    G = np.repeat(GS, len(NS))
    n = np.tile(NS, len(GS))
    N = G * n
    Tt = G * np.array([cm.row_tiles(v) for v in n])
    return G, N, Tt


def test_exact_two_regime_recovery():
    G, N, _ = _grid()
    p = dict(a=5.0, b=50.0, b2=0.0, c=2.0, beta=0.25)
    t = cm.predict(p, G, N)
    f = cm.fit_max_affine(G, N, t)
    for k in ("a", "b", "c", "beta"):
        assert f[k] == pytest.approx(p[k], rel=1e-9, abs=1e-9), k
    assert f["n_star"] == pytest.approx(200.0, rel=1e-9)
    assert f["rel_max"] < 1e-12


def test_exact_tile_aware_recovery():
    G, N, Tt = _grid()
    p = dict(a=3.0, b=40.0, b2=40.0, c=1.0, beta=0.2)  # two-tile experts at 320 and 384 rows stay flat
    t = cm.predict(p, G, N, Tt)
    f = cm.fit_max_affine(G, N, t, Tt=Tt)
    for k in ("a", "b", "b2", "c", "beta"):
        assert f[k] == pytest.approx(p[k], rel=1e-9, abs=1e-9), k
    # the points the fit puts in the flat regime are exactly those below the inflection
    flat_true = cm.predict(dict(p, c=-np.inf), G, N, Tt) >= p["c"] + p["beta"] * N
    assert f["flat"] == flat_true.tolist()


def test_recovery_under_noise():
    G, N, _ = _grid()
    p = dict(a=5.0, b=50.0, b2=0.0, c=2.0, beta=0.25)
    rng = np.random.default_rng(0)
    t = cm.predict(p, G, N) * (1.0 + 0.01 * rng.standard_normal(len(G)))
    f = cm.fit_max_affine(G, N, t)
    assert f["b"] == pytest.approx(50.0, rel=0.05)
    assert f["beta"] == pytest.approx(0.25, rel=0.05)
    assert f["n_star"] == pytest.approx(200.0, rel=0.1)
    assert f["rel_rms"] < 0.02


def test_one_regime_only():
    """All points flat (beta -> 0 limit): the fit keeps one plane and reports
    no inflection inside the data."""
    G, N, _ = _grid()
    t = 4.0 + 30.0 * G.astype(np.float64)
    f = cm.fit_max_affine(G, N, t)
    assert f["rel_max"] < 1e-9
    assert f["n_star"] > max(NS) or math.isinf(f["n_star"])


def test_routing_logits_and_tiles():
    lg = cm.routing_logits(3, 5, 8)
    assert lg.shape == (15, 8)
    assert np.argmax(lg, axis=1).tolist() == [0] * 5 + [1] * 5 + [2] * 5
    assert np.bincount(np.argmax(lg, axis=1), minlength=8).tolist() == [5, 5, 5, 0, 0, 0, 0, 0]
    assert [cm.row_tiles(v) for v in (1, 256, 257, 512, 513)] == [1, 1, 2, 2, 3]
