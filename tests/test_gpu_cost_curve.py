"""The cost-curve sweep on the GPU: it routes exactly n rows to each of G
experts, times the two grouped GEMMs, and the two-regime law of the TEMPO
verdict page (arXiv 2608.13057) fits the measured points (Qwen3-30B-A3B
expert shape, H = 2048, F = 768)."""
import pytest

from grouped_expert_gemm_router_b200 import cost_model as cm

pytestmark = pytest.mark.gpu


def test_sweep_and_fit():
    Gs, ns = [8, 32, 128], [1, 16, 64, 256, 512, 1024]
    pts = cm.sweep(2048, 768, 128, Gs, ns, reps=5)
    assert len(pts) == len(Gs) * len(ns)
    t = {(p["G"], p["n"]): p["t_us"] for p in pts}
    for G in Gs:
        assert t[(G, 16)] < 1.3 * t[(G, 1)]       # flat: a few rows cost what one row costs
        assert t[(G, 1024)] > 1.5 * t[(G, 1)]     # linear: 1024 rows per expert cost more
    assert t[(128, 1)] > 2 * t[(8, 1)]            # the flat cost grows with the experts touched
    f = cm.fit_max_affine([p["G"] for p in pts], [p["N"] for p in pts], [p["t_us"] for p in pts])
    assert f["b"] > 0 and f["beta"] > 0
    assert 32 < f["n_star"] < 1024
    assert f["rel_rms"] < 0.25
