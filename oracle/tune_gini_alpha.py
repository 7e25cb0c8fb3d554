"""Find the router-bias skew alpha that gives a per-expert token-count Gini of
about 0.3 for the DeepSeek-V2-Lite-shaped decode layer (T=128, H=2048, E=64,
k=6, seed 0), the band the "DODOCO" abstract (arXiv 2605.20982) reports for
MLA routing.  Routing is computed by the CPU oracle only.

Gini = sum_i sum_j |n_i - n_j| / (2 E^2 mean(n)).

Usage: python oracle/tune_gini_alpha.py   (prints the alpha to freeze)
"""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import synth  # noqa: E402
from oracle import Oracle  # noqa: E402


def gini(counts):
    n = np.asarray(counts, dtype=np.float64)
    return float(np.abs(n[:, None] - n[None, :]).sum() / (2 * len(n) ** 2 * n.mean()))


def counts_at(alpha, orc, base):
    cfg = base.with_(alpha=alpha)
    L = synth.make_layer(cfg, with_experts=False)
    idx, _, _ = orc.topk_softmax(orc.router_logits(L.x, L.w_router, L.bias), cfg.k)
    return np.bincount(idx.reshape(-1), minlength=cfg.E)


def main():
    orc = Oracle()
    base = synth.CONFIGS[4]
    lo, hi = 0.0, 2.0
    for _ in range(12):
        mid = (lo + hi) / 2
        g = gini(counts_at(mid, orc, base))
        if g < 0.30:
            lo = mid
        else:
            hi = mid
    for a in (lo, hi):
        c = counts_at(a, orc, base)
        print("alpha=%.7f gini=%.4f max=%d mean=%.2f overflow(C=16)=%d" %
              (a, gini(c), c.max(), c.mean(), np.maximum(c - 16, 0).sum()))


if __name__ == "__main__":
    main()
