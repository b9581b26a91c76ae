"""Fix the strength alpha of the skewed-routing workload's gate bias (run once; output committed).

The skewed workload (T=8192, d=7168, 256 experts, top-8) adds to every gate logit a per-expert
bias b_e = alpha * ln(rank_e ** -1.2), rank_e a seeded permutation of 1..256 (Zipf, s=1.2, over
expert rank), so that a few experts take most tokens and about 30 receive none.  This script
draws the workload's x / residual / gate weight with the ``synthetic`` generator, evaluates the
normed inputs and the unbiased gate logits with the oracle only, and bisects alpha so that the
number of experts that no token selects is the count closest to 30.  It writes c5_alpha.json.

    python tests/golden/make_c5_alpha.py
"""
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synthetic  # noqa: E402

TARGET_EMPTY = 30


def empty_experts(z, bias, k):
    sel = np.argpartition(-(z + bias[None, :]), k - 1, axis=1)[:, :k]
    used = np.zeros(z.shape[1], bool)
    used[np.unique(sel)] = True
    return int((~used).sum())


def main():
    t0 = time.time()
    shape = synthetic.CONFIGS["C5"]
    inp = synthetic.generate(shape, with_experts=False, alpha=0.0)
    o = oracle.Oracle(shape, dict(inp, gate_bias=None))
    xn = np.empty((shape.T, shape.d), np.uint16)
    x, r, g = (oracle._np(inp[n]) for n in ("x", "residual", "norm_w"))
    for t in range(shape.T):
        xn[t] = oracle.norm_token(x[t], r[t], g, shape.eps)[0]
    s = oracle.gate_scores(xn, o.a["gate_w"], None)
    s = np.clip(s, 1e-300, 1 - 1e-16)
    z = np.log(s) - np.log1p(-s)                       # logits recovered from the scores
    base = synthetic.zipf_bias(shape.seed, shape.E, 1.0).numpy().astype(np.float64)
    lo, hi = 0.0, 4.0
    best = None
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        n = empty_experts(z, mid * base, shape.k)
        if best is None or abs(n - TARGET_EMPTY) < abs(best[1] - TARGET_EMPTY):
            best = (mid, n)
        if n < TARGET_EMPTY:
            lo = mid
        else:
            hi = mid
    alpha, n_empty = best
    out = {"alpha": round(alpha, 6), "empty_experts_oracle": empty_experts(z, round(alpha, 6) * base, shape.k),
           "target_empty": TARGET_EMPTY, "workload": shape.name, "seed": shape.seed,
           "how": "bisection on alpha over the oracle's unbiased gate logits; tests/golden/make_c5_alpha.py"}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "c5_alpha.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(out, f"{time.time() - t0:.1f}s")


if __name__ == "__main__":
    main()
