"""Calibrate the strength alpha of the Zipf-ranked router-logit offset.

The skewed prefill workload adds b_e = -alpha * 1.1 * ln(rank_e) to the router logits so
that expert loads are imbalanced: some experts get about ten times the mean load
(T*k/E) and some receive no token.  With one Zipf offset these two goals pull apart
(the load at which the first expert empties already puts the top experts above 10x),
so alpha is the smallest value at which at least one expert is empty; the loads that
result are recorded.  This script finds it by bisection with the oracle's router on
the T=2048 full-shape layer (seed 1234, first draws of x), then writes zipf_alpha.json
beside itself.  It calls only `oracle` and
`synth`.

    python tests/golden/calibrate_zipf.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

SEED = 1234


def loads(logits, bias, k, E):
    l = logits + bias.astype(np.float64)
    idx = np.argsort(-l, axis=1, kind="stable")[:, :k]
    return np.bincount(idx.reshape(-1), minlength=E)


def main():
    shape = synth.PREFILL
    p = synth.make_router(SEED, shape)
    x = synth.x_rows(SEED + 1, shape.H, shape.T)
    r = oracle.router(oracle.bf16(x), oracle.bf16(p["router_scale"]), oracle.bf16(p["w_router"]),
                      None, oracle.bf16(p["per_expert_scale"]), shape.k, shape.eps)
    mean = shape.T * shape.k / shape.E
    lo, hi = 0.0, 1.0
    for _ in range(60):
        mid = 0.5 * (lo + hi)
        c = loads(r["logits"], synth.zipf_bias(SEED, shape.E, mid), shape.k, shape.E)
        if (c == 0).sum() == 0:
            lo = mid
        else:
            hi = mid
    alpha = hi
    c = loads(r["logits"], synth.zipf_bias(SEED, shape.E, alpha), shape.k, shape.E)
    out = {
        "_what": "strength of the Zipf(s=1.1)-ranked per-expert router-logit offset for the "
                 "skewed T=2048 prefill workload; written by calibrate_zipf.py from the oracle's router",
        "alpha": float(alpha),
        "seed": SEED,
        "max_load_over_mean": float(c.max() / mean),
        "empty_experts": int((c == 0).sum()),
        "experts_at_8x_or_more": int((c >= 8 * mean).sum()),
        "sorted_loads_top8": [int(v) for v in np.sort(c)[::-1][:8]],
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_alpha.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    print(out)


if __name__ == "__main__":
    main()
