"""Writes bit_routed_expert_sigmoid_b200/redraws.json (the synthetic generator's package data): for each synthetic router, how many times each token row of
x is redrawn so that the gap between its 6th and 7th sigmoid scores is at least 1e-4.

The workload definition asks for that resampling; the gap is computed by the fp64 oracle only.
Run from the repository root:  python tests/golden/make_redraws.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from bit_routed_expert_sigmoid_b200 import synthetic as S  # noqa: E402
from oracle import flint_moe_ref as R  # noqa: E402

GAP_MIN = 1e-4
ROUTERS = [  # (E, weight seed, skew, rows covered)
    (32, S.SEED_WEIGHTS, False, 4096),
    (256, S.SEED_WEIGHTS, False, 4096),
    (256, S.SEED_WEIGHTS, True, 4096),
    (256, 1000, False, 64),
]


def key(E, seed, skew):
    return f"E{E}_seed{seed}" + ("_skew" if skew else "")


def table(E, seed, skew, rows):
    L = S.make_layer(E, seed=seed, skew=skew) if E <= 32 else None
    if L is None:
        # only the router matters for the gap; draw it the same way make_layer does
        full = S.make_layer(E, seed=seed, skew=skew)
        L = {"router_w": full["router_w"]}
    x = S.make_x(rows, skew=skew)
    gap = R.router_gap(L, x)
    red = {}
    for r in np.nonzero(gap < GAP_MIN)[0]:
        d = 0
        while True:
            d += 1
            g = R.router_gap(L, S.x_row(int(r), d, skew=skew)[None, :])[0]
            if g >= GAP_MIN:
                break
        red[int(r)] = d
    return red


def main():
    out = {"gap_min": GAP_MIN, "tables": {}}
    for E, seed, skew, rows in ROUTERS:
        red = table(E, seed, skew, rows)
        out["tables"][key(E, seed, skew)] = {"rows": rows, "redraws": {str(k): v for k, v in sorted(red.items())}}
        print(key(E, seed, skew), len(red), "rows redrawn of", rows)
    with open(os.path.join(ROOT, "bit_routed_expert_sigmoid_b200", "redraws.json"), "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main()
