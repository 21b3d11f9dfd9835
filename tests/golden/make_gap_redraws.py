"""Write gap_redraws.json: which token rows of each named workload to redraw.

A row is redrawn (attempt 0, 1, ...) while the gap between its largest and
second-largest router logit, computed by the fp64 oracle, is below 1e-3.  This
makes the top-1 expert unique, so a fp32 router must choose the same expert.

Run from the repository root:  python tests/golden/make_gap_redraws.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
import oracle  # noqa: E402

GAP = 1e-3
SEED = 0


def redraws_for(spec, seed=SEED, chunk=8192):
    r = synth.make_router(spec, seed)
    W_r, b_r = r["W_r"], r["b_r"]
    x = synth.make_x(spec, seed)
    rows = {}
    todo = []
    for s in range(0, spec.T, chunk):
        gap = oracle.logit_gap(oracle.router_logits(x[s:s + chunk], W_r, b_r))
        todo += (np.nonzero(gap < GAP)[0] + s).tolist()
    while todo:
        nxt = []
        for t in todo:
            rows[t] = rows.get(t, -1) + 1
            xt = synth.draw((seed, spec.name, "x_redraw", t, rows[t]), (1, spec.d), "normal",
                            1.0, spec.dtype)
            if oracle.logit_gap(oracle.router_logits(xt, W_r, b_r))[0] < GAP:
                nxt.append(t)
        todo = nxt
    return rows


def main():
    out = {"gap": GAP, "note": "rows redrawn until the fp64 top-1/top-2 router-logit gap >= gap",
           "workloads": {}}
    for name, spec in synth.WORKLOADS.items():
        rows = redraws_for(spec)
        out["workloads"][name] = {"seed": SEED, "rows": {str(k): v for k, v in sorted(rows.items())}}
        print(name, "redrawn rows:", len(rows), flush=True)
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "gap_redraws.json"), "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main()
