"""Find the expert-0 logit bias of the long_skewed workload.

Bisects beta (bias vector (beta, 0, ..., 0)) until expert 0 receives about 40%
of the T*k slots under the CPU oracle's routing of the seeded x and router
weight, then writes tests/golden/long_skewed_bias.json. The value found is
copied into LONG_SKEWED_BETA in the inputs module (rounded to a multiple of
1/64 so it is exact in binary).

Run: python tests/golden/calibrate_long_skewed_bias.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from workloads import CONFIGS, make_inputs  # noqa: E402
from oracle import moe_oracle as O  # noqa: E402


def share(l64, beta, k):
    l = l64.copy()
    l[:, 0] += beta
    idx = O.topk_select(l.astype(np.float32), k)
    return float(np.mean(idx == 0))


def main():
    shape = CONFIGS["long_skewed"]
    inp = make_inputs(shape, experts=False)
    l64 = O.gate_logits(inp.x.float().numpy(), inp.wg.float().numpy(), None)
    lo, hi = 0.0, 8.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if share(l64, mid, shape.k) < 0.40:
            lo = mid
        else:
            hi = mid
    beta = round(0.5 * (lo + hi) * 64) / 64
    s = share(l64, beta, shape.k)
    out = {"workload": "long_skewed", "beta": beta, "expert0_share": s,
           "target": [0.39, 0.41],
           "how": "bisection on beta with the CPU oracle's top-k of the seeded inputs"}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "long_skewed_bias.json"), "w") as f:
        json.dump(out, f, indent=2)
    print(out)


if __name__ == "__main__":
    main()
