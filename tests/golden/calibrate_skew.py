"""Find the Zipf log-prior scale beta of the skewed-routing workload.

Input recipe (skewed prefill, T = 16384, d = 4096, E = 8, k = 2, seed 0):
channel d-1 of x is the constant 1 and the router weight of that channel for
expert e is b_e = -beta * 1.2 * ln(e + 1), rounded to bf16.  This script
bisects beta so that expert 0 receives 35% of the T*k assignments, using the
oracle's router and TopK, and writes tests/golden/skew_beta.json.  The value
is then copied into synth.gen.SKEW_BETA; a CPU test checks the share.

Run from the repository root:  python tests/golden/calibrate_skew.py
"""

import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.abspath(os.path.join(os.path.dirname(__file__), "..", "..")))

import oracle  # noqa: E402
import synth  # noqa: E402

TARGET = 0.35


def shares(g, b_bits, k):
    lg = g + synth.bf16_bits_to_f64(b_bits)[None, :]
    idx = oracle.topk_lower_index(lg, k)
    return np.bincount(idx.ravel(), minlength=g.shape[1]) / idx.size


def main():
    shp = synth.CONFIGS["skewed"]
    t = synth.host_inputs(shp, seed=0, skew_beta=0.0, with_experts=False)
    x = synth.bf16_bits_to_f64(t["x"])
    wg = synth.bf16_bits_to_f64(t["Wg"])
    g = oracle.router_logits(x, wg)  # bias channel is 0 here, so g excludes it
    lo, hi = 0.0, 4.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        s0 = shares(g, synth.skew_biases(shp.E, mid, "bf16"), shp.k)[0]
        if s0 < TARGET:
            lo = mid
        else:
            hi = mid
    beta = round(0.5 * (lo + hi), 6)
    sh = shares(g, synth.skew_biases(shp.E, beta, "bf16"), shp.k)
    out = {"beta": beta, "zipf_s": synth.SKEW_ZIPF_S, "seed": 0, "T": shp.T,
           "target_share_expert0": TARGET, "shares": [round(float(v), 5) for v in sh]}
    with open(os.path.join(os.path.dirname(__file__), "skew_beta.json"), "w") as fh:
        json.dump(out, fh, indent=1)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
