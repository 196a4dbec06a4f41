"""Writes tests/golden/zipf_alpha.json: the router-bias strength of the
long-prefill (T=16384) workload, chosen so that the busiest expert takes about
10x the mean load, as that workload's description asks.

Calls only the oracle's router (FP64 logits, softmax, top-8 with lowest-index
ties) on the seeded inputs. gen.ZIPF_ALPHA holds the value this script found;
tests/test_gen.py checks that the two agree and that the skew holds.

    python tests/golden/make_zipf_alpha.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import gen  # noqa: E402
from oracle import moe  # noqa: E402

TARGET = 10.0


def load_skew(alpha: float, x_bits, router_base, sh) -> tuple:
    router = router_base.copy()
    router[:, gen.ZIPF_CHANNEL] = gen.zipf_bias(gen.WORKLOADS["zipf"].w_seed, sh.E, alpha)
    r = moe.route(x_bits, router, sh.K)
    loads = np.bincount(r.idx.ravel(), minlength=sh.E)
    return loads.max() / loads.mean(), int((loads == 0).sum())


def main():
    wl = gen.WORKLOADS["zipf"]
    sh = wl.shape
    router = gen.normal_f32(wl.w_seed, gen.STREAM_ROUTER, sh.E * sh.H, 0.02).reshape(sh.E, sh.H)
    x = gen.make_x(wl.T, sh.H, wl.x_seed, wl.outliers, zipf=True)
    lo, hi = 0.3, 0.9
    for _ in range(14):
        mid = 0.5 * (lo + hi)
        skew, _ = load_skew(mid, x, router, sh)
        if skew < TARGET:
            lo = mid
        else:
            hi = mid
    alpha = round(0.5 * (lo + hi), 4)
    skew, empty = load_skew(alpha, x, router, sh)
    out = {"alpha": alpha, "max_over_mean": float(skew), "empty_experts": empty,
           "T": wl.T, "x_seed": wl.x_seed, "w_seed": wl.w_seed,
           "source": "oracle router (FP64) on the seeded T=16384 tokens"}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_alpha.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(out)


if __name__ == "__main__":
    main()
