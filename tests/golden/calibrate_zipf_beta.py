"""Calibrate the Zipf bias strength of the skewed workload with the oracle.

The skewed workload (T=16384 tokens, 256 experts, top-8) should send about
half of all T*k assignments to the 10% most loaded experts.  Its gate is
Wg = G + beta * V (see workloads.zipf_parts).  This script computes the fp64
oracle logits of the two parts once, then bisects beta so that the oracle's
top-k routing of logits(G) + beta * logits(V) gives a top-10% share of 0.50.
It writes zipf_beta.json next to itself; the constant ZIPF_BETA in
workloads.py is copied from there.

Only oracle/ computes here (the draws come from the workload generator).
Run:  python tests/golden/calibrate_zipf_beta.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from mixture_experts_ffn_17_b200 import workloads  # noqa: E402


def top10_share(counts):
    c = np.sort(counts)[::-1]
    n = max(1, int(round(0.10 * len(c))))
    return c[:n].sum() / c.sum()


def main():
    cfg = workloads.CONFIGS["skewed"]
    x, G, V = workloads.zipf_parts(cfg, "cpu")
    xd = oracle.decode(x)
    lg_g = oracle.logits(xd, G.double().numpy())
    lg_v = oracle.logits(xd, V.double().numpy())

    def share(beta):
        idx, _, _ = oracle.route_topk_softmax(lg_g + beta * lg_v, cfg.k)
        counts, _, _, _ = oracle.dispatch(idx, cfg.E)
        return top10_share(counts), int((counts == 0).sum()), int(counts.max())

    lo, hi = 0.0, 2.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        if share(mid)[0] < 0.50:
            lo = mid
        else:
            hi = mid
    beta = round(0.5 * (lo + hi), 4)
    s, empty, cmax = share(beta)
    out = {"beta": beta, "top10_share": round(float(s), 4), "empty_experts": empty, "max_count": cmax,
           "T": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k, "seed": cfg.seed,
           "note": "Zipf(1.1) log-popularity bias; the share target is the skewed workload's statement"}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_beta.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(out)


if __name__ == "__main__":
    main()
