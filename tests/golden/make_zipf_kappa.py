"""Writes tests/golden/zipf_kappa.json: the selection-bias strength of the
skewed (Zipf-like) stacked-layer workload.

The bias is b_e = -kappa * ln(rank_e), rank a seeded permutation of 1..E
(gen.zipf_bias).  kappa is found by bisection so that, over 65,536
calibration tokens (their own seeded stream) routed by layer 0's router, the
sorted per-expert pick frequencies follow a power law of slope -1.1 on a
log-log fit.  The scores come from the fp64 oracle (they do not depend on
kappa, so they are computed once); only the top-k of score + bias is redone
per bisection step.

    python tests/golden/make_zipf_kappa.py [--tokens 65536] [--procs 8]
"""
import argparse
import json
import multiprocessing as mp
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import gen  # noqa: E402

SEED = 0
TARGET_SLOPE = -gen.ZIPF_S


def _scores(args):
    lo, hi = args
    import oracle
    d = gen.V4
    # rows lo..hi of the calibration stream (the same rows gen.x_rows would draw)
    x = np.stack([gen.normal_bf16(gen.derive(SEED + 1, 0, gen.T_CALIB_X, t, 0), d.hidden) for t in range(lo, hi)])
    wr = gen.router_weight(SEED, 0, d.n_experts, d.hidden)
    _, _, s, _ = oracle.route(x, wr, None, d.top_k, d.route_scale)
    return s


def pick_slope(scores, bias, K):
    biased = scores + bias[None, :]
    top = np.argpartition(-biased, K - 1, axis=1)[:, :K]
    freq = np.bincount(top.reshape(-1), minlength=scores.shape[1]).astype(np.float64)
    f = np.sort(freq)[::-1]
    f = f[f > 0]
    ranks = np.arange(1, len(f) + 1, dtype=np.float64)
    slope = np.polyfit(np.log(ranks), np.log(f / f.sum()), 1)[0]
    return slope, freq


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--tokens", type=int, default=65536)
    ap.add_argument("--procs", type=int, default=os.cpu_count() or 1)
    a = ap.parse_args()
    d = gen.V4
    chunk = (a.tokens + a.procs - 1) // a.procs
    parts = [(i, min(a.tokens, i + chunk)) for i in range(0, a.tokens, chunk)]
    with mp.get_context("spawn").Pool(len(parts)) as pool:
        scores = np.concatenate(pool.map(_scores, parts))
    ranks = gen.bias_ranks(SEED, d.n_experts).astype(np.float64)
    lo, hi = 0.0, 4.0
    for _ in range(50):
        mid = 0.5 * (lo + hi)
        bias = gen.zipf_bias(SEED, d.n_experts, mid).astype(np.float64)
        slope, _ = pick_slope(scores, bias, d.top_k)
        if slope > TARGET_SLOPE:  # not steep enough
            lo = mid
        else:
            hi = mid
    kappa = 0.5 * (lo + hi)
    slope, freq = pick_slope(scores, gen.zipf_bias(SEED, d.n_experts, kappa).astype(np.float64), d.top_k)
    out = {"kappa": kappa, "slope": slope, "target_slope": TARGET_SLOPE, "seed": SEED,
           "calibration_tokens": a.tokens, "layer": 0,
           "pick_frequency_by_expert": [int(v) for v in freq],
           "note": "written by tests/golden/make_zipf_kappa.py from oracle scores; b_e = -kappa ln(rank_e)"}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_kappa.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(f"kappa = {kappa:.6f}, slope = {slope:.4f}, top-10 picks = {sorted(freq)[::-1][:10]}")


if __name__ == "__main__":
    main()
