"""Calibrate the planted tail of the long-context decode workload with the fp64 oracle.

The workload's configuration asks for a planted heavy tail of "2% of positions +3 sigma".  The
tail is planted in the indexer keys (the method's input), so "+3 sigma" is a statement about the
indexer scores: this script finds the shift beta of the planted keys (along the unit vector of
sum_h w[h] q[h], in key-element units) at which the median planted score lies 3 standard
deviations above the mean of the unplanted scores, all scores computed by the fp64 oracle from the
e4m3-quantised keys, on one request of the workload drawn on the CPU.  It writes the result to
planted_beta.json next to this file; dsa_inputs.PLANTED_BETA holds the same value.

    python tests/golden/make_planted_beta.py
"""
import json
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import dsa_inputs as di  # noqa: E402
import oracle  # noqa: E402


def draw_request(spec):
    """Request 0 of `spec` on the CPU, unplanted: (q_idx, w, kraw [rows, Di] f32, block table)."""
    bt, nblk = di.make_block_table(spec.lens, spec.seed)
    q_idx = di.normal((spec.T, spec.Hi, spec.Di), torch.bfloat16, "cpu", spec.seed, 1)
    w = di.uniform01((spec.T, spec.Hi), "cpu", spec.seed, 2)
    kraw = di.normal((nblk * di.BLOCK, spec.Di), torch.float32, "cpu", spec.seed, 3)
    return q_idx, w, kraw, bt, nblk


def scores_of(kraw_rows, q_idx, w):
    """Oracle scores of query 0 against the given key rows (quantised to e4m3 as the workload is)."""
    n = kraw_rows.shape[0]
    nb = -(-n // di.BLOCK)
    pad = torch.zeros((nb * di.BLOCK, kraw_rows.shape[1]), dtype=torch.float32)
    pad[:n] = kraw_rows
    codes, scale = di.quantize_e4m3(pad)
    bt = torch.arange(nb, dtype=torch.int32).view(1, nb)
    s = oracle.indexer_scores(q_idx[:1], w[:1], codes.view(nb, di.BLOCK, -1), scale.view(nb, di.BLOCK), bt,
                              torch.tensor([0], dtype=torch.int32), torch.tensor([n - 1], dtype=torch.int32))
    return s[0, :n]


def lift(beta, base, planted_rows, u, q_idx, w, mu, sd):
    """(median planted score - mean of the unplanted scores) / their standard deviation."""
    s = scores_of(base[planted_rows] + beta * u, q_idx, w)
    return (float(np.median(s)) - mu) / sd


def main():
    spec = di.long_decode(B=1)
    q_idx, w, kraw, bt, _ = draw_request(spec)
    L = spec.lens[0]
    rows = (bt[0].long()[torch.arange(L) // di.BLOCK] * di.BLOCK + torch.arange(L) % di.BLOCK)
    base = kraw[rows]  # request 0's keys in position order
    planted = di.planted_positions(spec, 0)
    mask = torch.ones(L, dtype=torch.bool)
    mask[planted] = False
    s_all = scores_of(base, q_idx, w)
    unpl = s_all[mask.numpy()]
    mu, sd = float(unpl.mean()), float(unpl.std())
    u = di.plant_direction(q_idx[0], w[0])
    lo, hi = 0.0, 32.0
    for _ in range(20):  # bisection on beta (the lift grows with beta), to 2^-15 of the bracket
        mid = 0.5 * (lo + hi)
        if lift(mid, base, planted, u, q_idx, w, mu, sd) < 3.0:
            lo = mid
        else:
            hi = mid
    beta = round(0.5 * (lo + hi) * 1024) / 1024  # a short binary fraction, stored exactly
    achieved = lift(beta, base, planted, u, q_idx, w, mu, sd)
    out = {"beta": beta, "achieved_lift_sigma": achieved, "unplanted_mean": mu, "unplanted_std": sd,
           "planted": int(planted.numel()), "positions": L, "seed": spec.seed,
           "how": "oracle scores of request 0 of the long-context decode workload drawn on the CPU; "
                  "median planted score = unplanted mean + 3 unplanted standard deviations"}
    with open(os.path.join(HERE, "planted_beta.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
