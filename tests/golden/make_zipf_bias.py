"""Write the per-expert router bias of the skewed-load prefill workload.

The workload adds a per-expert bias b to the router logits so that expert
popularity follows Zipf(s): expert e, ranked pi(e) by a seeded permutation,
should receive a share q_e proportional to (pi(e)+1)^-s of the T*k routed
slots, capped at T slots (one token picks an expert at most once; the mass
above the cap is spread over the other experts in proportion to q).

b is fitted on a calibration batch that is not the measured batch (x drawn
with seed+1, W_router the workload's own) by damped fixed-point steps
    b_e <- b_e + eta * (ln target_e - ln max(realised_e, 1/2)),
where realised_e is the oracle's routed-slot count of expert e under the
current b.  The logits are computed once; only the top-k is recomputed per
step.  This script calls nothing but the fp64 oracle and the seeded input
draws, and writes a plain text table that the input generator reads.

Usage:  python tests/golden/make_zipf_bias.py [--steps 200] [--eta 0.25]
"""
import argparse
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))

import oracle  # noqa: E402
from workloads import WORKLOADS, make_router, make_x, zipf_bias_path, zipf_permutation, \
    zipf_targets  # noqa: E402


def capped_targets(q: np.ndarray, total: float, cap: float) -> np.ndarray:
    """Water-filling: c_e = min(cap, lam * q_e) with sum c_e = total."""
    c = np.zeros_like(q)
    free = np.ones_like(q, dtype=bool)
    remaining = total
    while True:
        lam = remaining / q[free].sum()
        c[free] = lam * q[free]
        over = free & (c > cap)
        if not over.any():
            return c
        c[over] = cap
        free &= ~over
        remaining = total - c[~free].sum()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="skewed_prefill")
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--eta", type=float, default=0.25)
    args = ap.parse_args()
    wl = WORKLOADS[args.workload]

    g0 = torch.Generator().manual_seed(wl.seed)
    make_x(wl, g0)                    # the draw order puts x before W_router
    W_router = make_router(wl, g0)
    g1 = torch.Generator().manual_seed(wl.seed + 1)
    x_cal = make_x(wl, g1)

    logits = oracle.router_logits(x_cal, W_router, None)
    q = zipf_targets(wl.E, wl.zipf_s, zipf_permutation(wl)).numpy()
    target = capped_targets(q, float(wl.T * wl.k), float(wl.T))

    b = np.zeros(wl.E)
    for step in range(args.steps):
        idx, _, _ = oracle.route(logits + b[None, :], wl.k)
        realised = np.bincount(idx.reshape(-1), minlength=wl.E).astype(np.float64)
        err = np.log(target) - np.log(np.maximum(realised, 0.5))
        if step % 20 == 0 or step == args.steps - 1:
            rel = np.abs(realised - target) / target
            print(f"step {step:3d}  max|ln err| {np.abs(err).max():.4f}  "
                  f"median rel err {np.median(rel):.4f}  max count {realised.max():.0f}  "
                  f"min count {realised.min():.0f}")
        b = b + args.eta * err
    b32 = b.astype(np.float32)

    idx, _, _ = oracle.route(logits + b32.astype(np.float64)[None, :], wl.k)
    realised = np.bincount(idx.reshape(-1), minlength=wl.E)
    path = zipf_bias_path(wl)
    with open(path, "w") as f:
        f.write(f"# per-expert router bias for workload '{wl.name}' (E={wl.E}, k={wl.k}, "
                f"d={wl.d}, T={wl.T}, Zipf s={wl.zipf_s}, seed={wl.seed})\n")
        f.write(f"# written by tests/golden/make_zipf_bias.py --steps {args.steps} "
                f"--eta {args.eta} (oracle router on a seed+1 calibration batch)\n")
        f.write(f"# calibration-batch counts: max {realised.max()} min {realised.min()} "
                f"(targets: max {target.max():.1f} min {target.min():.1f})\n")
        for v in b32:
            f.write(f"{float(v):.9g}\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
