"""Oracle-only study of reading R4: the prior anchor's scale tau.  TEST
INFRASTRUCTURE ONLY (it runs the oracle and nothing else).

The MPQ note's hyper-parameter section fixes an anchor scale tau = 0.2 next to
T_vamp = 16 and rho_damp = 0.5, and key design 1 runs the denoiser "under the
prior anchor"; the ai.info summary calls the theory's tau -> inf limit
unanchored.  The pages give no formula for the anchor.  Reading R4: the
anchor pins each block to its own weights w_b with a width of tau codebook
units (grid steps of a scalar grid, lattice units of the E8 codebook), i.e.
log rho_b(c) = -|c - w_b|^2 / (2 tau^2 scale_b^2).

For each workload recipe (small, seeded, the generators of the bench
workloads) the script prints the mean final objective 1/2 |X (w - w_hat)|^2
of MPQ + CD3 for several tau, and of the greedy baseline (LDLQ) + CD3, each
divided by that of round-to-nearest + CD3.
Run:  python -m oracle.studies.anchor > oracle/studies/anchor.txt
"""
from __future__ import annotations

import math
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from oracle import mpq_oracle as orc  # noqa: E402
from oracle.studies.alpha_max import recipes  # noqa: E402

TAUS = (math.inf, 0.1, 0.2, 0.3, 0.5, 1.0)


def main():
    t0 = time.time()
    print("# reading R4: final objective / that of round-to-nearest + CD3 (mean over rows; "
          "lower is better); tau in codebook units")
    print("| workload | LDLQ + CD3 | " + " | ".join(f"MPQ tau={t:g}" for t in TAUS) + " |")
    print("|---|---|" + "---|" * len(TAUS))
    for name, W, X, cb, T in recipes():
        s, V = orc.spectrum(X)
        W = np.asarray(W, np.float64)
        rtn = orc.solve(W, cb, s, V, 0, 3).energy.mean()
        ld = orc.solve(W, cb, s, V, 0, 3, greedy_damp=0.01).energy.mean() / rtn
        vals = [orc.solve(W, cb, s, V, T, 3, tau=t).energy.mean() / rtn for t in TAUS]
        print(f"| {name} | {ld:.4f} | " + " | ".join(f"{v:.4f}" for v in vals) + " |", flush=True)
    print(f"# {time.time() - t0:.0f} s")


if __name__ == "__main__":
    main()
