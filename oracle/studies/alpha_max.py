"""Oracle-only study of reading R5: where the extrinsic updates clip the mean
divergence alpha at alpha_max.  TEST INFRASTRUCTURE ONLY (it runs the oracle
and nothing else; no value here comes from the CUDA library).

The pages write the extrinsic updates in the eta form (MPQ note, key design
1): gamma2 = eta1 - gamma1, r2 = (eta1 xhat1 - gamma1 r1) / gamma2.  With
alpha1 = gamma1 * sum_b tr(Sigma_1b) / n this is r2 = (xhat1 - alpha1 r1) /
(1 - alpha1) and gamma2 = gamma1 (1 - alpha1) / alpha1, which the pages leave
undefined at alpha1 >= 1 and which extrapolates by 1 / (1 - alpha1) as alpha1
approaches 1.  At the first iteration alpha1 is close to 1 by construction
(gamma1_0 = 1 / MSE of round-to-nearest, cavity r1 = w: the denoiser's
posterior variance is about the quantisation noise 1 / gamma1_0).

For each workload recipe (small, seeded, the generators of the bench
workloads) and for the anchored (tau = 0.2) and unanchored prior, the script
solves every row with the oracle for several values of alpha_max, the largest
(1 - 1e-9) being the eta form wherever alpha < 1, and prints the mean final
objective 1/2 |X (w - w_hat)|^2 divided by that of round-to-nearest + the
same CD, with the fraction of VAMP steps whose alpha reached 0.99.  Run:  python -m oracle.studies.alpha_max > oracle/studies/alpha_max.txt
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

import mpq_inputs as mi  # noqa: E402
from oracle import mpq_oracle as orc  # noqa: E402

ALPHAS = (0.9, 0.99, 0.999, 1 - 1e-5, 1 - 1e-9)


def recipes():
    """(name, W, X, codebook, T_vamp) for each workload recipe, small."""
    out = []
    p = mi.make_problem("tiny")
    out.append(("tiny: AR(0.7) Gaussian X 256x64, 3-bit, T=8", p.W, p.X, orc.scalar_levels(8), 8))
    for L, bits in ((8, 3), (16, 4)):
        g = np.random.default_rng(500 + L)
        X = mi.heavy_tailed_x(g, g, 512, 256)
        W = mi.lognormal_rows_w(g, 32, 256)
        out.append((f"bench recipe X 512x256 (t5, AR 0.5, outliers), {bits}-bit, T=16", W, X,
                    orc.scalar_levels(L), 16))
    g = np.random.default_rng(503)
    X = mi.heavy_tailed_x(g, g, 128, 512)
    W = mi.lognormal_rows_w(g, 16, 512)
    out.append(("rank-deficient X 128x512 (r = 128 < n), 3-bit, T=16", W, X, orc.scalar_levels(8), 16))
    g = np.random.default_rng(504)
    X = mi.gaussian_ar1_x(g, 512, 256, 0.9)
    W = mi.lognormal_rows_w(g, 32, 256)
    out.append(("AR(0.9) Gaussian X 512x256, 4-bit, T=16", W, X, orc.scalar_levels(16), 16))
    g = np.random.default_rng(505)
    X = mi.heavy_tailed_x(g, g, 256, 128)
    W = mi.lognormal_rows_w(g, 16, 128)
    signs = np.where(g.random(128) < 0.5, -1.0, 1.0)
    X = mi.random_hadamard_apply(X, signs)
    W = mi.random_hadamard_apply(W, signs)
    cb = mi.e8_codebook_cached()[:4096].astype(np.float64)
    out.append(("E8 (first 4096 codewords) after RHT, X 256x128, T=8", W, X, cb, 8))
    return out


def clip_fraction(W, cb, s, V, T, tau):
    """Fraction of extrinsic steps (both directions) whose alpha reaches 0.99."""
    st = orc.init(W, cb)
    g10 = st.gamma1.copy()
    R1, g1, beta = st.R1, st.gamma1.copy(), st.beta.copy()
    hit = tot = 0
    n = W.shape[1]
    for _ in range(T):
        dn = orc.denoise(R1, g1, cb, st.scale, st.offset, W, tau)
        a1 = g1 * dn.vsum / n
        lo = orc.linear_step(W, R1, g1, dn.xhat, dn.vsum, beta, s, V, g10)
        hit += int((a1 >= 0.99).sum() + (lo.alpha2 >= 0.99).sum())
        tot += 2 * W.shape[0]
        R1, g1, beta = lo.R1, lo.gamma1, lo.beta
    return hit / tot


def main():
    keep = orc.ALPHA_MAX
    t0 = time.time()
    cases = [(name, W, X, cb, T, orc.spectrum(X)) for name, W, X, cb, T in recipes()]
    try:
        for tau in (orc.TAU, math.inf):
            print(f"# reading R5 at tau = {tau:g}: final objective of MPQ + CD3 / that of "
                  "round-to-nearest + CD3 (mean over rows; lower is better)")
            print("# columns: alpha_max; 'clip' = share of extrinsic steps with alpha >= 0.99")
            print("| workload | " + " | ".join(f"{a:.9g}" for a in ALPHAS) + " | clip |")
            print("|---|" + "---|" * (len(ALPHAS) + 1))
            for name, W, X, cb, T, (s, V) in cases:
                W = np.asarray(W, np.float64)
                rtn = orc.solve(W, cb, s, V, 0, 3).energy.mean()
                vals = []
                for a in ALPHAS:
                    orc.ALPHA_MAX = a
                    vals.append(orc.solve(W, cb, s, V, T, 3, tau=tau).energy.mean() / rtn)
                orc.ALPHA_MAX = 0.99
                frac = clip_fraction(W, cb, s, V, T, tau)
                print(f"| {name} | " + " | ".join(f"{v:.4f}" for v in vals) + f" | {frac:.2f} |",
                      flush=True)
            print()
    finally:
        orc.ALPHA_MAX = keep
    print(f"# {time.time() - t0:.0f} s")


if __name__ == "__main__":
    main()
