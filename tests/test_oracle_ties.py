"""Pins of the oracle's tie bookkeeping, which decides every parity exemption
of the GPU tests: the denoiser's top-two logit gap, the CD's first near-tie
step and smallest relative gap, and the greedy baseline's top-two distance
gap.  Each is checked against a brute force that shares no arithmetic with
the oracle: logits summed term by term in plain Python, CD candidate energies
taken as whole objectives 1/2 |X (w - x)|^2 from the activations X (not from
the gradient h = H (w - x) the oracle carries), greedy targets from the
least-squares optimum of the blocks not yet committed, solved afresh per
block.  The tie rule is the one the MPQ solver's parity statement fixes: a CD
step is a near-tie when its top-two candidate energies differ by less than
tie_rel * |E|, E the row's energy when the step is taken."""
import math

import numpy as np
import pytest

import mpq_inputs as mi
from oracle import mpq_oracle as orc


# ----------------------------------------------------------------------------
# denoiser: top-two logit gap
# ----------------------------------------------------------------------------

def _top_two(values):
    """Largest and second largest of a list by one linear scan."""
    best = second = -math.inf
    for v in values:
        if v > best:
            best, second = v, best
        elif v > second:
            second = v
    return best, second


def _brute_gaps(R1, gamma1, cb, scale, offset, W=None, ga=None):
    m, n = R1.shape
    d = cb.shape[1]
    B = n // d
    out = np.zeros((m, B))
    for i in range(m):
        for b in range(B):
            logits = []
            for c in cb:
                e = math.fsum((float(R1[i, b * d + t]) - (scale[i] * c[t] + offset[i])) ** 2
                              for t in range(d))
                lg = -0.5 * gamma1[i] * e
                if ga is not None:
                    a = math.fsum((float(W[i, b * d + t]) - (scale[i] * c[t] + offset[i])) ** 2
                                  for t in range(d))
                    lg -= 0.5 * ga[i] * a
                logits.append(lg)
            best, second = _top_two(logits)
            out[i, b] = best - second
    return out


@pytest.mark.parametrize("d,anchor", [(1, False), (1, True), (8, False), (8, True)])
def test_denoise_gap_is_the_top_two_logit_difference(d, anchor):
    g = np.random.default_rng(11 + d + 2 * anchor)
    m, n = 3, 16
    if d == 1:
        cb = orc.scalar_levels(8)
        W = g.standard_normal((m, n))
        sc, off = orc.minmax_grid(W, 8)
    else:
        cb = mi.random_small_codebook(5, 24, 8).astype(np.float64)
        W = g.standard_normal((m, n))
        sc, off = orc.rms_scale(W)
    R1 = W + 0.3 * sc[:, None] * g.standard_normal((m, n))
    gamma1 = g.uniform(2.0, 30.0, m) / (sc * sc)
    tau = 0.7 if anchor else math.inf
    ga = 1.0 / (tau * sc) ** 2 if anchor else None
    dn = orc.denoise(R1, gamma1, cb, sc, off, W, tau)
    want = _brute_gaps(R1, gamma1, cb, sc, off, W, ga)
    scale = 1.0 + np.abs(want).max()
    assert np.allclose(dn.gap, want, rtol=0, atol=1e-10 * scale)
    assert np.all(dn.gap >= 0)


def test_denoise_gap_is_zero_at_an_exact_midpoint():
    # r exactly halfway between levels 2 and 3 of a unit grid: equal logits
    cb = orc.scalar_levels(8)
    R1 = np.array([[2.5, 0.25, 6.0, 3.5]])
    dn = orc.denoise(R1, np.array([4.0]), cb, np.array([1.0]), np.array([0.0]))
    assert dn.gap[0, 0] == 0.0 and dn.gap[0, 3] == 0.0
    assert dn.idx[0, 0] == 2 and dn.idx[0, 3] == 3           # lowest index on ties
    # away from a midpoint: gap = gamma/2 ((r - c2)^2 - (r - c1)^2)
    assert np.isclose(dn.gap[0, 1], 2.0 * ((0.25 - 1.0) ** 2 - 0.25 ** 2))
    assert np.isclose(dn.gap[0, 2], 2.0 * 1.0)


# ----------------------------------------------------------------------------
# CD: first near-tie step and the smallest relative gap
# ----------------------------------------------------------------------------

def _energy_x(w, x, X):
    y = X @ (w - x)
    return 0.5 * float(y @ y)


def _brute_cd(w, idx0, cb, scale, offset, X, sweeps, tie_rel):
    """Block CD from candidate energies taken as whole objectives."""
    n = w.size
    d = cb.shape[1]
    B = n // d
    cand = orc.block_candidates(cb, scale, offset, B)
    idx = np.array(idx0, dtype=np.int64)
    x = cand[np.arange(B), idx].reshape(-1).copy()
    first_tie, min_gap, step = -1, math.inf, 0
    changes, gaps = [], []
    for _ in range(sweeps):
        nchg = 0
        for b in range(B):
            E = _energy_x(w, x, X)
            Ec = []
            for k in range(cand.shape[1]):
                y = x.copy()
                y[b * d:(b + 1) * d] = cand[b, k]
                Ec.append(_energy_x(w, y, X))
            Ec = np.asarray(Ec)
            k = int(np.argmin(Ec))
            two = np.sort(Ec)[:2]
            gap = (two[1] - two[0]) / abs(E)
            gaps.append(gap)
            min_gap = min(min_gap, gap)
            if gap < tie_rel and first_tie < 0:
                first_tie = step
            if Ec[k] < E and k != idx[b]:
                x[b * d:(b + 1) * d] = cand[b, k]
                idx[b] = k
                nchg += 1
            step += 1
        changes.append(nchg)
        if nchg == 0:
            break
    return idx, first_tie, min_gap, changes, np.asarray(gaps)


@pytest.mark.parametrize("d", [1, 8])
def test_cd_first_tie_and_min_gap_match_whole_objective_brute_force(d):
    g = np.random.default_rng(40 + d)
    m, n = 3, 16 if d == 1 else 24
    X = mi.heavy_tailed_x(g, g, 40, n)
    W = mi.lognormal_rows_w(g, m, n)
    s, V = orc.spectrum(X)
    H = orc.hessian(s, V)
    if d == 1:
        cb = orc.scalar_levels(8)
        sc, off = orc.minmax_grid(W, 8)
    else:
        cb = mi.random_small_codebook(7, 32, 8).astype(np.float64)
        sc, off = orc.rms_scale(W)
    idx0 = orc.init(W, cb, sc, off).idx_rtn
    X64 = np.asarray(X, np.float64)
    seen_tie = False
    for tie_rel in (1e-5, 1e-3, 1e-2, 1e-1):
        out = orc.cd(W, idx0, cb, sc, off, H, 3, tie_rel=tie_rel)
        for i in range(m):
            idx, ft, mg, chg, gaps = _brute_cd(np.asarray(W[i], np.float64), idx0[i], cb, sc[i],
                                               off[i], X64, 3, tie_rel)
            assert np.array_equal(out.idx[i], idx), (tie_rel, i)
            assert list(out.changes[i, :len(chg)]) == chg
            assert out.first_tie[i] == ft, (tie_rel, i, out.first_tie[i], ft)
            # the gap is relative to the energy before the step, to ~1e-9
            assert math.isclose(out.min_gap_rel[i], mg, rel_tol=1e-7, abs_tol=1e-12), (i, mg)
            # every step's gap, and no gap recorded for steps not taken
            assert np.allclose(out.step_gap[i, :gaps.size], gaps, rtol=1e-7, atol=1e-12)
            assert np.all(np.isinf(out.step_gap[i, gaps.size:]))
            seen_tie |= ft >= 0
    assert seen_tie  # the larger thresholds make the first-tie branch live


def test_cd_planted_exact_tie_is_the_first_tie():
    # diagonal H: blocks decouple; column 5 sits exactly between levels 3 and 4
    # (its current level 3, from round-to-nearest's lowest index), so moving it
    # to 4 changes nothing: a zero gap at step 5.  Every other column sits a
    # quarter step from its level, far from a tie.
    n = 8
    X = np.diag(np.linspace(1.0, 2.0, n))
    s, V = orc.spectrum(X)
    H = orc.hessian(s, V)
    cb = orc.scalar_levels(8)
    w = np.array([[1.25, 2.75, 0.25, 6.25, 4.75, 3.5, 5.25, 1.75]])
    sc, off = np.array([1.0]), np.array([0.0])
    idx0 = orc.init(w, cb, sc, off).idx_rtn
    assert idx0[0, 5] == 3
    out = orc.cd(w, idx0, cb, sc, off, H, 3)
    assert out.first_tie[0] == 5
    assert out.min_gap_rel[0] < 1e-12
    assert np.array_equal(out.idx, idx0) and out.changes[0, 0] == 0
    # an exact tie with the current codeword is not a move
    _, ft, mg, chg, _ = _brute_cd(w[0], idx0[0], cb, 1.0, 0.0, X, 3, 1e-5)
    assert ft == 5 and chg == [0]


# ----------------------------------------------------------------------------
# greedy baseline: top-two distance gap
# ----------------------------------------------------------------------------

def test_ldlq_gap_matches_least_squares_targets():
    g = np.random.default_rng(61)
    m, n = 4, 12
    X = mi.heavy_tailed_x(g, g, 40, n)
    W = mi.lognormal_rows_w(g, m, n)
    s, V = orc.spectrum(X)
    H = orc.hessian(s, V)
    cb = orc.scalar_levels(8)
    sc, off = orc.minmax_grid(W, 8)
    damp = 0.01
    out = orc.ldlq(W, cb, sc, off, H, damp)
    Ht = orc.damped_hessian(H, damp)
    for i in range(m):
        w = np.asarray(W[i], np.float64)
        x = np.zeros(n)
        for b in range(n):
            e_fixed = w[:b] - x[:b]
            e_free = -np.linalg.solve(Ht[b:, b:], Ht[b:, :b] @ e_fixed) if b else np.zeros(n)
            target = w[b] - e_free[0]
            dist = sorted(((target - (sc[i] * k + off[i])) ** 2, k) for k in range(8))
            want = (dist[1][0] - dist[0][0]) / (sc[i] * sc[i])
            assert math.isclose(out.gap[i, b], want, rel_tol=1e-8, abs_tol=1e-10), (i, b)
            x[b] = sc[i] * out.idx[i, b] + off[i]
            assert out.idx[i, b] == dist[0][1] or want < 1e-9
