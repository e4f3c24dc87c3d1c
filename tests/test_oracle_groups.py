"""Pins of the oracle's group-wise scalar grids (one min-max grid per group of
consecutive columns of a row; the MPQ note's experimental setup quantises
scalar weights with group 128).  Each pin fixes the grouped mode by something
other than itself: the per-row formula applied group by group, a 50-digit
brute-force posterior over each element's own grid, exact agreement with the
per-row mode when every group shares the row's grid, and a brute-force
local-optimum check of the converged CD."""
import numpy as np
import pytest

import mpq_inputs as mi
from oracle import mpq_oracle as orc
from tests.test_oracle_pins import _mp_posterior


def test_minmax_grid_per_group_is_the_row_formula_per_group():
    g = np.random.default_rng(31)
    W = g.normal(0, 1, size=(3, 12))
    W[1, 4:8] = 0.7                      # a constant group
    sc, off = orc.minmax_grid(W, 8, group=4)
    assert sc.shape == (3, 3) and off.shape == (3, 3)
    rs, ro = orc.minmax_grid(W.reshape(9, 4), 8)
    assert np.array_equal(sc.reshape(-1), rs) and np.array_equal(off.reshape(-1), ro)
    # a group whose range contains zero (the zero point is not clipped) is
    # covered by its grid to half a step
    covered = 0
    for i in range(3):
        for k in range(3):
            w = W[i, 4 * k:4 * k + 4]
            if not (w.min() <= 0.0 <= w.max()):
                continue
            covered += 1
            lv = sc[i, k] * np.arange(8) + off[i, k]
            assert np.all(np.min(np.abs(w[:, None] - lv[None, :]), axis=1) <= 0.5 * sc[i, k] + 1e-12)
    assert covered >= 3


def test_denoiser_groups_vs_50_digit_brute_force():
    g = np.random.default_rng(32)
    L = 8
    cb = orc.scalar_levels(L)
    R1 = g.normal(0, 1.2, size=(2, 8))
    gam = np.array([1.5, 20.0])
    sc = np.array([[0.4, 0.25], [0.3, 0.5]])
    off = np.array([[-1.4, -0.8], [-1.0, -1.7]])
    out = orc.denoise(R1, gam, cb, sc, off)
    for i in range(2):
        for j in range(8):
            cand = orc.row_candidates(cb, sc[i, j // 4], off[i, j // 4])
            mean, var = _mp_posterior([R1[i, j]], gam[i], cand)
            assert abs(out.xhat[i, j] - mean[0]) <= 1e-12 * (1 + abs(mean[0]))
            assert abs(out.vblock[i, j] - var) <= 1e-12 * max(var, 1e-300) + 1e-300


def test_groups_sharing_the_row_grid_reproduce_the_per_row_mode():
    p = mi.make_problem("tiny")
    cb = orc.scalar_levels(p.levels)
    s, V = orc.spectrum(p.X)
    H = orc.hessian(s, V)
    sc, off = orc.minmax_grid(p.W, p.levels)
    ng = p.n // 16
    scg, offg = np.repeat(sc[:, None], ng, axis=1), np.repeat(off[:, None], ng, axis=1)
    a, b = orc.init(p.W, cb, sc, off), orc.init(p.W, cb, scg, offg)
    assert np.array_equal(a.idx_rtn, b.idx_rtn) and np.array_equal(a.gamma1, b.gamma1)
    R1 = p.W + 0.05
    da, db = orc.denoise(R1, a.gamma1, cb, sc, off), orc.denoise(R1, a.gamma1, cb, scg, offg)
    assert np.array_equal(da.xhat, db.xhat) and np.array_equal(da.vblock, db.vblock)
    ca = orc.cd(p.W, a.idx_rtn, cb, sc, off, H, 3)
    cg = orc.cd(p.W, a.idx_rtn, cb, scg, offg, H, 3)
    assert np.array_equal(ca.idx, cg.idx) and np.array_equal(ca.x, cg.x)


def test_cd_groups_converge_to_a_brute_force_local_optimum():
    p = mi.make_problem("tiny")
    cb = orc.scalar_levels(p.levels)
    s, V = orc.spectrum(p.X)
    H = orc.hessian(s, V)
    st = orc.init(p.W, cb, group=16)
    assert st.scale.shape == (p.m_out, p.n // 16)
    E_prev = orc.energy_direct(p.W, orc.decode(st.idx_rtn, cb, st.scale, st.offset), p.X)
    idx = st.idx_rtn
    for _ in range(3):
        out = orc.cd(p.W, idx, cb, st.scale, st.offset, H, 1)
        E = orc.energy_direct(p.W, orc.decode(out.idx, cb, st.scale, st.offset), p.X)
        assert np.all(E <= E_prev * (1 + 1e-12))
        idx, E_prev = out.idx, E
    full = orc.cd(p.W, st.idx_rtn, cb, st.scale, st.offset, H, 60)
    assert np.all(full.changes[np.arange(p.m_out), full.sweeps_run - 1] == 0)
    for i in range(4):
        x = full.x[i]
        E0 = orc.energy_direct(p.W[i:i + 1], x[None], p.X)[0]
        for j in range(p.n):
            for c in orc.row_candidates(cb, st.scale[i, j // 16], st.offset[i, j // 16])[:, 0]:
                y = x.copy()
                y[j] = c
                assert orc.energy_direct(p.W[i:i + 1], y[None], p.X)[0] >= E0 - 1e-9 * E0


def test_grouped_solve_runs_and_beats_round_to_nearest():
    p = mi.make_problem("tiny")
    cb = orc.scalar_levels(p.levels)
    s, V = orc.spectrum(p.X)
    out = orc.solve(p.W, cb, s, V, 4, 3, group=16)
    st = orc.init(p.W, cb, group=16)
    e_rtn = orc.energy(p.W, orc.decode(st.idx_rtn, cb, st.scale, st.offset), s, V)
    assert out.energy.sum() < e_rtn.sum()
    # the grouped grid fits the row better than one grid for the whole row
    per_row = orc.solve(p.W, cb, s, V, 4, 3)
    assert out.energy.sum() < per_row.energy.sum()


# ----------------------------------------------------------------------------
# adaptive CD: rows above a terminal precision keep the marginal MAP
# ----------------------------------------------------------------------------

def test_cd_skip_precision_extremes():
    p = mi.make_problem("tiny")
    cb = orc.scalar_levels(p.levels)
    s, V = orc.spectrum(p.X)
    full = orc.solve(p.W, cb, s, V, 4, 3)
    prec = orc.terminal_precision(full.gamma1, orc.init(p.W, cb).scale)
    # a threshold above every row's precision changes nothing
    hi = orc.solve(p.W, cb, s, V, 4, 3, cd_skip_precision=2 * prec.max())
    assert np.array_equal(hi.idx, full.idx) and np.array_equal(hi.energy, full.energy)
    # below every row's precision: no CD at all, the marginal MAP is the answer
    lo = orc.solve(p.W, cb, s, V, 4, 3, cd_skip_precision=0.5 * prec.min())
    none = orc.solve(p.W, cb, s, V, 4, 0)
    assert np.array_equal(lo.idx, none.idx) and np.array_equal(lo.energy, none.energy)
    assert np.all(lo.cd.changes == 0)
    # in between: each row follows its own precision
    mid = float(np.median(prec))
    mix = orc.solve(p.W, cb, s, V, 4, 3, cd_skip_precision=mid)
    skip = prec > mid
    assert 0 < skip.sum() < p.m_out
    assert np.array_equal(mix.idx[skip], none.idx[skip])
    assert np.array_equal(mix.idx[~skip], full.idx[~skip])
