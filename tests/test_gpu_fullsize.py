"""Full-size parity in the launch configuration bench.py times.

1. Stage parity at the bench's exact shapes: the linear module (both
   tensor-core GEMMs with K = n and K = r, the beta M-step, the extrinsic
   updates) on injected state for every row of the layer, compared with the
   float64 oracle on a seeded sample of rows (rows are independent problems)
   at the per-stage bar: 1e-4 per-row relative l2 and 1e-4 on scalars.

2. The whole solve: the plan is built on the device from X
   (mpq_plan_create_from_x), every row is solved in one mpq_solve, and a
   sample of rows is checked against the oracle (its own spectrum from X).
   A row is compared at the stated bar (exact indices, final energy within
   1e-3) unless the oracle meets a near-tie on it: an argmax whose top-two
   logit gap is below 1e-4, or a CD step whose top-two energy gap is below
   1e-5 |E|.  From such a step on the two trajectories may legitimately part
   (at these sizes the oracle's gaps go down to 1e-9 |E|, far below fp32
   resolution), so for tie-exempt rows only a sanity bound is checked: each
   final energy within 5% of the oracle's, and the mean relative difference
   over the sample within 1% (no systematic bias)."""
import numpy as np
import pytest
import torch

import mpq_inputs as mi
from oracle import mpq_oracle as orc
from tests.helpers import (assert_rows_close, assert_scalars_close, codebook_for, cu, host,
                           idx_np, injected_state)

pytestmark = pytest.mark.gpu

ENERGY_TOL = 1e-3
EXEMPT_ROW_TOL = 5e-2
EXEMPT_MEAN_TOL = 1e-2
_CACHE = {}


def _plan_and_spectrum(name):
    import post_weight_quantization_row_b200 as mpq
    if name not in _CACHE:
        p = mi.make_problem(name)
        X = torch.from_numpy(p.X).cuda()
        plan = mpq.Plan.from_x(X, p.d, p.levels, codebook=p.codebook if p.d == 8 else None)
        del X
        s, V = orc.spectrum(p.X)
        assert s.size == plan.r
        _CACHE[name] = (p, plan, s, V)
    return _CACHE[name]


def _stage_linear(name, sample_rows):
    p, plan, s, V = _plan_and_spectrum(name)
    sc = (orc.minmax_grid(p.W, p.levels)[0] if p.d == 1 else orc.rms_scale(p.W)[0])
    R1, g1, X1, vsum, beta, g0 = injected_state(29, p.W, sc, s)
    out = plan.stage_linear(cu(p.W), cu(R1), cu(g1, torch.float64), cu(X1),
                            cu(vsum, torch.float64), cu(g0, torch.float64), cu(beta, torch.float64))
    rows = np.sort(np.random.default_rng(3).choice(p.m_out, sample_rows, replace=False))
    ref = orc.linear_step(p.W[rows], R1[rows], g1[rows], X1[rows], vsum[rows], beta[rows], s, V,
                          g0[rows])
    assert np.all(ref.clamps == 0)
    # the two sides take eigenvectors from different eigensolvers (device
    # Jacobi vs LAPACK), so singular vectors may differ in sign: compare only
    # quantities that do not depend on the basis (not U' = D u)
    assert_rows_close("r2", host(out["R2"])[rows], ref.R2)
    assert_rows_close("xhat2", host(out["xhat2"])[rows], ref.xhat2)
    assert_scalars_close("alpha2", host(out["alpha2"])[rows], ref.alpha2)
    assert_scalars_close("beta_hat", host(out["beta_hat"])[rows], ref.beta_hat)
    assert_scalars_close("gamma1'", host(out["gamma1"])[rows], ref.gamma1)
    assert_rows_close("r1'", host(out["R1"])[rows], ref.R1)


def _solve(name, sample_rows, seed=7):
    p, plan, s, V = _plan_and_spectrum(name)
    out = plan.solve(torch.from_numpy(p.W).cuda(), p.T_vamp, p.cd_sweeps, stats=True)
    e_gpu = host(out["energy"]).astype(np.float64)
    rows = np.sort(np.random.default_rng(seed).choice(p.m_out, sample_rows, replace=False))
    cb = codebook_for(p)
    ref = orc.solve(p.W[rows], cb, s, V, p.T_vamp, p.cd_sweeps)
    rel = np.abs(e_gpu[rows] - ref.energy) / ref.energy
    clean = np.all(ref.map_gap > 1e-4, axis=1) & (ref.cd.first_tie < 0)
    got = idx_np(out["idx"])[rows]
    if clean.any():
        assert np.array_equal(got[clean], ref.idx[clean])
        assert rel[clean].max() <= ENERGY_TOL
    assert rel.max() <= EXEMPT_ROW_TOL, (rows, e_gpu[rows], ref.energy)
    assert np.mean((e_gpu[rows] - ref.energy) / ref.energy) <= EXEMPT_MEAN_TOL
    # the outputs agree with each other on the device
    wh = host(out["w_hat"])[rows]
    sc, off = (orc.minmax_grid(p.W[rows], p.levels) if p.d == 1 else orc.rms_scale(p.W[rows]))
    dec = orc.decode(got, cb, sc, off)
    assert np.allclose(wh, dec, rtol=1e-5, atol=1e-6 * np.abs(dec).max())
    # the device energy of w_hat agrees with the oracle's energy of the same
    # w_hat at the final-energy bar (with r < n most of the residual lies in
    # the null space, so its projection carries ~1e-4 fp32 relative error)
    e_direct = orc.energy(p.W[rows], wh, s, V)
    assert np.all(np.abs(e_direct - e_gpu[rows]) <= ENERGY_TOL * e_direct)
    # the solve beats round-to-nearest on the sample
    st = orc.init(p.W[rows], cb)
    e_rtn = orc.energy(p.W[rows], orc.decode(st.idx_rtn, cb, st.scale, st.offset), s, V)
    assert e_gpu[rows].sum() < e_rtn.sum()


def test_fullsize_stage_linear_q4096():
    _stage_linear("q4096", 16)


def test_fullsize_stage_linear_down_rank_space():
    _stage_linear("down", 8)


def test_fullsize_solve_l1b():
    _solve("l1b", 8)


def test_fullsize_solve_q4096():
    _solve("q4096", 4)


def test_fullsize_solve_down_rank_space():
    _solve("down", 3)
    assert _CACHE["down"][1].r == 4096 and _CACHE["down"][1].n == 14336


def test_fullsize_solve_e8_lattice():
    _solve("e8t8", 1)
