"""Group-wise scalar grids (mpq_params.group_size = 128: one min-max grid per
group of 128 consecutive columns of a row, the MPQ note's experimental
setting) against the oracle on identical inputs: init exactly, the denoiser
at the stage bar in every precision regime, CD indices exactly outside ties
(with several panels, so that Delta carries the group scales through the
panel GEMM), and the whole solve."""
import math

import numpy as np
import pytest
import torch

import mpq_inputs as mi
from oracle import mpq_oracle as orc
from tests.helpers import (assert_vec_close, ENERGY_TOL, assert_rows_close, assert_scalars_close, cu, host, idx_np,
                           injected_state, spectrum_cuda)

pytestmark = pytest.mark.gpu

G = 128
LOGIT_TIE = 1e-3


@pytest.fixture(scope="module")
def mpq():
    import post_weight_quantization_row_b200 as m
    return m


def case(seed, m_out=20, n=640, m=900, L=8):
    return mi.small_problem(seed, m_out, n, m, d=1, levels=L, T_vamp=4, cd_sweeps=3)


def plan_for(mpq, p, **kw):
    _, _, s_cu, V_cu = spectrum_cuda(p.X)
    return mpq.Plan.from_spectrum(s_cu, V_cu, 1, p.levels, group_size=G, **kw)


def grid_f32(p):
    sc, off = orc.minmax_grid(p.W, p.levels, G)
    return sc.astype(np.float32), off.astype(np.float32)


def test_init_grouped_grid(mpq):
    p = case(801)
    plan = plan_for(mpq, p)
    out = plan.stage_init(cu(p.W))
    sc, off = grid_f32(p)
    assert host(out["scale"]).shape == (p.m_out, p.n // G)
    assert np.array_equal(host(out["scale"]), sc)
    assert np.array_equal(host(out["offset"]), off)
    cb = orc.scalar_levels(p.levels)
    st = orc.init(p.W, cb, sc.astype(np.float64), off.astype(np.float64))
    t = (p.W - np.repeat(off, G, axis=1)) / np.repeat(sc, G, axis=1)
    tie = np.abs(t - np.floor(t) - 0.5) < 1e-5
    assert np.array_equal(idx_np(out["idx"])[~tie], st.idx_rtn[~tie])
    assert_scalars_close("gamma1_0", host(out["gamma1_0"]), st.gamma1, 1e-5)


@pytest.mark.parametrize("g_lo,g_hi,tau", [(1.0, 40.0, math.inf), (0.05, 0.5, math.inf),
                                           (100.0, 1e4, math.inf), (1.0, 40.0, 0.2),
                                           (0.05, 0.5, 0.2)])
def test_denoise_grouped(mpq, g_lo, g_hi, tau):
    # with the anchor, each group's anchor is tau steps of its own grid
    p = case(802)
    plan = plan_for(mpq, p, tau=tau)
    sc, off = grid_f32(p)
    s, _ = orc.spectrum(p.X)
    # the precision is per row; the groups' scales make gamma1 s^2 (and with
    # it the precision regime) differ from group to group
    R1, g1, _, _, _, _ = injected_state(11, p.W, sc.mean(axis=1), s, g_lo, g_hi)
    ref = orc.denoise(R1, g1, orc.scalar_levels(p.levels), sc.astype(np.float64),
                      off.astype(np.float64), p.W, tau)
    out = plan.stage_denoise(cu(R1), cu(g1, torch.float64), cu(sc), cu(off),
                             cu(p.W) if math.isfinite(tau) else None)
    assert_vec_close("xhat1", host(out["xhat"]), ref.xhat)
    assert_vec_close("vblock", host(out["vblock"]), ref.vblock)
    assert_scalars_close("vsum", host(out["vsum"]), ref.vsum)
    ok = ref.gap > LOGIT_TIE
    assert np.array_equal(idx_np(out["idx"])[ok], ref.idx[ok])


def test_cd_grouped_several_panels(mpq):
    p = case(803, m_out=24, n=512, m=700)
    plan = plan_for(mpq, p, cd_panel=256)
    sc, off = grid_f32(p)
    cb = orc.scalar_levels(p.levels)
    s, V = orc.spectrum(p.X)
    st = orc.init(p.W, cb, sc.astype(np.float64), off.astype(np.float64))
    ref = orc.cd(p.W, st.idx_rtn, cb, sc.astype(np.float64), off.astype(np.float64),
                 orc.hessian(s, V), 3)
    out = plan.stage_cd(cu(p.W), cu(sc), cu(off),
                        cu(st.idx_rtn.astype(np.uint16).view(np.int16), torch.int16), 3)
    got = idx_np(out["idx"])
    clean = ref.first_tie < 0
    assert clean.mean() >= 0.25
    assert np.array_equal(got[clean], ref.idx[clean])
    assert np.array_equal(host(out["changes"])[clean], ref.changes[clean])
    assert (ref.changes[clean, 1] > 0).any()
    e_gpu = orc.energy(p.W, orc.decode(got, cb, sc.astype(np.float64), off.astype(np.float64)), s, V)
    e_ref = orc.energy(p.W, ref.x, s, V)
    assert np.all(np.abs(e_gpu - e_ref) <= ENERGY_TOL * e_ref)


def test_solve_grouped(mpq):
    p = case(804, m_out=24, n=384, m=600)
    plan = plan_for(mpq, p)
    sc, off = grid_f32(p)
    cb = orc.scalar_levels(p.levels)
    s, V = orc.spectrum(p.X)
    ref = orc.solve(p.W, cb, s, V, p.T_vamp, p.cd_sweeps, sc.astype(np.float64),
                    off.astype(np.float64))
    out = plan.solve(cu(p.W), p.T_vamp, p.cd_sweeps, row_scale=cu(sc), row_offset=cu(off),
                     stats=True)
    got = idx_np(out["idx"])
    e_gpu = host(out["energy"]).astype(np.float64)
    clean = np.all(ref.map_gap > 1e-4, axis=1) & (ref.cd.first_tie < 0)
    assert clean.mean() >= 0.25
    assert np.array_equal(got[clean], ref.idx[clean])
    assert np.all(np.abs(e_gpu[clean] - ref.energy[clean]) <= ENERGY_TOL * ref.energy[clean])
    assert abs(e_gpu.sum() - ref.energy.sum()) <= ENERGY_TOL * ref.energy.sum()
    # the library's own grid (no row_scale given) is the same grid
    own = plan.solve(cu(p.W), p.T_vamp, p.cd_sweeps)
    assert abs(host(own["energy"]).astype(np.float64).sum() - e_gpu.sum()) <= ENERGY_TOL * e_gpu.sum()
    # and group-wise grids fit the rows better than one grid per row
    per_row = orc.solve(p.W, cb, s, V, p.T_vamp, p.cd_sweeps)
    assert e_gpu.sum() < per_row.energy.sum()


# ------------------------------------------------------------- adaptive CD ---

@pytest.mark.parametrize("group", [0, G])
def test_adaptive_cd_rows_follow_their_terminal_precision(mpq, group):
    # rows whose terminal precision gamma1 s^2 exceeds the threshold keep the
    # marginal MAP (as a solve without CD), the others run the full CD (as a
    # solve without the threshold); the device decides from its own terminal
    # gamma1, the oracle's decisions agree away from the threshold
    p = case(805, m_out=32, n=384, m=600)
    _, _, s_cu, V_cu = spectrum_cuda(p.X)
    plans = {k: mpq.Plan.from_spectrum(s_cu, V_cu, 1, p.levels, group_size=group, **kw)
             for k, kw in (("full", {}), ("skip", {"cd_skip_precision": 1.0}))}
    W = cu(p.W)
    full = plans["full"].solve(W, p.T_vamp, p.cd_sweeps, stats=True)
    none = plans["full"].solve(W, p.T_vamp, 0, stats=True)
    sc = host(plans["full"].stage_init(W)["scale"]).astype(np.float64)
    smax = sc if sc.ndim == 1 else sc.max(axis=1)
    prec = host(full["gamma1"]) * smax * smax
    thr = float(np.median(prec))
    pl = mpq.Plan.from_spectrum(s_cu, V_cu, 1, p.levels, group_size=group, cd_skip_precision=thr)
    mix = pl.solve(W, p.T_vamp, p.cd_sweeps, stats=True)
    skip = prec > thr
    assert 0 < skip.sum() < p.m_out
    got, g_full, g_none = idx_np(mix["idx"]), idx_np(full["idx"]), idx_np(none["idx"])
    assert np.array_equal(got[skip], g_none[skip])
    assert np.array_equal(got[~skip], g_full[~skip])
    assert np.all(host(mix["cd_changes"])[skip] == 0)
    # the oracle's decisions on the same threshold, away from it
    cb = orc.scalar_levels(p.levels)
    s, V = orc.spectrum(p.X)
    ref = orc.solve(p.W, cb, s, V, p.T_vamp, p.cd_sweeps, group=group, cd_skip_precision=thr)
    st = orc.init(p.W, cb, group=group)
    prec_ref = orc.terminal_precision(ref.gamma1, st.scale)
    far = np.abs(prec_ref / thr - 1.0) > 0.05
    assert np.array_equal((prec_ref > thr)[far], skip[far])
