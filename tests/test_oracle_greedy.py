"""Pins of the oracle's greedy baseline (LDLQ / GPTQ) against things other
than itself: its definition solved afresh per block (least-squares optimum of
the blocks not yet committed, by a linear solve), the diagonal-H case where it
is round-to-nearest, and a two-column closed form."""
import numpy as np
import pytest

import mpq_inputs as mi
from oracle import mpq_oracle as orc


def case(seed, m, n, m_calib, d=1, L=8, group=0, K=64):
    g = np.random.default_rng(seed)
    X = mi.heavy_tailed_x(g, g, m_calib, n)
    W = mi.lognormal_rows_w(g, m, n)
    s, V = orc.spectrum(X)
    H = orc.hessian(s, V)
    if d == 1:
        cb = orc.scalar_levels(L)
        sc, off = orc.minmax_grid(W, L, group)
    else:
        cb = mi.e8_codebook_cached()[:K].astype(np.float64)
        sc, off = orc.rms_scale(W)
    return W, cb, sc, off, H, s, V


@pytest.mark.parametrize("seed,m_calib,damp,group", [
    (1, 40, 0.01, 0), (2, 40, 0.1, 0), (3, 6, 0.01, 0), (4, 40, 0.01, 4), (5, 40, 1e-6, 0)])
def test_ldlq_equals_its_definition_scalar(seed, m_calib, damp, group):
    W, cb, sc, off, H, _, _ = case(seed, 6, 12, m_calib, group=group)
    g = orc.ldlq(W, cb, sc, off, H, damp)
    Ht = orc.damped_hessian(H, damp)
    clean = np.all(g.gap > 1e-9, axis=1)
    assert clean.sum() >= 5
    for i in np.flatnonzero(clean):
        assert np.array_equal(g.idx[i], orc.greedy_conditional(W[i], cb, sc[i], off[i], Ht)), i


def test_ldlq_equals_its_definition_e8():
    W, cb, sc, off, H, _, _ = case(6, 4, 24, 60, d=8, K=64)
    g = orc.ldlq(W, cb, sc, off, H, 0.01)
    Ht = orc.damped_hessian(H, 0.01)
    for i in range(W.shape[0]):
        assert np.array_equal(g.idx[i], orc.greedy_conditional(W[i], cb, sc[i], off[i], Ht))


@pytest.mark.parametrize("d", [1, 8])
def test_ldlq_on_a_diagonal_hessian_is_round_to_nearest(d):
    W, cb, sc, off, _, _, _ = case(7, 5, 32, 50, d=d)
    H = np.diag(np.random.default_rng(8).uniform(0.5, 3.0, W.shape[1]))
    g = orc.ldlq(W, cb, sc, off, H, 0.05)
    assert np.array_equal(g.idx, orc.init(W, cb, sc, off).idx_rtn)


def test_ldlq_two_columns_closed_form():
    # n = 2: q1 = RTN(w1); q2 = RTN(w2 + (w1 - q1) H12 / H22)
    # (the optimum of column 2 given column 1, from d/de2 e^T H e = 0)
    g = np.random.default_rng(9)
    cb = orc.scalar_levels(16)
    for _ in range(50):
        w = g.standard_normal((1, 2))
        A = g.standard_normal((2, 2))
        H = A @ A.T + 0.1 * np.eye(2)
        sc, off = np.array([0.3]), np.array([-2.0])
        got = orc.ldlq(w, cb, sc, off, H, 0.0).idx[0]
        rtn = lambda v: int(np.clip(np.floor((v - off[0]) / sc[0] + 0.5), 0, 15))
        q1 = rtn(w[0, 0])
        x1 = sc[0] * q1 + off[0]
        q2 = rtn(w[0, 1] + (w[0, 0] - x1) * H[0, 1] / H[1, 1])
        assert got.tolist() == [q1, q2]


def test_solve_with_greedy_init():
    W, cb, sc, off, H, s, V = case(10, 5, 16, 40)
    g = orc.ldlq(W, cb, sc, off, H, 0.01)
    out = orc.solve(W, cb, s, V, 0, 0, sc, off, greedy_damp=0.01)
    assert np.array_equal(out.idx, g.idx) and np.array_equal(out.idx_map, g.idx)
    assert np.allclose(out.energy, orc.energy(W, orc.decode(g.idx, cb, sc, off), s, V))
    # CD after the greedy init never raises the energy of a row
    out3 = orc.solve(W, cb, s, V, 0, 3, sc, off, greedy_damp=0.01)
    assert np.all(out3.energy <= out.energy * (1 + 1e-12))
    # without greedy_damp, T_vamp = 0 stays round-to-nearest
    rtn = orc.solve(W, cb, s, V, 0, 0, sc, off)
    assert np.array_equal(rtn.idx, orc.init(W, cb, sc, off).idx_rtn)


def test_input_recipe_rotation_is_the_sylvester_hadamard():
    # the e8 / e8t8 inputs rotate W and X by Q = H_n diag(signs) / sqrt(n);
    # the generator's fast transform must equal the dense Sylvester matrix and
    # leave the objective's Gram spectrum unchanged
    import math
    import scipy.linalg
    g = np.random.default_rng(21)
    for n in (1, 2, 8, 64, 256):
        a = g.standard_normal((5, n))
        signs = np.where(g.random(n) < 0.5, -1.0, 1.0)
        dense = a @ (signs[:, None] * scipy.linalg.hadamard(n)) / math.sqrt(n)
        assert np.allclose(mi.random_hadamard_apply(a, signs), dense, rtol=1e-12, atol=1e-12)
    X = g.standard_normal((40, 64))
    signs = np.where(g.random(64) < 0.5, -1.0, 1.0)
    Xr = mi.random_hadamard_apply(X, signs)
    assert np.allclose(np.linalg.svd(X, compute_uv=False), np.linalg.svd(Xr, compute_uv=False))
