"""Shared helpers for the parity tests: comparisons and injected states."""
from __future__ import annotations

import numpy as np
import torch

import mpq_inputs as mi
from oracle import mpq_oracle as orc

VEC_TOL = 1e-4      # per-row relative l2 for vector outputs (fp32 vs fp64)
SCAL_TOL = 1e-4     # relative for per-row scalars
ENERGY_TOL = 1e-3   # final energies


def cu(x, dtype=torch.float32):
    return torch.as_tensor(np.ascontiguousarray(x)).to(dtype=dtype, device="cuda").contiguous()


def host(t):
    return t.detach().cpu().numpy()


def row_rel_l2(gpu: np.ndarray, ref: np.ndarray) -> np.ndarray:
    gpu = np.asarray(gpu, np.float64).reshape(ref.shape[0], -1)
    ref = np.asarray(ref, np.float64).reshape(ref.shape[0], -1)
    num = np.linalg.norm(gpu - ref, axis=1)
    den = np.maximum(np.linalg.norm(ref, axis=1), 1e-300)
    return num / den


def assert_rows_close(name, gpu, ref, tol=VEC_TOL, rows=None):
    err = row_rel_l2(gpu, ref)
    if rows is not None:
        err = err[rows]
    worst = float(err.max()) if err.size else 0.0
    assert worst <= tol, f"{name}: worst per-row relative l2 {worst:.3e} > {tol:.0e}"
    return worst


ELEM_FLOOR = 2.0 ** -18   # 16 x 2^-22 of the row norm: fp32 rounding of a row, with headroom


def assert_elems_close(name, gpu, ref, tol=VEC_TOL, rows=None):
    """Element-wise companion of assert_rows_close: every element within
    tol * |ref| + 2^-18 * |ref row|_2.  The floor is what fp32 (and the
    22-significand-bit tensor-core contractions) can promise an element that
    is small next to its row: its absolute error carries the rounding of the
    row's larger terms, a few 2^-22 times the row norm (a posterior mean
    formed as scale * level + offset near zero; a GEMM output summing up to
    n = 14336 products, measured at up to 8 x 2^-22); the floor gives 16 x.
    It is 1/26 of what the per-row l2 bound lets a single element be off, so
    one bad element cannot hide behind larger ones."""
    gpu = np.asarray(gpu, np.float64).reshape(ref.shape[0], -1)
    ref = np.asarray(ref, np.float64).reshape(ref.shape[0], -1)
    if rows is not None:
        gpu, ref = gpu[rows], ref[rows]
    norm = np.linalg.norm(ref, axis=1, keepdims=True)
    bound = tol * np.abs(ref) + ELEM_FLOOR * norm
    excess = np.abs(gpu - ref) / np.maximum(bound, 1e-300)
    worst = float(excess.max()) if excess.size else 0.0
    if worst > 1.0:
        i, j = np.unravel_index(np.argmax(excess), excess.shape)
        raise AssertionError(f"{name}: element ({i}, {j}) {gpu[i, j]:.9g} vs {ref[i, j]:.9g} "
                             f"(row l2 {norm[i, 0]:.3g}) exceeds its bound by {worst:.2f}x")
    return worst


def assert_vec_close(name, gpu, ref, tol=VEC_TOL, rows=None):
    """Per-row relative l2 and the element-wise bound."""
    assert_rows_close(name, gpu, ref, tol, rows)
    return assert_elems_close(name, gpu, ref, tol, rows)


def assert_scalars_close(name, gpu, ref, tol=SCAL_TOL, rows=None):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref) / np.maximum(np.abs(ref), 1e-300)
    if rows is not None:
        err = err[rows]
    worst = float(err.max()) if err.size else 0.0
    assert worst <= tol, f"{name}: worst relative error {worst:.3e} > {tol:.0e}"
    return worst


def idx_np(t: torch.Tensor) -> np.ndarray:
    return host(t).view(np.uint16).astype(np.int64)


def spectrum_cuda(X):
    s, V = orc.spectrum(X)
    return s, V, cu(s, torch.float64), cu(V, torch.float64)


def codebook_for(p: mi.Problem) -> np.ndarray:
    return orc.scalar_levels(p.levels) if p.d == 1 else p.codebook.astype(np.float64)


def oracle_grid_f32(p: mi.Problem):
    """The oracle's default per-row scale/offset, rounded to fp32 (given to both sides)."""
    cb = codebook_for(p)
    st = orc.init(p.W, cb)
    return st.scale.astype(np.float32), st.offset.astype(np.float32)


def injected_state(seed: int, W: np.ndarray, scale: np.ndarray, s: np.ndarray, g_lo=1.0, g_hi=40.0):
    """A seeded VAMP state for stage tests: cavity r1 near w, precisions with
    gamma1 * scale^2 in [g_lo, g_hi] (the temperatures a solve visits),
    posterior means near w, alpha1 in (0.2, 0.8), beta around gamma1/median(s^2)."""
    g = np.random.default_rng(seed)
    m, n = W.shape
    sc = np.asarray(scale, np.float64)
    R1 = W + 0.3 * sc[:, None] * g.standard_normal((m, n))
    gamma1 = g.uniform(g_lo, g_hi, m) / (sc * sc)
    X1 = W + 0.2 * sc[:, None] * g.standard_normal((m, n))
    alpha1 = g.uniform(0.2, 0.8, m)
    vsum = alpha1 * n / gamma1
    beta = gamma1 / np.median(s * s) * np.exp(g.uniform(-1.0, 1.0, m))
    gamma1_0 = gamma1 * np.exp(g.uniform(-0.5, 0.5, m))
    return (R1.astype(np.float32), gamma1, X1.astype(np.float32), vsum, beta, gamma1_0)
