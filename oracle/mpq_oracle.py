"""Float64 CPU oracle of the MPQ row solver.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this module.  It shares no code with the CUDA library: it is a
plain, slow restatement of what the MPQ method computes, in float64 NumPy,
one row at a time, so that a reader can check it against the pages by eye.

Sources (cited by page title and section):
  [MPQ-note]  "MPQ: A Message-Passing View of Post-Training Quantization",
              papernotes.org NeurIPS 2026 note: sections "Overall framework"
              (整体框架), "Key design 1/2/3" (关键设计), "Loss / training
              strategy" (损失函数 / 训练策略, the hyper-parameters), and the
              flowchart.
  [MPQ-sum]   same title, ai.info AI summary, "Methodology in Plain English".
  [NeUQI]     "NeUQI: Near-Optimal Uniform Quantization Parameter
              Initialization for Low-Bit LLMs" note, section "Existing pain
              points" (现有痛点): the min-max scale / zero-point formula.

Readings where the pages are silent (the CUDA library takes the same ones):
  R1  rank cut: keep Gram eigenvalues lambda_l > lambda_max * max(m, n) * 2^-52
      (the NumPy matrix_rank convention applied to the Gram matrix).
  R2  scalar grid: per-row min-max, s=(max-min)/(L-1), z=clip(rint(-min/s)),
      level k = s*(k - z); a constant row uses s = |w| (or 1 for zero).
  R3  lattice scale: codeword c maps to RMS(w) * c.
  R4  initial cavity r1 = w; beta0 = 1.  The prior anchor pins each block
      to its own weights with a width of tau codebook units (grid steps of a
      scalar grid, lattice units of a vector codebook):
      log rho_b(c) = -|c - w_b|^2 / (2 tau^2 scale_b^2) in weight units.
      tau = 0.2 is the pages' default; tau = inf means uniform rho_b.
  R5  extrinsic updates use the divergence form (identical to the pages'
      eta form when nothing is clipped): mean divergences alpha are clipped
      into [1e-10, 0.99] before the extrinsic mean is formed, and the
      extrinsic precisions into [1e-10, 1e10] * gamma1_0.
  R6  alpha2 counts null-space directions (n - r) as passing r2 through.
  R7  damping acts on beta (not 1/beta): beta <- (1-rho) beta + rho beta_hat.
  R8  the marginal-MAP argmax comes from one more denoiser call on the last
      (r1, gamma1); T_vamp = 0 therefore gives round-to-nearest.
  R9  CD: blocks in order, argmin over all codewords (lowest index on ties),
      accept iff the energy change is strictly negative; stop after a sweep
      that changes nothing.
  R16 greedy baseline (LDLQ / GPTQ): blocks in order, each committed to its
      nearest codeword in the Euclidean metric (lowest index on ties), the
      error passed on through the factor of (H + lambda I)^-1 with
      lambda = damp * mean(diag H); damp defaults to 0.01.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

GAMMA_LO_REL = 1e-10
GAMMA_HI_REL = 1e10
ALPHA_MIN = 1e-10
ALPHA_MAX = 0.99
TAU = 0.2   # anchor scale, [MPQ-note] hyper-parameter section (reading R4)


# ----------------------------------------------------------------------------
# a1: setup -- compact SVD of X via the smaller Gram matrix
# ----------------------------------------------------------------------------

def spectrum(X: np.ndarray):
    """Singular values s (descending) and right singular vectors V (n x r) of
    X, r = numerical rank.  [MPQ-note] Key design 1 and the flowchart: the
    compact SVD A = U Sigma_A V^T with A = X, T = Sigma_A V^T (r x n)."""
    X = np.asarray(X, dtype=np.float64)
    m, n = X.shape
    if n <= m:
        lam, V = np.linalg.eigh(X.T @ X)
        order = np.argsort(lam)[::-1]
        lam, V = lam[order], V[:, order]
        s = np.sqrt(np.clip(lam, 0.0, None))
    else:
        lam, U = np.linalg.eigh(X @ X.T)
        order = np.argsort(lam)[::-1]
        lam, U = lam[order], U[:, order]
        s = np.sqrt(np.clip(lam, 0.0, None))
        V = None
    # rank cut on the eigenvalues of the Gram matrix actually decomposed
    tol = (lam[0] if lam.size else 0.0) * max(m, n) * 2.0 ** -52
    r = int(np.count_nonzero(lam > tol))
    s = s[:r]
    if V is None:
        V = (X.T @ U[:, :r]) / s[None, :]
    else:
        V = V[:, :r]
    return s, np.ascontiguousarray(V)


def left_vectors(X: np.ndarray, s: np.ndarray, V: np.ndarray) -> np.ndarray:
    """U = X V Sigma^-1 (m x r), the left factor of the compact SVD."""
    return (np.asarray(X, np.float64) @ V) / s[None, :]


def hessian(s: np.ndarray, V: np.ndarray) -> np.ndarray:
    """H = T^T T = V diag(s^2) V^T (n x n)."""
    return (V * (s * s)[None, :]) @ V.T


# ----------------------------------------------------------------------------
# codebooks and a2: init
# ----------------------------------------------------------------------------

def minmax_grid(W: np.ndarray, L: int, group: int = 0):
    """Uniform grid of L levels (reading R2), following the min-max formula
    of the [NeUQI] note ("Existing pain points"):
    s = (max w - min w) / (2^k - 1), z = -round(min w / s).
    Returns (scale, offset) with level k = scale * k + offset: one grid per
    row (m), or with ``group`` > 0 one grid per group of that many
    consecutive columns of a row (m x n/group; the pages' group-wise setting,
    [MPQ-note] experimental setup "group 128")."""
    W = np.asarray(W, np.float64)
    m, n = W.shape
    Wg = W.reshape(m, n // group, group) if group else W[:, None, :]
    lo, hi = Wg.min(axis=2), Wg.max(axis=2)
    scale = (hi - lo) / (L - 1)
    const = ~(hi > lo)
    scale[const] = np.where(hi[const] != 0.0, np.abs(hi[const]), 1.0)
    z = np.clip(np.rint(-lo / scale), 0, L - 1)
    offset = -scale * z
    return (scale, offset) if group else (scale[:, 0], offset[:, 0])


def rms_scale(W: np.ndarray):
    """Per-row RMS scale for the lattice codebook (reading R3)."""
    W = np.asarray(W, np.float64)
    rho = np.sqrt(np.mean(W * W, axis=1))
    rho[rho == 0.0] = 1.0
    return rho, np.zeros_like(rho)


def row_candidates(codebook: np.ndarray, scale: float, offset: float) -> np.ndarray:
    """All codewords of one row's block codebook C_b, K x d, in weight units."""
    return scale * np.asarray(codebook, np.float64) + offset


def block_candidates(codebook: np.ndarray, scale_i, offset_i, B: int) -> np.ndarray:
    """The codebooks C_b of every block of one row, B x K x d: the same for
    all blocks with a per-row grid (scalar scale_i), or the grid of each
    block's group (scale_i of length n/group, B a multiple of it)."""
    s = np.asarray(scale_i, np.float64)
    o = np.asarray(offset_i, np.float64)
    cb = np.asarray(codebook, np.float64)
    if s.ndim == 0:
        return np.broadcast_to(s * cb + o, (B,) + cb.shape)
    per = B // s.size  # blocks per group
    return np.repeat(s, per)[:, None, None] * cb[None] + np.repeat(o, per)[:, None, None]


def scalar_levels(L: int) -> np.ndarray:
    return np.arange(L, dtype=np.float64)[:, None]


def nearest_codewords(w: np.ndarray, cand: np.ndarray):
    """Blockwise nearest codeword (lowest index on ties)."""
    d = cand.shape[1]
    blocks = np.asarray(w, np.float64).reshape(-1, d)
    dist = ((blocks[:, None, :] - cand[None, :, :]) ** 2).sum(axis=2)
    return np.argmin(dist, axis=1)


@dataclass
class InitState:
    scale: np.ndarray
    offset: np.ndarray
    idx_rtn: np.ndarray
    gamma1: np.ndarray
    R1: np.ndarray
    beta: np.ndarray


def init(W: np.ndarray, codebook: np.ndarray, scale=None, offset=None, beta0: float = 1.0,
         group: int = 0) -> InitState:
    """[MPQ-note] hyper-parameter section: gamma1_0 = 1 / MSE(w, w_rtn);
    cavity r1_0 = w (R4); beta_0 = 1.  Scale/offset default to the min-max
    grid (d = 1; per row, or per group of ``group`` columns) or the RMS
    lattice scale (d > 1)."""
    W = np.asarray(W, np.float64)
    d = codebook.shape[1]
    if scale is None:
        if d == 1:
            scale, offset = minmax_grid(W, codebook.shape[0], group)
        else:
            scale, offset = rms_scale(W)
    scale = np.asarray(scale, np.float64)
    offset = np.asarray(offset, np.float64)
    m, n = W.shape
    B = n // d
    idx = np.zeros((m, B), dtype=np.int64)
    g1 = np.zeros(m)
    for i in range(m):
        cand = block_candidates(codebook, scale[i], offset[i], B)      # B x K x d
        blocks = W[i].reshape(B, d)
        idx[i] = np.argmin(((blocks[:, None, :] - cand) ** 2).sum(axis=2), axis=1)
        w_rtn = cand[np.arange(B), idx[i]].reshape(-1)
        mse = np.mean((W[i] - w_rtn) ** 2)
        g1[i] = 1.0 / max(mse, 1e-30)
    return InitState(scale, offset, idx, g1, W.copy(), np.full(m, float(beta0)))


# ----------------------------------------------------------------------------
# a3: blockwise discrete denoiser
# ----------------------------------------------------------------------------

@dataclass
class DenoiseOut:
    xhat: np.ndarray     # m x n posterior means
    vblock: np.ndarray   # m x B traces of the posterior covariances
    vsum: np.ndarray     # m, sum over blocks
    idx: np.ndarray      # m x B argmax codeword
    gap: np.ndarray      # m x B top-two logit gap (for tie exemptions)


def block_scales(scale_i, B: int) -> np.ndarray:
    """The scale of each of a row's B blocks (its group's with group-wise
    grids)."""
    s = np.atleast_1d(np.asarray(scale_i, np.float64))
    return np.repeat(s, B // s.size)


def denoise(R1, gamma1, codebook, scale, offset, W=None, tau: float = math.inf) -> DenoiseOut:
    """[MPQ-note] Key design 1: for every block b and codeword c,
    q_b(c) proportional to rho_b(c) exp(-gamma1/2 |c - r1_b|^2); returns the
    posterior mean, the trace of the posterior covariance and the argmax.
    With a finite ``tau`` the prior anchors the block to its weights w_b
    ("the prior anchor", ibid.; reading R4):
    rho_b(c) = exp(-|c - w_b|^2 / (2 tau^2 scale_b^2)), a width of tau
    codebook units; tau = inf gives the uniform prior."""
    R1 = np.asarray(R1, np.float64)
    m, n = R1.shape
    d = codebook.shape[1]
    B = n // d
    xhat = np.zeros((m, n))
    vblock = np.zeros((m, B))
    idx = np.zeros((m, B), dtype=np.int64)
    gap = np.zeros((m, B))
    for i in range(m):
        cand = block_candidates(codebook, scale[i], offset[i], B)      # B x K x d
        r = R1[i].reshape(B, d)
        logit = -0.5 * gamma1[i] * ((r[:, None, :] - cand) ** 2).sum(axis=2)
        if math.isfinite(tau):
            wb = np.asarray(W[i], np.float64).reshape(B, d)
            ga = 1.0 / (tau * tau * block_scales(scale[i], B) ** 2)    # B anchor precisions
            logit = logit - 0.5 * ga[:, None] * ((wb[:, None, :] - cand) ** 2).sum(axis=2)
        top = np.argmax(logit, axis=1)
        mx = logit[np.arange(B), top]
        q = np.exp(logit - mx[:, None])
        q /= q.sum(axis=1, keepdims=True)
        # moments centred on the argmax codeword (no cancellation)
        cstar = cand[np.arange(B), top]                                 # B x d
        dc = cand - cstar[:, None, :]                                   # B x K x d
        m1 = np.einsum("bk,bkd->bd", q, dc)
        m2 = np.einsum("bk,bk->b", q, (dc * dc).sum(axis=2))
        xhat[i] = (cstar + m1).reshape(-1)
        vblock[i] = np.maximum(m2 - (m1 * m1).sum(axis=1), 0.0)
        idx[i] = top
        srt = np.sort(logit, axis=1)
        gap[i] = srt[:, -1] - srt[:, -2] if logit.shape[1] > 1 else np.inf
    return DenoiseOut(xhat, vblock, vblock.sum(axis=1), idx, gap)


# ----------------------------------------------------------------------------
# a4-a6: extrinsic updates, Gaussian linear module, EB M-step for beta
# ----------------------------------------------------------------------------

@dataclass
class LinearOut:
    gamma2: np.ndarray
    eta1: np.ndarray
    R2: np.ndarray
    u: np.ndarray        # m x r cavity residual  u = y~ - s * V^T r2
    Uprime: np.ndarray   # m x r  D * u
    xhat2: np.ndarray
    alpha2: np.ndarray
    eta2: np.ndarray
    beta_hat: np.ndarray
    beta: np.ndarray     # damped
    gamma1: np.ndarray   # new
    R1: np.ndarray       # new
    clamps: np.ndarray   # number of clamps applied per row in this step


def _clamp(v, lo, hi):
    """Clip into [lo, hi] (NaN -> lo); also return 1 where clipping acted."""
    v = np.asarray(v, np.float64)
    c = np.where(np.isnan(v), lo, np.clip(v, lo, hi))
    return c, (c != v).astype(np.int64)


def linear_step(W, R1, gamma1, xhat1, vsum, beta, s, V, gamma1_0, damping=0.5) -> LinearOut:
    """One VAMP half-iteration after the denoiser.

    Extrinsic update denoiser -> linear ([MPQ-note] Key design 1: the
    extrinsic step removes the denoiser's self-feedback).  With the
    denoiser's mean divergence alpha1 = gamma1 * sum_b tr(Sigma_1b) / n:
    eta1 = gamma1 / alpha1, gamma2 = eta1 - gamma1 = gamma1 (1-alpha1)/alpha1,
    r2 = (eta1 xhat1 - gamma1 r1) / gamma2 = (xhat1 - alpha1 r1) / (1 - alpha1).
    Reading R5: alpha is clipped into [ALPHA_MIN, ALPHA_MAX] before r2 and
    gamma2 are formed, and gamma2 is then clipped into [1e-10, 1e10]*gamma1_0.

    Gaussian linear module: xhat2 solves (beta T^T T + gamma2 I) x =
    beta T^T y~ + gamma2 r2, evaluated in the singular basis
    ([MPQ-note] Key design 1 "analytic solution"; [MPQ-note] Highlights: no
    large inverse in rank space): with p = V^T r2, u = y~ - s*p,
    xhat2 = r2 + V (beta s / (beta s^2 + gamma2) * u), and its mean divergence
    alpha2 = [sum_l gamma2/(beta s_l^2 + gamma2) + (n - r)] / n (R6).

    EB M-step ([MPQ-note] Key design 2 equation):
    1/beta_hat = (1/r) sum_l [(gamma2/(beta s_l^2+gamma2))^2 u_l^2
                              + s_l^2/(beta s_l^2+gamma2)],
    then beta <- (1 - rho) beta + rho beta_hat (R7), rho = 0.5
    ([MPQ-note] hyper-parameter section).

    Extrinsic update linear -> denoiser: eta2 = gamma2/alpha2,
    gamma1' = eta2 - gamma2 = gamma2 (1-alpha2)/alpha2,
    r1' = (eta2 xhat2 - gamma2 r2)/gamma1' = (xhat2 - alpha2 r2)/(1 - alpha2),
    with the same clipping of alpha2 and gamma1'."""
    W = np.asarray(W, np.float64)
    R1 = np.asarray(R1, np.float64)
    xhat1 = np.asarray(xhat1, np.float64)
    m, n = W.shape
    r = s.size
    lo = GAMMA_LO_REL * gamma1_0
    hi = GAMMA_HI_REL * gamma1_0
    a1, c1 = _clamp(gamma1 * vsum / n, ALPHA_MIN, ALPHA_MAX)
    gamma2, c2 = _clamp(gamma1 * (1.0 - a1) / a1, lo, hi)
    eta1 = gamma1 / a1
    R2 = (xhat1 - a1[:, None] * R1) / (1.0 - a1[:, None])
    ytil = (W @ V) * s[None, :]                      # y~ = U^T X w = s * V^T w
    p = R2 @ V
    u = ytil - s[None, :] * p
    den = beta[:, None] * (s * s)[None, :] + gamma2[:, None]
    D = beta[:, None] * s[None, :] / den
    Up = D * u
    xhat2 = R2 + Up @ V.T
    alpha2_raw = ((gamma2[:, None] / den).sum(axis=1) + (n - r)) / n
    inv_bhat = (((gamma2[:, None] / den) ** 2) * u * u + (s * s)[None, :] / den).sum(axis=1) / r
    beta_hat = 1.0 / inv_bhat
    beta_new = (1.0 - damping) * beta + damping * beta_hat
    a2, c3 = _clamp(alpha2_raw, ALPHA_MIN, ALPHA_MAX)
    gamma1_new, c4 = _clamp(gamma2 * (1.0 - a2) / a2, lo, hi)
    eta2 = gamma2 / a2
    R1_new = (xhat2 - a2[:, None] * R2) / (1.0 - a2[:, None])
    return LinearOut(gamma2, eta1, R2, u, Up, xhat2, alpha2_raw, eta2, beta_hat, beta_new,
                     gamma1_new, R1_new, c1 + c2 + c3 + c4)


# ----------------------------------------------------------------------------
# a8-a9: exact block coordinate descent in the metric H
# ----------------------------------------------------------------------------

@dataclass
class CDOut:
    idx: np.ndarray
    x: np.ndarray
    changes: np.ndarray      # m x sweeps
    sweeps_run: np.ndarray   # m
    first_tie: np.ndarray    # m: global step index of the first near-tie (or -1)
    min_gap_rel: np.ndarray  # m: smallest top-two gap / |E| seen
    step_gap: np.ndarray     # m x (sweeps*B): top-two gap / |E| of each step (inf: not run)


def decode(idx, codebook, scale, offset):
    idx = np.asarray(idx)
    m = idx.shape[0]
    out = []
    for i in range(m):
        B = idx[i].size
        cand = block_candidates(codebook, scale[i], offset[i], B)
        out.append(cand[np.arange(B), idx[i]].reshape(-1))
    return np.asarray(out)


def cd(W, idx0, codebook, scale, offset, H, sweeps: int, tie_rel: float = 1e-5) -> CDOut:
    """[MPQ-note] Key design 3: with residual u = y~ - T x, the block objective
    F_b(c) = 1/2 |u - T_b (c - x_b)|^2 is minimised over all c in C_b, which
    equals the Mahalanobis nearest-codeword problem in G_b = T_b^T T_b.
    Written with h = T^T u = H (w - x):  F_b(c) - F_b(x_b) =
    -delta^T h_b + 1/2 delta^T G_b delta, delta = c - x_b.  Blocks are
    visited in order; the argmin is accepted when the change is negative
    and h is updated by -H[:, b] delta.  At most ``sweeps`` sweeps, stopping
    after one without any change ([MPQ-note] hyper-parameter section)."""
    W = np.asarray(W, np.float64)
    m, n = W.shape
    d = codebook.shape[1]
    B = n // d
    idx = np.array(idx0, dtype=np.int64, copy=True)
    X = decode(idx, codebook, scale, offset)
    changes = np.zeros((m, sweeps), dtype=np.int64)
    sweeps_run = np.zeros(m, dtype=np.int64)
    first_tie = np.full(m, -1, dtype=np.int64)
    min_gap = np.full(m, np.inf)
    step_gap = np.full((m, sweeps * B), np.inf)
    for i in range(m):
        cand = block_candidates(codebook, scale[i], offset[i], B)      # B x K x d
        x = X[i].copy()
        h = H @ (W[i] - x)
        step = 0
        for sw in range(sweeps):
            sweeps_run[i] = sw + 1
            nchg = 0
            for b in range(B):
                sl = slice(b * d, (b + 1) * d)
                G = H[sl, sl]
                delta = cand[b] - x[sl][None, :]
                dE = -delta @ h[sl] + 0.5 * np.einsum("kd,de,ke->k", delta, G, delta)
                k = int(np.argmin(dE))
                E = 0.5 * float((W[i] - x) @ h)
                if dE.size > 1:
                    two = np.partition(dE, 1)[:2]
                    g = (two[1] - two[0]) / max(abs(E), 1e-300)
                    step_gap[i, step] = g
                    min_gap[i] = min(min_gap[i], g)
                    if g < tie_rel and first_tie[i] < 0:
                        first_tie[i] = step
                if dE[k] < 0.0:
                    dlt = delta[k]
                    h -= H[:, sl] @ dlt
                    x[sl] = cand[b, k]
                    idx[i, b] = k
                    nchg += 1
                step += 1
            changes[i, sw] = nchg
            if nchg == 0:
                break
        X[i] = x
    return CDOut(idx, X, changes, sweeps_run, first_tie, min_gap, step_gap)


# ----------------------------------------------------------------------------
# greedy baseline: LDLQ / GPTQ
# ----------------------------------------------------------------------------

@dataclass
class GreedyOut:
    idx: np.ndarray          # m x B
    gap: np.ndarray          # m x B: top-two distance gap of each decision / scale^2


def damped_hessian(H, damp: float):
    """H + lambda I, lambda = damp * mean(diag H) (reading R16)."""
    H = np.asarray(H, np.float64)
    lam = damp * float(np.trace(H)) / H.shape[0]
    return H + lam * np.eye(H.shape[0])


def ldlq(W, codebook, scale, offset, H, damp: float = 0.01) -> GreedyOut:
    """The greedy hard-decision solver MPQ is measured against ([MPQ-note]
    motivation: GPTQ and LDLQ visit the blocks in order, commit each one to a
    single codeword at once and pass its hard error on to the blocks not yet
    quantised; ablation table: "LDLQ baseline" = T_vamp 0, CD 0, and
    "LDLQ + CD3").  Error feedback in the GPTQ form: with U the upper
    Cholesky factor of (H + lambda I)^-1 = U^T U, committing column j to q_j
    moves every later column k by -(v_j - q_j) U[j, k] / U[j, j], which puts
    the not-yet-quantised weights at their least-squares optimum given the
    committed ones.  A block is committed to the codeword nearest (Euclidean)
    its current values, then its columns feed back one after another."""
    W = np.asarray(W, np.float64)
    m, n = W.shape
    d = codebook.shape[1]
    B = n // d
    U = np.linalg.cholesky(np.linalg.inv(damped_hessian(H, damp))).T
    idx = np.zeros((m, B), dtype=np.int64)
    gap = np.full((m, B), np.inf)
    for i in range(m):
        cand = block_candidates(codebook, scale[i], offset[i], B)      # B x K x d
        si = np.atleast_1d(np.asarray(scale[i], np.float64))
        sc = np.repeat(si, B // si.size)                              # scale of each block
        v = W[i].copy()
        for b in range(B):
            sl = slice(b * d, (b + 1) * d)
            dist = ((v[sl][None, :] - cand[b]) ** 2).sum(axis=1)
            k = int(np.argmin(dist))
            if dist.size > 1:
                two = np.partition(dist, 1)[:2]
                gap[i, b] = (two[1] - two[0]) / (sc[b] * sc[b])
            q = cand[b, k]
            for t, j in enumerate(range(b * d, (b + 1) * d)):
                err = (v[j] - q[t]) / U[j, j]
                v[j + 1:] -= err * U[j, j + 1:]
            idx[i, b] = k
    return GreedyOut(idx, gap)


# ----------------------------------------------------------------------------
# a10: energies
# ----------------------------------------------------------------------------

def energy(W, What, s, V):
    """E = 1/2 |T (w - w_hat)|^2 per row with T = diag(s) V^T
    ([MPQ-note] Overall framework: the row objective 1/2 |Xw - X w_hat|^2)."""
    e = np.asarray(W, np.float64) - np.asarray(What, np.float64)
    p = (e @ V) * s[None, :]
    return 0.5 * (p * p).sum(axis=1)


def energy_direct(W, What, X):
    e = np.asarray(W, np.float64) - np.asarray(What, np.float64)
    y = e @ np.asarray(X, np.float64).T
    return 0.5 * (y * y).sum(axis=1)


# ----------------------------------------------------------------------------
# the whole solve
# ----------------------------------------------------------------------------

@dataclass
class SolveOut:
    idx: np.ndarray
    w_hat: np.ndarray
    energy: np.ndarray
    idx_map: np.ndarray
    map_gap: np.ndarray
    gamma1: np.ndarray
    beta: np.ndarray
    clamps: np.ndarray
    cd: Optional[CDOut]
    trace: list = field(default_factory=list)


def terminal_precision(gamma1, scale):
    """Terminal VAMP precision in grid units, gamma1 s^2, with s the row's
    scale (its largest group scale with group-wise grids)."""
    s = np.asarray(scale, np.float64)
    s = s if s.ndim == 1 else s.max(axis=1)
    return np.asarray(gamma1, np.float64) * s * s


def solve(W, codebook, s, V, T_vamp: int, cd_sweeps: int, scale=None, offset=None,
          beta0: float = 1.0, damping: float = 0.5, tau: float = TAU,
          keep_trace: bool = False, group: int = 0, cd_skip_precision: float = 0.0,
          greedy_damp: Optional[float] = None) -> SolveOut:
    """The MPQ solve of every row ([MPQ-note] flowchart and Overall
    framework): init -> T_vamp x (denoiser -> extrinsic -> linear module ->
    M-step) -> marginal MAP argmax -> exact block CD -> energies, with the
    denoiser's prior anchored at ``tau`` codebook units (default 0.2, the
    [MPQ-note] hyper-parameter section; tau = inf is the unanchored form).
    With ``cd_skip_precision`` > 0, rows whose terminal precision (see
    terminal_precision) exceeds it keep the marginal MAP and run no CD: the
    [MPQ-note] diagnostics report terminal precisions near 1e5 at 3-bit
    scalar with CD changing almost no block (reading R13).
    With T_vamp = 0 and ``greedy_damp`` given, the hard init that CD refines
    is the greedy baseline ldlq(..., damp=greedy_damp) instead of
    round-to-nearest (the ablation's LDLQ and LDLQ + CD rows)."""
    W = np.asarray(W, np.float64)
    st = init(W, codebook, scale, offset, beta0, group)
    g10 = st.gamma1.copy()
    R1, g1, beta = st.R1, st.gamma1.copy(), st.beta.copy()
    clamps = np.zeros(W.shape[0], dtype=np.int64)
    trace = []
    for _ in range(T_vamp):
        dn = denoise(R1, g1, codebook, st.scale, st.offset, W, tau)
        lo = linear_step(W, R1, g1, dn.xhat, dn.vsum, beta, s, V, g10, damping)
        if keep_trace:
            trace.append((dn, lo))
        R1, g1, beta = lo.R1, lo.gamma1, lo.beta
        clamps += lo.clamps
    if T_vamp == 0 and greedy_damp is not None:
        gr = ldlq(W, codebook, st.scale, st.offset, hessian(s, V), greedy_damp)
        idx_map, map_gap = gr.idx, gr.gap
    else:
        dn = denoise(R1, g1, codebook, st.scale, st.offset, W, tau)
        idx_map, map_gap = dn.idx, dn.gap
    cdo = None
    idx = idx_map
    if cd_sweeps > 0:
        H = hessian(s, V)
        cdo = cd(W, idx_map, codebook, st.scale, st.offset, H, cd_sweeps)
        idx = cdo.idx
        if cd_skip_precision > 0:
            skip = terminal_precision(g1, st.scale) > cd_skip_precision
            idx = np.where(skip[:, None], idx_map, cdo.idx)
            cdo.idx = idx
            cdo.changes[skip] = 0
            cdo.first_tie[skip] = -1
            cdo.x = decode(idx, codebook, st.scale, st.offset)
    w_hat = decode(idx, codebook, st.scale, st.offset)
    E = energy(W, w_hat, s, V)
    return SolveOut(idx, w_hat, E, idx_map, map_gap, g1, beta, clamps, cdo, trace)


# ----------------------------------------------------------------------------
# brute force helpers for pins
# ----------------------------------------------------------------------------

def greedy_conditional(w, codebook, scale, offset, Ht):
    """The greedy baseline by its definition, for pins on short rows: block b
    takes the codeword nearest the b-part of the least-squares optimum of the
    blocks >= b given the committed blocks < b (minimising e^T Ht e over the
    free part of the error e = w - x), solved afresh for every block."""
    w = np.asarray(w, np.float64)
    n = w.size
    d = codebook.shape[1]
    B = n // d
    cand = block_candidates(codebook, scale, offset, B)
    x = np.zeros(n)
    idx = np.zeros(B, dtype=np.int64)
    for b in range(B):
        c0 = b * d
        e_fixed = w[:c0] - x[:c0]
        e_free = -np.linalg.solve(Ht[c0:, c0:], Ht[c0:, :c0] @ e_fixed) if c0 else np.zeros(n)
        target = w[c0:c0 + d] - e_free[:d]
        k = int(np.argmin(((target[None, :] - cand[b]) ** 2).sum(axis=1)))
        idx[b] = k
        x[c0:c0 + d] = cand[b, k]
    return idx


def exhaustive_min_energy(w, codebook, scale, offset, H):
    """Exact minimum of 1/2 (w-x)^T H (w-x) over every assignment of a short
    row (d = 1), by splitting the coordinates in two halves and enumerating
    all pairs: E = a_i + b_j + e_A,i^T H_AB e_B,j."""
    w = np.asarray(w, np.float64)
    n = w.size
    cand = row_candidates(codebook, scale, offset)[:, 0]
    L = cand.size
    na = n // 2
    A, Bi = np.arange(na), np.arange(na, n)

    def all_err(cols):
        k = len(cols)
        grid = np.stack(np.meshgrid(*([np.arange(L)] * k), indexing="ij"), -1).reshape(-1, k)
        return w[cols][None, :] - cand[grid], grid

    eA, gA = all_err(A)
    eB, gB = all_err(Bi)
    HAA, HBB, HAB = H[np.ix_(A, A)], H[np.ix_(Bi, Bi)], H[np.ix_(A, Bi)]
    a = 0.5 * np.einsum("ij,jk,ik->i", eA, HAA, eA)
    b = 0.5 * np.einsum("ij,jk,ik->i", eB, HBB, eB)
    tot = a[:, None] + b[None, :] + eA @ HAB @ eB.T
    k = np.unravel_index(np.argmin(tot), tot.shape)
    return float(tot[k]), np.concatenate([gA[k[0]], gB[k[1]]])
