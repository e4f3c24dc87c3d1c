"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This module holds no arithmetic of the solver itself: it only draws weight
rows W and calibration activations X of the shapes and value distributions
of the MPQ paper's workloads, builds the offset-E8 codebook that the 2-bit
configuration quantises onto (a fixed table that is an *input* of the
solver), applies the randomised Hadamard preprocessing that the paper names
for its lattice setting, and draws injected solver states for per-stage
parity tests.

Workloads (stand-ins for Llama layers and 128x2048 C4 calibration
activations, which are not available here; no dataset item is used):

* ``tiny``  -- W 16x64 ~ N(0,1); X 256x64 with AR(1) rho=0.7 columns;
  3-bit per-row min-max grid; T_vamp=8; plus 4 rows of n=12 at 2-bit
  (``tiny12``) for exhaustive checks.
* ``l1b``   -- W 2048x2048, N(0,1/n) rows with log-normal(0.5) row std;
  X 4096x2048, Student-t(5) innovations through AR(1) rho=0.5, 1% of
  channels x10; 3-bit; T_vamp=16.
* ``q4096`` -- W 4096x4096, X 8192x4096, same generators; 4-bit; T=16.
* ``e8``    -- as q4096, then W <- W Q^T, X <- X Q^T with Q a seeded
  random-sign Sylvester Hadamard / sqrt(n); offset-E8 codebook K=65536,
  d=8; T_vamp=16 (``e8t8``: T_vamp=8).
* ``down``  -- W 4096x14336 log-normal rows; X 4096x14336 with the same
  t/AR/outlier generator (rank 4096 < n); 3-bit; T=16.

Seeds: ``numpy.random.default_rng(20261202 + 10*config + k)`` with k = 0
for W, 1 for X, 2 for outlier channels, 3 for Hadamard signs.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Optional

import numpy as np

SEED_BASE = 20261202

# name -> (config number, m_out, n, m_calib, d, levels or K, T_vamp, cd sweeps)
WORKLOADS = {
    "tiny": (1, 16, 64, 256, 1, 8, 8, 3),
    "tiny12": (1, 4, 12, 256, 1, 4, 8, 3),
    "l1b": (2, 2048, 2048, 4096, 1, 8, 16, 3),
    "q4096": (3, 4096, 4096, 8192, 1, 16, 16, 3),
    "e8": (4, 4096, 4096, 8192, 8, 65536, 16, 3),
    "e8t8": (4, 4096, 4096, 8192, 8, 65536, 8, 3),
    "down": (5, 4096, 14336, 4096, 1, 8, 16, 3),
}


def rng_for(config: int, k: int) -> np.random.Generator:
    return np.random.default_rng(SEED_BASE + 10 * config + k)


# ----------------------------------------------------------------------------
# activations and weights
# ----------------------------------------------------------------------------

def ar1_columns(innov: np.ndarray, rho: float) -> np.ndarray:
    """Run the AR(1) recursion x_j = rho x_{j-1} + sqrt(1-rho^2) z_j across
    the columns of ``innov`` (m x n), so that each row has AR(1) covariance
    rho^|i-j| between channels i and j (up to the innovation variance)."""
    z = np.asarray(innov, dtype=np.float64)
    out = np.empty_like(z)
    c = math.sqrt(1.0 - rho * rho)
    out[:, 0] = z[:, 0]
    for j in range(1, z.shape[1]):
        out[:, j] = rho * out[:, j - 1] + c * z[:, j]
    return out


def gaussian_ar1_x(rng: np.random.Generator, m: int, n: int, rho: float) -> np.ndarray:
    return ar1_columns(rng.standard_normal((m, n)), rho)


def heavy_tailed_x(rng_x: np.random.Generator, rng_out: np.random.Generator,
                   m: int, n: int, rho: float = 0.5, nu: float = 5.0,
                   outlier_frac: float = 0.01, outlier_gain: float = 10.0) -> np.ndarray:
    x = ar1_columns(rng_x.standard_t(nu, size=(m, n)), rho)
    n_out = int(outlier_frac * n)
    if n_out > 0:
        cols = rng_out.choice(n, size=n_out, replace=False)
        x[:, np.sort(cols)] *= outlier_gain
    return x


def lognormal_rows_w(rng: np.random.Generator, m_out: int, n: int, sigma: float = 0.5) -> np.ndarray:
    xi = rng.standard_normal(m_out)
    w = rng.standard_normal((m_out, n)) / math.sqrt(n)
    return w * np.exp(sigma * xi)[:, None]


def fwht_rows(a: np.ndarray) -> np.ndarray:
    """Unnormalised Sylvester-Hadamard transform of every row (n a power of 2):
    returns a @ H_n with H_1 = [1], H_2k = [[H_k, H_k], [H_k, -H_k]]."""
    a = np.array(a, dtype=np.float64, copy=True)
    m, n = a.shape
    assert n & (n - 1) == 0, "Hadamard size must be a power of two"
    h = 1
    while h < n:
        v = a.reshape(m, n // (2 * h), 2, h)
        x, y = v[:, :, 0, :].copy(), v[:, :, 1, :].copy()
        v[:, :, 0, :] = x + y
        v[:, :, 1, :] = x - y
        h *= 2
    return a


def random_hadamard_apply(a: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """Rows of a times Q^T, Q = H_n diag(signs) / sqrt(n) (orthogonal).
    a Q^T = a diag(signs) H_n^T / sqrt(n) and H_n is symmetric."""
    n = a.shape[1]
    return fwht_rows(a * signs[None, :]) / math.sqrt(n)


# ----------------------------------------------------------------------------
# offset-E8 codebook
# ----------------------------------------------------------------------------

def e8_points_in_box(box: float = 3.5, offset: float = 0.25):
    """All points x of E8 = {x in Z^8 u (Z+1/2)^8 : sum(x) even} whose shifted
    coordinates c = x + offset all satisfy |c_i| <= box.  Returned as int8
    arrays of 4c (exact; 4c is an integer for offset 1/4) and of 2x."""
    out4c, out2x = [], []
    for half in (0, 1):
        lo = math.ceil(-box - offset - 0.5 * half)
        hi = math.floor(box - offset - 0.5 * half)
        vals = np.arange(lo, hi + 1)  # integer part k, x_i = k + half/2
        grids = np.meshgrid(*([vals] * 8), indexing="ij")
        k = np.stack([g.reshape(-1) for g in grids], axis=1).astype(np.int16)
        two_x = 2 * k + half  # 2x, integer
        s = two_x.sum(axis=1)  # 2 * sum(x); sum(x) even <=> s % 4 == 0
        keep = (s % 4) == 0
        two_x = two_x[keep]
        four_c = 2 * two_x + int(round(4 * offset))
        inside = np.all(np.abs(four_c) <= int(round(4 * box)), axis=1)
        out4c.append(four_c[inside].astype(np.int8))
        out2x.append(two_x[inside].astype(np.int8))
    return np.concatenate(out4c), np.concatenate(out2x)


def e8_offset_codebook(K: int = 65536, offset: float = 0.25, box: float = 3.5) -> np.ndarray:
    """The first K points of E8 + offset*1, ordered by squared norm of the
    shifted point, ties broken by ascending lexicographic order of its
    coordinates.  Returns a float32 K x 8 array (every entry is an odd
    multiple of 1/4, exact in any float format with >= 4 significand bits).

    The enumeration box |c_i| <= box contains every point whose squared norm
    is <= box^2; the assertion below checks that the K-th point lies inside
    that ball, so no point that should precede it can be missing."""
    four_c, _ = e8_points_in_box(box, offset)
    n16 = (four_c.astype(np.int32) ** 2).sum(axis=1)  # 16 * |c|^2, exact
    keys = [four_c[:, j] for j in range(7, -1, -1)] + [n16]
    order = np.lexsort(keys)
    assert order.size >= K
    cut16 = int(n16[order[K - 1]])
    assert cut16 < 16 * box * box, "enumeration box too small for K"
    cb = four_c[order[:K]].astype(np.float32) / 4.0
    return np.ascontiguousarray(cb)


def codebook_sha256(cb: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(cb, dtype=np.float32).tobytes()).hexdigest()


# ----------------------------------------------------------------------------
# problems
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Problem:
    name: str
    W: np.ndarray            # m_out x n float32
    X: np.ndarray            # m x n float32 (calibration activations)
    d: int                   # block size
    levels: int              # scalar grid levels L (d=1) or codebook size K (d=8)
    codebook: Optional[np.ndarray]  # K x d float32 for d > 1, None for scalar grids
    T_vamp: int
    cd_sweeps: int
    beta0: float = 1.0
    damping: float = 0.5
    tau: float = math.inf
    seeds: dict = dataclasses.field(default_factory=dict)

    @property
    def m_out(self):
        return self.W.shape[0]

    @property
    def n(self):
        return self.W.shape[1]


_E8_CACHE = {}


def e8_codebook_cached(K: int = 65536) -> np.ndarray:
    if K not in _E8_CACHE:
        _E8_CACHE[K] = e8_offset_codebook(K)
    return _E8_CACHE[K]


def make_problem(name: str, rows: Optional[np.ndarray] = None, with_x: bool = True) -> Problem:
    """Build workload ``name``; ``rows`` selects a subset of weight rows (the
    rows are independent problems, so a subset is a valid smaller case)."""
    cfg, m_out, n, m, d, levels, T, sweeps = WORKLOADS[name]
    seeds = {"W": SEED_BASE + 10 * cfg, "X": SEED_BASE + 10 * cfg + 1}
    if name in ("tiny", "tiny12"):
        kw = 0 if name == "tiny" else 4
        kx = 1 if name == "tiny" else 5
        seeds = {"W": SEED_BASE + 10 * cfg + kw, "X": SEED_BASE + 10 * cfg + kx}
        W = rng_for(cfg, kw).standard_normal((m_out, n))
        X = gaussian_ar1_x(rng_for(cfg, kx), m, n, 0.7) if with_x else None
    else:
        W = lognormal_rows_w(rng_for(cfg, 0), m_out, n)
        X = heavy_tailed_x(rng_for(cfg, 1), rng_for(cfg, 2), m, n) if with_x else None
        seeds["outliers"] = SEED_BASE + 10 * cfg + 2
    codebook = None
    if d == 8:
        signs = np.where(rng_for(cfg, 3).random(n) < 0.5, -1.0, 1.0)
        seeds["signs"] = SEED_BASE + 10 * cfg + 3
        W = random_hadamard_apply(W, signs)
        if X is not None:
            X = random_hadamard_apply(X, signs)
        codebook = e8_codebook_cached(levels)
    if rows is not None:
        W = W[np.asarray(rows)]
    W = np.ascontiguousarray(W, dtype=np.float32)
    if X is not None:
        X = np.ascontiguousarray(X, dtype=np.float32)
    return Problem(name, W, X, d, levels, codebook, T, sweeps, seeds=seeds)


def small_problem(seed: int, m_out: int, n: int, m: int, d: int = 1, levels: int = 8,
                  T_vamp: int = 4, cd_sweeps: int = 3, heavy: bool = True,
                  codebook: Optional[np.ndarray] = None) -> Problem:
    """A small seeded problem with the generators of the large workloads, for
    parity tests at sizes that span several tiles and a ragged tail."""
    r = np.random.default_rng(seed)
    if heavy:
        W = lognormal_rows_w(r, m_out, n)
        X = heavy_tailed_x(r, r, m, n)
    else:
        W = r.standard_normal((m_out, n))
        X = gaussian_ar1_x(r, m, n, 0.7)
    return Problem(f"small{seed}", np.ascontiguousarray(W, np.float32),
                   np.ascontiguousarray(X, np.float32), d, levels, codebook,
                   T_vamp, cd_sweeps, seeds={"all": seed})


def random_small_codebook(seed: int, K: int, d: int) -> np.ndarray:
    """A random codebook of K distinct points on the 1/4 grid in [-2, 2]^d."""
    r = np.random.default_rng(seed)
    seen = set()
    out = []
    while len(out) < K:
        p = tuple(int(v) for v in r.integers(-8, 9, size=d))
        if p not in seen:
            seen.add(p)
            out.append(p)
    return np.asarray(out, dtype=np.float32) / 4.0


def orthonormal_spectrum(seed: int, n: int, r: int, cond: float = 1e3):
    """A random (s, V) pair: V n x r with orthonormal columns (QR of a Gaussian),
    s descending, log-uniform over [1, cond] times a scale -- for stage tests
    that inject a spectrum directly."""
    g = np.random.default_rng(seed)
    Q, _ = np.linalg.qr(g.standard_normal((n, r)))
    s = np.sort(np.exp(g.uniform(0.0, math.log(cond), size=r)))[::-1] * 3.0
    return np.ascontiguousarray(s), np.ascontiguousarray(Q)
