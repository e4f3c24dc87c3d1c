// Greedy baseline: LDLQ / GPTQ, batched over rows (scalar grids and d = 8
// codebooks).
//
// Source: "MPQ: A Message-Passing View of Post-Training Quantization"
// (papernotes.org note): the motivation (GPTQ and LDLQ commit each block to
// one codeword at once and pass its hard error on to the blocks not yet
// quantised) and the ablation table (LDLQ baseline: T_vamp = 0 and no CD;
// LDLQ + CD3: the same init refined by three CD sweeps).
//
// Error feedback in the GPTQ form: with (H + lambda I)^-1 = L L^T (L the
// lower Cholesky factor) and B = L diag(L)^-1 (unit lower), committing
// column j to its nearest level q_j moves every later column k of the row by
// -(v_j - q_j) B[k, j]; the uncommitted weights are then at their
// least-squares optimum given the committed ones.  lambda = damp * mean(diag H).
//
// Setup, fp64: (H + lambda I)^-1 from the spectrum, V diag(1/(s^2 + lambda))
// V^T, plus (I - V V^T)/lambda when r < n; then its Cholesky factor by a
// blocked right-looking algorithm: per panel of 32 columns one warp factors
// the diagonal block in shared memory, one kernel solves the rows below it
// against it, and the fp64 SIMT GEMM updates the trailing matrix.
//
// Solve: the columns go in tiles of 128 inside L2-resident panels, as in the
// last CD sweep.  One warp per row walks a tile column by column in registers
// (the lane's 4 columns of the working row, the tile's block of B^T in shared
// memory); the tile's errors leave, divided by the row's scale, as the fp16
// hi/lo A operand of the tensor-core update W_work[:, ahead] -= E B[ahead, tile]^T.
#include <math.h>

#include <vector>

#include "mpq_internal.cuh"

namespace mpq {
namespace {

constexpr int CH_NB = 32;     // Cholesky panel width
constexpr int CH_ROWS = 128;  // rows of the panel per CTA
constexpr int LQ_WARPS = 16;  // rows per tile CTA
constexpr int LQ_SLOTS = CD_TILE / 32;
constexpr int LQ_SMEM = CD_TILE * CD_TILE * 4;

unsigned grid_for(int64_t count) {
  return (unsigned)std::min<int64_t>(cdiv(count, 256), 148 * 16);
}

// out = V diag(c), c_l = 1/(s_l^2 + lambda) - (full ? 0 : 1/lambda)
__global__ void k_hinv_cols(const double* __restrict__ V, const double* __restrict__ s, int64_t n,
                            int64_t r, double lam, int full, double* __restrict__ out) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * r;
       e += (int64_t)gridDim.x * blockDim.x) {
    const double s2 = s[e % r] * s[e % r];
    const double c = 1.0 / (s2 + lam) - (full ? 0.0 : 1.0 / lam);
    out[e] = V[e] * c;
  }
}

__global__ void k_add_diag(double* __restrict__ A, int64_t n, double v) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) A[i * n + i] += v;
}

// Diagonal block of the panel [k0, k0 + kb) of the blocked Cholesky, in
// place: one warp, lane i owning row i (zeros written above the diagonal).
// A pivot that is not positive sets *bad and continues with 1.
__global__ void __launch_bounds__(32)
    k_chol_diag(double* __restrict__ A, int64_t n, int64_t k0, int kb, int* __restrict__ bad) {
  __shared__ double L11[CH_NB][CH_NB + 1];
  const int t = threadIdx.x;
  for (int e = t; e < CH_NB * CH_NB; e += 32) {
    const int i = e / CH_NB, j = e % CH_NB;
    L11[i][j] = (i < kb && j <= i) ? A[(k0 + i) * n + k0 + j] : (i == j ? 1.0 : 0.0);
  }
  __syncwarp();
  for (int c = 0; c < kb; ++c) {
    double d = L11[c][c];
    if (!(d > 0.0)) {
      if (t == c) *bad = 1;
      d = 1.0;
    }
    const double sd = sqrt(d);
    __syncwarp();
    if (t == c) L11[c][c] = sd;
    if (t > c && t < kb) L11[t][c] /= sd;
    __syncwarp();
    if (t > c && t < kb)
      for (int j = c + 1; j <= t; ++j) L11[t][j] -= L11[t][c] * L11[j][c];
    __syncwarp();
  }
  if (t < kb)
    for (int j = 0; j < kb; ++j) A[(k0 + t) * n + k0 + j] = j <= t ? L11[t][j] : 0.0;
}

// Rows below the factored diagonal block: every thread takes one row and
// solves x L11^T = A[row, panel] by forward substitution, in place.
__global__ void __launch_bounds__(CH_ROWS)
    k_chol_panel(double* __restrict__ A, int64_t n, int64_t k0, int kb) {
  __shared__ double L11[CH_NB][CH_NB + 1];
  const int t = threadIdx.x;
  for (int e = t; e < CH_NB * CH_NB; e += blockDim.x) {
    const int i = e / CH_NB, j = e % CH_NB;
    L11[i][j] = (i < kb && j <= i) ? A[(k0 + i) * n + k0 + j] : (i == j ? 1.0 : 0.0);
  }
  __syncthreads();
  const int64_t row = k0 + kb + (int64_t)blockIdx.x * CH_ROWS + t;
  if (row >= n) return;
  double* Ar = A + row * n + k0;
  double x[CH_NB];
#pragma unroll
  for (int j = 0; j < CH_NB; ++j) {
    x[j] = 0.0;
    if (j < kb) {
      double v = Ar[j];
#pragma unroll
      for (int q = 0; q < j; ++q) v -= x[q] * L11[j][q];
      x[j] = v / L11[j][j];
    }
  }
#pragma unroll
  for (int j = 0; j < CH_NB; ++j)
    if (j < kb) Ar[j] = x[j];
}

// out (M x kb, contiguous) = -A[r0.., c0 .. c0 + kb)
__global__ void k_neg_panel(const double* __restrict__ A, int64_t n, int64_t r0, int64_t c0,
                            int64_t M, int kb, double* __restrict__ out) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < M * kb;
       e += (int64_t)gridDim.x * blockDim.x)
    out[e] = -A[(r0 + e / kb) * n + c0 + e % kb];
}

// B = L diag(L)^-1 (fp32, n x n, zero above the diagonal) and, per tile of
// CD_TILE columns, the tile's diagonal block of B^T (unit upper):
// Ud[tile][j][c] = B[c][j] for columns j, c of the tile.
__global__ void k_ldlq_factors(const double* __restrict__ Lf, int64_t n, float* __restrict__ Bl,
                               float* __restrict__ Ud) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * n;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = e / n, j = e % n;
    const float v = j < c ? (float)(Lf[e] / Lf[j * n + j]) : (j == c ? 1.0f : 0.0f);
    Bl[e] = v;
    if (c / CD_TILE == j / CD_TILE)
      Ud[(j / CD_TILE) * CD_TILE * CD_TILE + (j % CD_TILE) * CD_TILE + c % CD_TILE] = v;
  }
}

// One tile [t0, t0 + tw) of the greedy pass for a warp per row.  Lane l holds
// columns l, l + 32, l + 64, l + 96 of the working row v (W plus the feedback
// of every earlier tile).  Column j: its owner rounds v_j to the nearest level
// (the lower on an exact half, clamped to the grid), the error e = v_j - q_j
// goes to all lanes, and every later column moves by -e B[c, j] (row j of the
// tile's unit upper block: 1 on the diagonal, zeros before it, so the owner's
// own value just becomes q_j).  The errors leave as e / aref in the A operand
// (aref = the row's scale, or its largest group scale), with -aref as the
// operand's row factor.
__global__ void __launch_bounds__(LQ_WARPS * 32, 2)
    k_ldlq_tile(int64_t m, int64_t n, int L, int64_t t0, int tw, const float* __restrict__ scale,
                const float* __restrict__ offset, int ng, int gi, const float* __restrict__ sref,
                const float* __restrict__ Ud_tile, const float* __restrict__ Wk, int64_t ldw,
                uint16_t* __restrict__ idx, __half* __restrict__ dhi, __half* __restrict__ dlo,
                int64_t lda, float* __restrict__ d_unscale) {
  extern __shared__ float lq_smem[];
  {
    const float4* src = reinterpret_cast<const float4*>(Ud_tile);
    float4* dst = reinterpret_cast<float4*>(lq_smem);
    for (int e = threadIdx.x; e < CD_TILE * CD_TILE / 4; e += blockDim.x) dst[e] = src[e];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * LQ_WARPS + wid;
  if (row >= m) return;
  const float sc = scale[row * ng + gi], off = offset[row * ng + gi];
  const float aref = sref ? sref[row] : sc;
  const float inv_a = 1.0f / aref;
  if (lane == 0) d_unscale[row] = -aref;
  const float* wr = Wk + row * ldw + t0;
  const float Lm1 = (float)(L - 1);
  float v[LQ_SLOTS], a[LQ_SLOTS];
  int k[LQ_SLOTS];
#pragma unroll
  for (int q = 0; q < LQ_SLOTS; ++q) {
    const int col = 32 * q + lane;
    v[q] = col < tw ? wr[col] : 0.0f;
    a[q] = 0.0f;
    k[q] = 0;
  }
#pragma unroll
  for (int q = 0; q < LQ_SLOTS; ++q) {
    if (32 * q >= tw) break;
    const int cnt = min(32, tw - 32 * q);
    for (int jj = 0; jj < cnt; ++jj) {
      float e = 0.0f;
      if (lane == jj) {
        const float t = (v[q] - off) / sc;
        const float kk = fminf(fmaxf(ceil_small(t - 0.5f), 0.0f), Lm1);
        k[q] = (int)kk;
        e = v[q] - fmaf(sc, kk, off);
        a[q] = e * inv_a;
      }
      e = __shfl_sync(0xffffffffu, e, jj);
      const float* Uj = lq_smem + (32 * q + jj) * CD_TILE + lane;
#pragma unroll
      for (int qq = q; qq < LQ_SLOTS; ++qq) v[qq] = fmaf(-e, Uj[32 * qq], v[qq]);
    }
  }
  uint16_t* ir = idx + row * n + t0;
  __half* drow_hi = dhi + row * lda;
  __half* drow_lo = dlo + row * lda;
#pragma unroll
  for (int q = 0; q < LQ_SLOTS; ++q) {
    const int col = 32 * q + lane;
    if (col < tw) ir[col] = (uint16_t)k[q];
    const __half h = __float2half_rn(a[q]);
    drow_hi[col] = h;
    drow_lo[col] = __float2half_rn(a[q] - __half2float(h));
  }
}

// ---------------------------------------------------------------- d = 8 --
// Block b of a tile: the codeword nearest (Euclidean, in codebook units) the
// block's current working values, t = v_b / scale: argmin_c 1/2 |c|^2 - c.t
// (lowest index on ties).  Kernel A scans one chunk of LQ8_CHUNK codewords
// for LQ8_ROWS rows: the chunk sits transposed in shared memory, each warp
// takes groups of 8 rows with the lanes splitting the codewords, so every
// codeword read from shared memory serves 8 rows (8 independent FMA chains).
// Kernel B (a warp per row) combines the chunk minima, commits the codeword,
// and feeds the block's 8 errors, one column after another, to the later
// columns of the tile through the block's 8 rows of B^T.
constexpr int LQ8_CHUNK = 1024;
constexpr int LQ8_ROWS = 256;
constexpr int LQ8_APPLY_WARPS = 16;

__global__ void __launch_bounds__(256)
    k_ldlq8_eval(int64_t m, int K, int64_t b, const float* __restrict__ cb,
                 const float* __restrict__ cb_norm, const float* __restrict__ scale,
                 const float* __restrict__ Wk, int64_t ldw, float* __restrict__ part_val,
                 int* __restrict__ part_idx, int nchunks) {
  __shared__ float scb[8][LQ8_CHUNK];  // transposed: lanes read consecutive codewords
  __shared__ float sq[LQ8_CHUNK];      // 1/2 |c|^2
  __shared__ float st[LQ8_ROWS][8];    // the rows' targets t
  const int chunk = blockIdx.x;
  const int64_t r0 = (int64_t)blockIdx.y * LQ8_ROWS;
  const int c0 = chunk * LQ8_CHUNK;
  const int cn = min(LQ8_CHUNK, K - c0);
  for (int e = threadIdx.x; e < cn * 8; e += blockDim.x) scb[e % 8][e / 8] = cb[(int64_t)c0 * 8 + e];
  for (int e = threadIdx.x; e < cn; e += blockDim.x) sq[e] = 0.5f * cb_norm[c0 + e];
  for (int rl = threadIdx.x; rl < LQ8_ROWS; rl += blockDim.x) {
    const int64_t row = r0 + rl;
    if (row < m) {
      const float inv = 1.0f / scale[row];
#pragma unroll
      for (int i = 0; i < 8; ++i) st[rl][i] = Wk[row * ldw + 8 * b + i] * inv;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) st[rl][i] = 0.0f;
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int grp = w; grp < LQ8_ROWS / 8; grp += blockDim.x / 32) {
    if (r0 + 8 * grp >= m) break;
    float g[8][8];
#pragma unroll
    for (int rr = 0; rr < 8; ++rr)
#pragma unroll
      for (int i = 0; i < 8; ++i) g[rr][i] = st[8 * grp + rr][i];
    float best[8];
    int bidx[8];
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      best[rr] = INFINITY;
      bidx[rr] = 0x7fffffff;
    }
    for (int c = lane; c < cn; c += 32) {
      float cv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) cv[i] = scb[i][c];
      const float q = sq[c];
#pragma unroll
      for (int rr = 0; rr < 8; ++rr) {
        float sc = q;
#pragma unroll
        for (int i = 0; i < 8; ++i) sc = fmaf(-cv[i], g[rr][i], sc);
        if (sc < best[rr]) {
          best[rr] = sc;
          bidx[rr] = c0 + c;
        }
      }
    }
    // warp minimum per row, lowest index on ties
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      float v = best[rr];
      int k = bidx[rr];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
        const int k2 = __shfl_xor_sync(0xffffffffu, k, o);
        if (v2 < v || (v2 == v && k2 < k)) {
          v = v2;
          k = k2;
        }
      }
      const int64_t row = r0 + 8 * grp + rr;
      if (lane == 0 && row < m) {
        part_val[row * nchunks + chunk] = v;
        part_idx[row * nchunks + chunk] = k;
      }
    }
  }
}

__global__ void __launch_bounds__(LQ8_APPLY_WARPS * 32)
    k_ldlq8_apply(int64_t m, int64_t n, int K, int64_t b, int64_t t0, int tw,
                  const float* __restrict__ cb, const float* __restrict__ scale,
                  const float* __restrict__ Ud_tile, float* __restrict__ Wk, int64_t ldw,
                  uint16_t* __restrict__ idx, const float* __restrict__ part_val,
                  const int* __restrict__ part_idx, int nchunks, __half* __restrict__ dhi,
                  __half* __restrict__ dlo, int64_t lda, float* __restrict__ d_unscale) {
  __shared__ float s_u[8][CD_TILE];  // the block's rows of the tile's unit upper block
  const int jl0 = (int)(8 * b - t0);  // tile-local first column of the block
  for (int e = threadIdx.x; e < 8 * CD_TILE; e += blockDim.x)
    s_u[e / CD_TILE][e % CD_TILE] = Ud_tile[(int64_t)(jl0 + e / CD_TILE) * CD_TILE + e % CD_TILE];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * LQ8_APPLY_WARPS + (threadIdx.x >> 5);
  if (row >= m) return;
  const float sc = scale[row];
  const float inv = 1.0f / sc;
  __half* drow_hi = dhi + row * lda;
  __half* drow_lo = dlo + row * lda;
  if (jl0 == 0) {  // first block of the tile: clear the operand row (zeros past tw)
    for (int i = lane; i < CD_TILE; i += 32) {
      drow_hi[i] = __float2half_rn(0.0f);
      drow_lo[i] = __float2half_rn(0.0f);
    }
    if (lane == 0) d_unscale[row] = -sc;
  }
  float v = INFINITY;
  int k = 0x7fffffff;
  for (int c = lane; c < nchunks; c += 32) {
    const float v2 = part_val[row * nchunks + c];
    const int k2 = part_idx[row * nchunks + c];
    if (v2 < v || (v2 == v && k2 < k)) {
      v = v2;
      k = k2;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
    const int k2 = __shfl_xor_sync(0xffffffffu, k, o);
    if (v2 < v || (v2 == v && k2 < k)) {
      v = v2;
      k = k2;
    }
  }
  k = min(max(k, 0), K - 1);
  // working values of the tile's columns from this block on
  float* wr = Wk + row * ldw + t0;
  float w[LQ_SLOTS];
#pragma unroll
  for (int q = 0; q < LQ_SLOTS; ++q) {
    const int col = 32 * q + lane;
    w[q] = (col >= jl0 && col < tw) ? wr[col] : 0.0f;
  }
  // the block's columns, one after another: error e_j = v_j - scale c_j
#pragma unroll
  for (int jj = 0; jj < 8; ++jj) {
    const int j = jl0 + jj;
    const int owner = j & 31, slot = j >> 5;
    float vj = 0.0f;
#pragma unroll
    for (int q = 0; q < LQ_SLOTS; ++q)
      if (q == slot) vj = w[q];
    const float e = __shfl_sync(0xffffffffu, vj, owner) - sc * cb[(int64_t)k * 8 + jj];
#pragma unroll
    for (int q = 0; q < LQ_SLOTS; ++q) w[q] = fmaf(-e, s_u[jj][32 * q + lane], w[q]);
    if (lane == jj) {
      const float a = e * inv;
      const __half h = __float2half_rn(a);
      drow_hi[j] = h;
      drow_lo[j] = __float2half_rn(a - __half2float(h));
    }
  }
#pragma unroll
  for (int q = 0; q < LQ_SLOTS; ++q) {
    const int col = 32 * q + lane;
    if (col >= jl0 + 8 && col < tw) wr[col] = w[q];
  }
  if (lane == 0) idx[row * (n / 8) + b] = (uint16_t)k;
}

}  // namespace

mpq_status ldlq_factor(const mpq_plan_s* p, double damp, float* Bl, float* Ud, cudaStream_t st) {
  const int64_t n = p->n, r = p->r;
  std::vector<double> hs(r);
  MPQ_CUDA(cudaMemcpyAsync(hs.data(), p->s64, sizeof(double) * r, cudaMemcpyDeviceToHost, st));
  MPQ_CUDA(cudaStreamSynchronize(st));
  double tr = 0.0;  // trace(H) = sum s^2 (V has orthonormal columns)
  for (double v : hs) tr += v * v;
  const double lam = damp * tr / (double)n;
  if (!(lam > 0.0) && r < n)
    return fail(MPQ_ERR_RANK, "greedy baseline: H is singular (rank < n); set greedy_damp > 0");
  const bool full = r == n;
  double *Vc = nullptr, *A = nullptr, *neg = nullptr;
  int* bad = nullptr;
  mpq_status rc = MPQ_OK;
  auto cuda_ok = [&](cudaError_t e, const char* what) {
    if (rc == MPQ_OK && e != cudaSuccess) rc = cuda_fail(e, what);
    return rc == MPQ_OK;
  };
  cuda_ok(cudaMallocAsync(&Vc, sizeof(double) * n * r, st), "ldlq alloc");
  cuda_ok(cudaMallocAsync(&A, sizeof(double) * n * n, st), "ldlq alloc");
  cuda_ok(cudaMallocAsync(&neg, sizeof(double) * n * CH_NB, st), "ldlq alloc");
  cuda_ok(cudaMallocAsync(&bad, sizeof(int), st), "ldlq alloc");
  if (rc == MPQ_OK) cuda_ok(cudaMemsetAsync(bad, 0, sizeof(int), st), "ldlq memset");
  if (rc == MPQ_OK) {
    {
      ProfScope ps_("k_hinv_cols", st);
      k_hinv_cols<<<grid_for(n * r), 256, 0, st>>>(p->V64, p->s64, n, r, lam, full ? 1 : 0, Vc);
    }
    count_launch();
    rc = check_launch("k_hinv_cols");
  }
  if (rc == MPQ_OK) rc = gemm_nt_f64(Vc, r, p->V64, r, A, n, n, n, r, st);  // V diag(c) V^T
  if (rc == MPQ_OK && !full) {
    {
      ProfScope ps_("k_add_diag", st);
      k_add_diag<<<(unsigned)cdiv(n, 256), 256, 0, st>>>(A, n, 1.0 / lam);
    }
    count_launch();
    rc = check_launch("k_add_diag");
  }
  for (int64_t k0 = 0; k0 < n && rc == MPQ_OK; k0 += CH_NB) {
    const int kb = (int)std::min<int64_t>(CH_NB, n - k0);
    {
      ProfScope ps_("k_chol_diag", st);
      k_chol_diag<<<1, 32, 0, st>>>(A, n, k0, kb, bad);
    }
    count_launch();
    rc = check_launch("k_chol_diag");
    const int64_t r0 = k0 + kb, M = n - r0;
    if (rc != MPQ_OK || M <= 0) continue;
    {
      ProfScope ps_("k_chol_panel", st);
      k_chol_panel<<<(unsigned)cdiv(M, CH_ROWS), CH_ROWS, 0, st>>>(A, n, k0, kb);
    }
    count_launch();
    rc = check_launch("k_chol_panel");
    if (rc != MPQ_OK) continue;
    {
      ProfScope ps_("k_neg_panel", st);
      k_neg_panel<<<grid_for(M * kb), 256, 0, st>>>(A, n, r0, k0, M, kb, neg);
    }
    count_launch();
    rc = check_launch("k_neg_panel");
    // A22 += (-L21) L21^T
    if (rc == MPQ_OK)
      rc = gemm_nt_f64(neg, kb, A + r0 * n + k0, n, A + r0 * n + r0, n, M, M, kb, st, true);
  }
  if (rc == MPQ_OK) {
    {
      ProfScope ps_("k_ldlq_factors", st);
      k_ldlq_factors<<<grid_for(n * n), 256, 0, st>>>(A, n, Bl, Ud);
    }
    count_launch();
    rc = check_launch("k_ldlq_factors");
  }
  int hbad = 0;
  if (rc == MPQ_OK) cuda_ok(cudaMemcpyAsync(&hbad, bad, sizeof(int), cudaMemcpyDeviceToHost, st), "ldlq flag");
  if (rc == MPQ_OK) cuda_ok(cudaStreamSynchronize(st), "ldlq sync");
  if (Vc) cudaFreeAsync(Vc, st);
  if (A) cudaFreeAsync(A, st);
  if (neg) cudaFreeAsync(neg, st);
  if (bad) cudaFreeAsync(bad, st);
  if (rc == MPQ_OK && hbad)
    return fail(MPQ_ERR_RANK, "greedy baseline: (H + lambda I)^-1 is not positive definite in fp64");
  return rc;
}

mpq_status launch_ldlq(mpq_plan_s* p, const float* W, int64_t m, const float* scale,
                       const float* offset, uint16_t* idx, cudaStream_t st) {
  if (m <= 0) return MPQ_OK;
  if (!p->ldlq_diag) return fail(MPQ_ERR_INVALID_ARG, "the plan was created without greedy_init");
  Workspace& w = p->ws;
  const int64_t n = p->n;
  // working rows W_work = W, in the CD gradient buffer (free until CD starts)
  MPQ_CUDA(cudaMemcpy2DAsync(w.Hg, sizeof(float) * w.ldh, W, sizeof(float) * n, sizeof(float) * n,
                             m, cudaMemcpyDeviceToDevice, st));
  if (p->G) MPQ_TRY(launch_row_max(scale, m, p->ng, w.sref, st));
  const int64_t P = p->params.cd_panel > 0 ? std::min<int64_t>(p->params.cd_panel, round_up(n, CD_TILE))
                                           : cd_panel_cols(m, n);
  const int np = (int)cdiv(n, P);
  MPQ_CUDA(cudaFuncSetAttribute(k_ldlq_tile, cudaFuncAttributeMaxDynamicSharedMemorySize, LQ_SMEM));
  // d = 8: per-row minima of the nearest-codeword scan over slices of the
  // codebook (tensor cores for lattice codebooks, else SIMT chunks)
  const bool tc = p->d == 8 && p->vec_tc;
  const int nchunks = p->d != 8 ? 0 : tc ? cd_scan_slices(m, p->K) : (int)cdiv(p->K, LQ8_CHUNK);
  float* part_val = nullptr;
  int* part_idx = nullptr;
  if (p->d == 8) {
    if (!p->cb_norm) return fail(MPQ_ERR_INVALID_ARG, "the plan has no codebook tables");
    MPQ_CUDA(cudaMallocAsync(&part_val, sizeof(float) * m * nchunks, st));
    MPQ_CUDA(cudaMallocAsync(&part_idx, sizeof(int) * m * nchunks, st));
  }
  mpq_status rc = MPQ_OK;
  auto update = [&](int64_t a_k0, int64_t b_k0, int64_t K, int64_t c0, int64_t c1,
                    const char* tag) -> mpq_status {
    if (c1 <= c0) return MPQ_OK;
    GemmOpts o;
    o.a_k0 = a_k0;
    o.b_k0 = b_k0;
    o.n0 = c0;
    o.accumulate = true;
    o.c_reduce = &w.tm_hg;
    return gemm_tc(w.As, w.tm_an_hi, w.tm_an_lo, p->Lq_s, p->tm_lq_hi, p->tm_lq_lo, w.Hg, w.ldh, m,
                   c1 - c0, K, p->Lq_s.unscale_host, p->status, st, tag, o);
  };
  for (int pi = 0; pi < np && rc == MPQ_OK; ++pi) {
    const int64_t ps = (int64_t)pi * P, pe = std::min<int64_t>(n, ps + P);
    for (int64_t t0 = ps; t0 < pe && rc == MPQ_OK; t0 += CD_TILE) {
      const int tw = (int)std::min<int64_t>(CD_TILE, n - t0);
      const float* Ud = p->ldlq_diag + (t0 / CD_TILE) * CD_TILE * CD_TILE;
      __half* dhi = w.As.hi + (t0 - ps);
      __half* dlo = w.As.lo + (t0 - ps);
      if (p->d == 1) {
        {
          ProfScope ps_("k_ldlq_tile", st);
          k_ldlq_tile<<<(unsigned)cdiv(m, LQ_WARPS), LQ_WARPS * 32, LQ_SMEM, st>>>(
              m, n, p->K, t0, tw, scale, offset, (int)p->ng, p->G ? (int)(t0 / p->G) : 0,
              p->G ? w.sref : nullptr, Ud, w.Hg, w.ldh, idx, dhi, dlo, w.As.ld, w.As.row_unscale);
        }
        count_launch();
        rc = check_launch("k_ldlq_tile");
      } else {
        for (int64_t b = t0 / 8; b < (t0 + tw) / 8 && rc == MPQ_OK; ++b) {
          if (tc) {
            rc = launch_ldlq_vec_scan(p, m, b, scale, w.Hg, w.ldh, part_val, part_idx, nchunks, st);
            if (rc != MPQ_OK) break;
          } else {
            ProfScope ps_("k_ldlq8_eval", st);
            dim3 ge((unsigned)nchunks, (unsigned)cdiv(m, LQ8_ROWS));
            k_ldlq8_eval<<<ge, LQ8_ROWS, 0, st>>>(m, p->K, b, p->cb, p->cb_norm, scale, w.Hg,
                                                  w.ldh, part_val, part_idx, nchunks);
          }
          {
            ProfScope ps_("k_ldlq8_apply", st);
            k_ldlq8_apply<<<(unsigned)cdiv(m, LQ8_APPLY_WARPS), LQ8_APPLY_WARPS * 32, 0, st>>>(
                m, n, p->K, b, t0, tw, p->cb, scale, Ud, w.Hg, w.ldh, idx, part_val, part_idx,
                nchunks, dhi, dlo, w.As.ld, w.As.row_unscale);
          }
          count_launch(tc ? 1 : 2);
          rc = check_launch("k_ldlq8");
        }
      }
      // later columns of the panel
      if (rc == MPQ_OK) rc = update(t0 - ps, t0, tw, t0 + tw, pe, "gemm_ldlq_update");
    }
    // every column after the panel
    if (rc == MPQ_OK && np > 1) rc = update(0, ps, pe - ps, pe, n, "gemm_ldlq_panel");
  }
  if (part_val) cudaFreeAsync(part_val, st);
  if (part_idx) cudaFreeAsync(part_idx, st);
  return rc;
}

}  // namespace mpq
