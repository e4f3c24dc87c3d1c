// Setup: the compact SVD of the calibration activations X through the
// smaller Gram matrix, on the device, in fp64.
//
// Source: "MPQ: A Message-Passing View of Post-Training Quantization"
// (papernotes.org note), key design 1 and the flowchart: A = X = U Sigma V^T
// (compact), T = Sigma V^T in the rank space r = rank(A).
//
// Eigensolver: the cyclic Jacobi method for symmetric matrices with the
// parallel round-robin ("tournament") ordering of Brent and Luk; each 2x2
// rotation is the symmetric Schur decomposition of Golub & Van Loan,
// Matrix Computations, section 8.5 (Jacobi methods).  In round k the pairs
// are (0, 1 + k) and (1 + (k+i) mod (N-1), 1 + (k-i) mod (N-1)); both index
// runs are contiguous in i, so every round streams the matrix with coalesced
// accesses.  Rank cut: lambda > lambda_max * max(m, n) * 2^-52.
#include <math.h>

#include <vector>

#include "mpq_internal.cuh"

namespace mpq {
namespace {

constexpr int JACOBI_MAX_SWEEPS = 40;

__device__ __forceinline__ void rr_pair(int64_t N, int64_t k, int64_t i, int64_t* p, int64_t* q) {
  if (i == 0) {
    *p = 0;
    *q = 1 + k;
  } else {
    const int64_t M = N - 1;
    *p = 1 + (k + i) % M;
    *q = 1 + ((k - i) % M + M) % M;
  }
}

__global__ void k_jacobi_rot(const double* __restrict__ A, int64_t N, int64_t k,
                             double* __restrict__ cs) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N / 2) return;
  int64_t p, q;
  rr_pair(N, k, i, &p, &q);
  const double app = A[p * N + p], aqq = A[q * N + q], apq = A[p * N + q];
  double c = 1.0, s = 0.0;
  if (apq != 0.0 && fabs(apq) > 1e-300) {
    const double tau = (aqq - app) / (2.0 * apq);
    const double t = (tau >= 0.0) ? 1.0 / (tau + sqrt(1.0 + tau * tau))
                                   : -1.0 / (-tau + sqrt(1.0 + tau * tau));
    c = 1.0 / sqrt(1.0 + t * t);
    s = t * c;
  }
  cs[2 * i] = c;
  cs[2 * i + 1] = s;
}

// A <- J^T A J on all 2x2 blocks (pair I rows, pair J cols)
__global__ void k_jacobi_apply(double* __restrict__ A, int64_t N, int64_t k,
                               const double* __restrict__ cs) {
  const int64_t half = N / 2;
  const int64_t J = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t I = blockIdx.y;
  if (J >= half) return;
  int64_t pI, qI, pJ, qJ;
  rr_pair(N, k, I, &pI, &qI);
  rr_pair(N, k, J, &pJ, &qJ);
  const double cI = cs[2 * I], sI = cs[2 * I + 1];
  const double cJ = cs[2 * J], sJ = cs[2 * J + 1];
  const double m00 = A[pI * N + pJ], m01 = A[pI * N + qJ];
  const double m10 = A[qI * N + pJ], m11 = A[qI * N + qJ];
  // M R_J
  const double a00 = cJ * m00 - sJ * m01, a01 = sJ * m00 + cJ * m01;
  const double a10 = cJ * m10 - sJ * m11, a11 = sJ * m10 + cJ * m11;
  // R_I^T (M R_J)
  double b00 = cI * a00 - sI * a10, b01 = cI * a01 - sI * a11;
  double b10 = sI * a00 + cI * a10, b11 = sI * a01 + cI * a11;
  if (I == J) {
    b01 = 0.0;
    b10 = 0.0;
  }
  A[pI * N + pJ] = b00;
  A[pI * N + qJ] = b01;
  A[qI * N + pJ] = b10;
  A[qI * N + qJ] = b11;
}

// V <- V J  (columns p, q of every row)
__global__ void k_jacobi_vec(double* __restrict__ V, int64_t N, int64_t k,
                             const double* __restrict__ cs) {
  const int64_t J = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t row = blockIdx.y;
  if (J >= N / 2) return;
  int64_t p, q;
  rr_pair(N, k, J, &p, &q);
  const double c = cs[2 * J], s = cs[2 * J + 1];
  const double vp = V[row * N + p], vq = V[row * N + q];
  V[row * N + p] = c * vp - s * vq;
  V[row * N + q] = s * vp + c * vq;
}

__global__ void k_offdiag(const double* __restrict__ A, int64_t N, double* __restrict__ out) {
  __shared__ double so[256], sd[256];
  double off = 0.0, dg = 0.0;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < N * N;
       e += (int64_t)gridDim.x * blockDim.x) {
    const double v = A[e];
    if (e / N == e % N) dg += v * v;
    else off += v * v;
  }
  so[threadIdx.x] = off;
  sd[threadIdx.x] = dg;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) {
      so[threadIdx.x] += so[threadIdx.x + s];
      sd[threadIdx.x] += sd[threadIdx.x + s];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    out[2 * blockIdx.x] = so[0];
    out[2 * blockIdx.x + 1] = sd[0];
  }
}

// ----------------------------------------------------- blocked Jacobi --
// The same cyclic Jacobi method on blocks (Golub & Van Loan, section 8.5,
// block Jacobi): the columns form blocks of BJ_B, block pairs follow the
// round-robin ordering above, and in every round each pair's 2BJ_B x 2BJ_B
// diagonal submatrix gets one cyclic sweep of 2x2 rotations (k_bj_inner, in
// shared memory), whose product Q_I is then applied to the whole matrix at
// once: A <- Q^T A Q tile by tile (k_bj_apply_a, tiles of rows of pair I and
// columns of pair J: Q_I^T A_IJ Q_J) and V <- V Q (k_bj_apply_v).  A round
// thus moves A and V through memory once instead of once per 2x2 round.
constexpr int BJ_B = 32, BJ_P = 2 * BJ_B;  // block and pair width
constexpr int BJ_LD = BJ_P + 2;            // padded rows of the product tiles (16-byte aligned)
constexpr int BJ_TILE = BJ_P * BJ_LD;      // doubles per shared tile
constexpr int BJ_LDI = BJ_P + 1;           // rows of the rotation tiles: odd, so that a column
                                           // read by 32 lanes touches every bank pair once

__device__ __forceinline__ void bj_pair_index(int64_t nb, int64_t k, int64_t pi, int* gi) {
  int64_t p, q;
  rr_pair(nb, k, pi, &p, &q);
  for (int t = 0; t < BJ_P; ++t) gi[t] = (int)(t < BJ_B ? p * BJ_B + t : q * BJ_B + t - BJ_B);
}

// One sweep of the 2x2 cyclic Jacobi on the pair's submatrix; Q (64 x 64,
// row-major) is the product of its rotations.
__global__ void __launch_bounds__(256)
    k_bj_inner(const double* __restrict__ A, int64_t N, int64_t nb, int64_t k,
               double* __restrict__ Qout) {
  extern __shared__ double bj_in[];
  double(*S)[BJ_LDI] = reinterpret_cast<double(*)[BJ_LDI]>(bj_in);
  double(*Q)[BJ_LDI] = reinterpret_cast<double(*)[BJ_LDI]>(bj_in + BJ_P * BJ_LDI);
  __shared__ double cs[BJ_B][2];
  __shared__ int pr[BJ_B][2];
  __shared__ int gi[BJ_P];
  const int t = threadIdx.x;
  if (t == 0) bj_pair_index(nb, k, blockIdx.x, gi);
  __syncthreads();
  for (int e = t; e < BJ_P * BJ_P; e += blockDim.x) {
    const int i = e / BJ_P, j = e % BJ_P;
    S[i][j] = A[(int64_t)gi[i] * N + gi[j]];
    Q[i][j] = (i == j) ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int kk = 0; kk < BJ_P - 1; ++kk) {
    if (t < BJ_B) {
      int64_t pp, qq;
      rr_pair(BJ_P, kk, t, &pp, &qq);
      const double app = S[pp][pp], aqq = S[qq][qq], apq = S[pp][qq];
      double c = 1.0, sn = 0.0;
      if (apq != 0.0 && fabs(apq) > 1e-300) {
        const double tau = (aqq - app) / (2.0 * apq);
        const double tt = (tau >= 0.0) ? 1.0 / (tau + sqrt(1.0 + tau * tau))
                                       : -1.0 / (-tau + sqrt(1.0 + tau * tau));
        c = 1.0 / sqrt(1.0 + tt * tt);
        sn = tt * c;
      }
      cs[t][0] = c;
      cs[t][1] = sn;
      pr[t][0] = (int)pp;
      pr[t][1] = (int)qq;
    }
    __syncthreads();
    for (int e = t; e < BJ_B * BJ_P; e += blockDim.x) {  // rows: J^T S
      const int r = e / BJ_P, j = e % BJ_P;
      const int pp = pr[r][0], qq = pr[r][1];
      const double c = cs[r][0], sn = cs[r][1];
      const double sp = S[pp][j], sq = S[qq][j];
      S[pp][j] = c * sp - sn * sq;
      S[qq][j] = sn * sp + c * sq;
    }
    __syncthreads();
    for (int e = t; e < BJ_B * BJ_P; e += blockDim.x) {  // columns: (J^T S) J, and Q J
      const int r = e / BJ_P, i = e % BJ_P;
      const int pp = pr[r][0], qq = pr[r][1];
      const double c = cs[r][0], sn = cs[r][1];
      const double sp = S[i][pp], sq = S[i][qq];
      S[i][pp] = c * sp - sn * sq;
      S[i][qq] = sn * sp + c * sq;
      const double qp = Q[i][pp], qv = Q[i][qq];
      Q[i][pp] = c * qp - sn * qv;
      Q[i][qq] = sn * qp + c * qv;
    }
    __syncthreads();
    if (t < BJ_B) S[pr[t][0]][pr[t][1]] = S[pr[t][1]][pr[t][0]] = 0.0;  // annihilated
    __syncthreads();
  }
  double* qo = Qout + (int64_t)blockIdx.x * BJ_P * BJ_P;
  for (int e = t; e < BJ_P * BJ_P; e += blockDim.x) qo[e] = Q[e / BJ_P][e % BJ_P];
}

// 64 x 64 x 64 products in shared memory, acc = (Xt^T Y) block (Xt holds X
// transposed, so that both operands are read along rows): each of 256
// threads owns a 4 x 4 block of the result, rows ti.., columns tj.., and
// reads 4 + 4 values per k as 16-byte loads.
constexpr int BJ_THREADS = 256;
__device__ __forceinline__ void bj_mm(const double (*Xt)[BJ_LD], const double (*Y)[BJ_LD],
                                      double (&acc)[4][4]) {
  const int ti = (threadIdx.x / 16) * 4, tj = (threadIdx.x % 16) * 4;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
#pragma unroll 4
  for (int kk = 0; kk < BJ_P; ++kk) {
    const double2 x0 = *reinterpret_cast<const double2*>(&Xt[kk][ti]);
    const double2 x1 = *reinterpret_cast<const double2*>(&Xt[kk][ti + 2]);
    const double2 y0 = *reinterpret_cast<const double2*>(&Y[kk][tj]);
    const double2 y1 = *reinterpret_cast<const double2*>(&Y[kk][tj + 2]);
    const double xv[4] = {x0.x, x0.y, x1.x, x1.y}, yv[4] = {y0.x, y0.y, y1.x, y1.y};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fma(xv[a], yv[b], acc[a][b]);
  }
}

// a thread's 4 x 4 result block to rows gr[ti + a], columns gc[tj .. tj+3] of
// M (the 4 columns lie in one 32-column block: two 16-byte stores per row)
__device__ __forceinline__ void bj_store(double* __restrict__ M, int64_t N, const int* gr,
                                         int64_t r0, const int* gc, const double (&acc)[4][4]) {
  const int ti = (threadIdx.x / 16) * 4, tj = (threadIdx.x % 16) * 4;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    double* dst = M + (gr ? (int64_t)gr[ti + a] : r0 + ti + a) * N + gc[tj];
    *reinterpret_cast<double2*>(dst) = make_double2(acc[a][0], acc[a][1]);
    *reinterpret_cast<double2*>(dst + 2) = make_double2(acc[a][2], acc[a][3]);
  }
}

// two tiles of shared memory per CTA: three CTAs (24 warps) fit an SM
constexpr int BJ_APPLY_SMEM = 2 * BJ_TILE * (int)sizeof(double);

// A[rows of pair I, cols of pair J] <- Q_I^T A_IJ Q_J (the tiles partition A):
// U = Q_I^T T into registers, U^T over Q_I's tile, Q_J over T's, then U Q_J
// straight to A
__global__ void __launch_bounds__(BJ_THREADS)
    k_bj_apply_a(double* __restrict__ A, int64_t N, int64_t nb, int64_t k,
                 const double* __restrict__ Qall) {
  extern __shared__ __align__(16) double bj_sm[];
  double(*X)[BJ_LD] = reinterpret_cast<double(*)[BJ_LD]>(bj_sm);
  double(*Y)[BJ_LD] = reinterpret_cast<double(*)[BJ_LD]>(bj_sm + BJ_TILE);
  __shared__ int gI[BJ_P], gJ[BJ_P];
  const int t = threadIdx.x;
  if (t == 0) {
    bj_pair_index(nb, k, blockIdx.y, gI);
    bj_pair_index(nb, k, blockIdx.x, gJ);
  }
  __syncthreads();
  const double* qi = Qall + (int64_t)blockIdx.y * BJ_P * BJ_P;
  const double* qj = Qall + (int64_t)blockIdx.x * BJ_P * BJ_P;
  for (int e = t; e < BJ_P * BJ_P; e += blockDim.x) {
    const int i = e / BJ_P, j = e % BJ_P;
    X[i][j] = qi[e];
    Y[i][j] = A[(int64_t)gI[i] * N + gJ[j]];
  }
  __syncthreads();
  double acc[4][4];
  bj_mm(X, Y, acc);  // U = Q_I^T T
  __syncthreads();
  const int ti = (t / 16) * 4, tj = (t % 16) * 4;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) X[tj + b][ti + a] = acc[a][b];  // U^T
  for (int e = t; e < BJ_P * BJ_P; e += blockDim.x) Y[e / BJ_P][e % BJ_P] = qj[e];
  __syncthreads();
  bj_mm(X, Y, acc);  // U Q_J
  bj_store(A, N, gI, 0, gJ, acc);
}

// V[rows r0 .. r0+63, cols of pair J] <- V[.., pair J] Q_J
__global__ void __launch_bounds__(BJ_THREADS)
    k_bj_apply_v(double* __restrict__ V, int64_t N, int64_t nb, int64_t k,
                 const double* __restrict__ Qall) {
  extern __shared__ __align__(16) double bj_sm[];
  double(*Tt)[BJ_LD] = reinterpret_cast<double(*)[BJ_LD]>(bj_sm);
  double(*QJ)[BJ_LD] = reinterpret_cast<double(*)[BJ_LD]>(bj_sm + BJ_TILE);
  __shared__ int gJ[BJ_P];
  const int t = threadIdx.x;
  const int64_t r0 = (int64_t)blockIdx.y * BJ_P;
  if (t == 0) bj_pair_index(nb, k, blockIdx.x, gJ);
  __syncthreads();
  const double* qj = Qall + (int64_t)blockIdx.x * BJ_P * BJ_P;
  for (int e = t; e < BJ_P * BJ_P; e += blockDim.x) {
    const int i = e / BJ_P, j = e % BJ_P;
    Tt[j][i] = V[(r0 + i) * N + gJ[j]];  // the tile, transposed
    QJ[i][j] = qj[e];
  }
  __syncthreads();
  double acc[4][4];
  bj_mm(Tt, QJ, acc);  // T Q_J
  bj_store(V, N, nullptr, r0, gJ, acc);
}

__global__ void k_eye(double* V, int64_t N) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < N * N;
       e += (int64_t)gridDim.x * blockDim.x)
    V[e] = (e / N == e % N) ? 1.0 : 0.0;
}

// fp32 m x n -> fp64, optionally transposed (out n x m), zero-padded to Np
__global__ void k_x_to_f64(const float* __restrict__ X, int64_t m, int64_t n, int transpose,
                           double* __restrict__ out) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < m * n;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / n, j = e % n;
    if (transpose) out[j * m + i] = (double)X[e];
    else out[e] = (double)X[e];
  }
}

// copy the N0 x N0 Gram into an N x N zero-padded matrix
__global__ void k_pad(const double* __restrict__ G, int64_t N0, int64_t N, double* __restrict__ A) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < N * N;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / N, j = e % N;
    A[e] = (i < N0 && j < N0) ? G[i * N0 + j] : 0.0;
  }
}

// descending rank of each eigenvalue (ties by index): rank_i = #{j: l_j > l_i or (l_j == l_i and j < i)}
__global__ void k_rank(const double* __restrict__ A, int64_t N, int64_t N0, int* __restrict__ rank) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N0) return;
  const double li = A[i * N + i];
  int r = 0;
  for (int64_t j = 0; j < N0; ++j) {
    const double lj = A[j * N + j];
    r += (lj > li) || (lj == li && j < i);
  }
  rank[i] = r;
}

// eigen-pairs in descending order: lam[rank] and vectors E[:, rank] (E N0 x N0)
__global__ void k_gather_sorted(const double* __restrict__ A, const double* __restrict__ V,
                                int64_t N, int64_t N0, const int* __restrict__ rank,
                                double* __restrict__ lam, double* __restrict__ E) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= N0 * N0) return;
  const int64_t row = e / N0, col = e % N0;
  const int rk = rank[col];
  E[row * N0 + rk] = V[row * N + col];
  if (row == 0) lam[rk] = A[col * N + col];
}

__global__ void k_sqrt_first(const double* __restrict__ lam, int64_t r, double* __restrict__ s) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < r) s[i] = sqrt(fmax(lam[i], 0.0));
}

// first r columns of E (N0 x N0) -> out (N0 x r)
__global__ void k_take_cols(const double* __restrict__ E, int64_t N0, int64_t r, double* __restrict__ out) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= N0 * r) return;
  out[e] = E[(e / r) * N0 + e % r];
}

// Ut (r x m) = E[:, :r]^T
__global__ void k_take_cols_t(const double* __restrict__ E, int64_t N0, int64_t r, double* __restrict__ out) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= N0 * r) return;
  const int64_t l = e / N0, i = e % N0;
  out[e] = E[i * N0 + l];
}

__global__ void k_div_cols(double* __restrict__ V, int64_t n, int64_t r, const double* __restrict__ s) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * r;
       e += (int64_t)gridDim.x * blockDim.x)
    V[e] /= s[e % r];
}

unsigned g1(int64_t count) { return (unsigned)std::min<int64_t>(cdiv(count, 256), 148 * 32); }

template <typename T>
struct DevBuf {
  T* p = nullptr;
  ~DevBuf() {
    if (p) cudaFree(p);
  }
  mpq_status alloc(int64_t count) {
    cudaError_t e = cudaMalloc((void**)&p, sizeof(T) * (size_t)std::max<int64_t>(count, 1));
    if (e != cudaSuccess) {
      cudaGetLastError();
      p = nullptr;
      return fail(MPQ_ERR_OOM, "setup allocation failed");
    }
    return MPQ_OK;
  }
};

// Symmetric eigendecomposition of the N0 x N0 matrix G (device, fp64):
// descending eigenvalues lam (N0) and eigenvectors E (N0 x N0, columns).
mpq_status jacobi_eig_blocked(const double* G, int64_t N0, double* lam, double* E,
                              cudaStream_t st);

mpq_status jacobi_eig(const double* G, int64_t N0, double* lam, double* E, cudaStream_t st) {
  if (N0 >= 256) return jacobi_eig_blocked(G, N0, lam, E, st);
  const int64_t N = N0 + (N0 & 1);  // even; the pad row/col is zero
  DevBuf<double> A, V, cs, red;
  DevBuf<int> rank;
  MPQ_TRY(A.alloc(N * N));
  MPQ_TRY(V.alloc(N * N));
  MPQ_TRY(cs.alloc(N));
  const int red_blocks = 256;
  MPQ_TRY(red.alloc(2 * red_blocks));
  MPQ_TRY(rank.alloc(N0));
  {
    ProfScope ps_("k_pad", st);
    k_pad<<<g1(N * N), 256, 0, st>>>(G, N0, N, A.p);
  }
  {
    ProfScope ps_("k_eye", st);
    k_eye<<<g1(N * N), 256, 0, st>>>(V.p, N);
  }
  count_launch(2);
  MPQ_TRY(check_launch("jacobi init"));
  std::vector<double> h(2 * red_blocks);
  const int64_t half = N / 2;
  bool converged = (N <= 1);
  for (int sweep = 0; sweep < JACOBI_MAX_SWEEPS && !converged; ++sweep) {
    for (int64_t k = 0; k < N - 1; ++k) {
      {
        ProfScope ps_("k_jacobi_rot", st);
        k_jacobi_rot<<<(unsigned)cdiv(half, 256), 256, 0, st>>>(A.p, N, k, cs.p);
      }
      dim3 ga((unsigned)cdiv(half, 128), (unsigned)half);
      {
        ProfScope ps_("k_jacobi_apply", st);
        k_jacobi_apply<<<ga, 128, 0, st>>>(A.p, N, k, cs.p);
      }
      dim3 gv((unsigned)cdiv(half, 128), (unsigned)N);
      {
        ProfScope ps_("k_jacobi_vec", st);
        k_jacobi_vec<<<gv, 128, 0, st>>>(V.p, N, k, cs.p);
      }
      count_launch(3);
    }
    MPQ_TRY(check_launch("jacobi sweep"));
    {
      ProfScope ps_("k_offdiag", st);
      k_offdiag<<<red_blocks, 256, 0, st>>>(A.p, N, red.p);
    }
    count_launch();
    MPQ_CUDA(cudaMemcpyAsync(h.data(), red.p, sizeof(double) * 2 * red_blocks, cudaMemcpyDeviceToHost, st));
    MPQ_CUDA(cudaStreamSynchronize(st));
    double off = 0.0, dg = 0.0;
    for (int b = 0; b < red_blocks; ++b) {
      off += h[2 * b];
      dg += h[2 * b + 1];
    }
    converged = !(off > 1e-28 * dg) || dg == 0.0;
  }
  if (!converged) return fail(MPQ_ERR_TIMEOUT, "Jacobi eigensolver did not converge in 40 sweeps");
  {
    ProfScope ps_("k_rank", st);
    k_rank<<<(unsigned)cdiv(N0, 256), 256, 0, st>>>(A.p, N, N0, rank.p);
  }
  {
    ProfScope ps_("k_gather_sorted", st);
    k_gather_sorted<<<(unsigned)cdiv(N0 * N0, 256), 256, 0, st>>>(A.p, V.p, N, N0, rank.p, lam, E);
  }
  count_launch(2);
  return check_launch("jacobi sort");
}

// Blocked cyclic Jacobi (k_bj_*): N0 padded with zero rows and columns to a
// multiple of the pair width (a zero row never rotates, so the padding stays
// decoupled and the first N0 diagonal entries are G's eigenvalues).
mpq_status jacobi_eig_blocked(const double* G, int64_t N0, double* lam, double* E,
                              cudaStream_t st) {
  const int64_t N = round_up(N0, BJ_P);
  const int64_t nb = N / BJ_B, npairs = nb / 2;
  DevBuf<double> A, V, Q, red;
  DevBuf<int> rank;
  MPQ_TRY(A.alloc(N * N));
  MPQ_TRY(V.alloc(N * N));
  MPQ_TRY(Q.alloc(npairs * BJ_P * BJ_P));
  const int red_blocks = 256;
  MPQ_TRY(red.alloc(2 * red_blocks));
  MPQ_TRY(rank.alloc(N0));
  MPQ_CUDA(cudaFuncSetAttribute(k_bj_inner, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                2 * BJ_TILE * (int)sizeof(double)));
  MPQ_CUDA(cudaFuncSetAttribute(k_bj_apply_a, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                BJ_APPLY_SMEM));
  MPQ_CUDA(cudaFuncSetAttribute(k_bj_apply_v, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                BJ_APPLY_SMEM));
  {
    ProfScope ps_("k_pad", st);
    k_pad<<<g1(N * N), 256, 0, st>>>(G, N0, N, A.p);
  }
  {
    ProfScope ps_("k_eye", st);
    k_eye<<<g1(N * N), 256, 0, st>>>(V.p, N);
  }
  count_launch(2);
  MPQ_TRY(check_launch("jacobi init"));
  std::vector<double> h(2 * red_blocks);
  bool converged = false;
  for (int sweep = 0; sweep < JACOBI_MAX_SWEEPS && !converged; ++sweep) {
    {
      ProfScope ps_("k_offdiag", st);
      k_offdiag<<<red_blocks, 256, 0, st>>>(A.p, N, red.p);
    }
    count_launch();
    MPQ_CUDA(cudaMemcpyAsync(h.data(), red.p, sizeof(double) * 2 * red_blocks, cudaMemcpyDeviceToHost, st));
    MPQ_CUDA(cudaStreamSynchronize(st));
    double off = 0.0, dg = 0.0;
    for (int b = 0; b < red_blocks; ++b) {
      off += h[2 * b];
      dg += h[2 * b + 1];
    }
    converged = !(off > 1e-28 * dg) || dg == 0.0;
    if (converged) break;
    for (int64_t k = 0; k < nb - 1; ++k) {
      {
        ProfScope ps_("k_bj_inner", st);
        k_bj_inner<<<(unsigned)npairs, 256, 2 * BJ_TILE * sizeof(double), st>>>(A.p, N, nb, k, Q.p);
      }
      {
        ProfScope ps_("k_bj_apply_a", st);
        k_bj_apply_a<<<dim3((unsigned)npairs, (unsigned)npairs), BJ_THREADS, BJ_APPLY_SMEM, st>>>(
            A.p, N, nb, k, Q.p);
      }
      {
        ProfScope ps_("k_bj_apply_v", st);
        k_bj_apply_v<<<dim3((unsigned)npairs, (unsigned)(N / BJ_P)), BJ_THREADS, BJ_APPLY_SMEM,
                       st>>>(V.p, N, nb, k, Q.p);
      }
      count_launch(3);
    }
    MPQ_TRY(check_launch("blocked jacobi sweep"));
  }
  if (!converged) return fail(MPQ_ERR_TIMEOUT, "Jacobi eigensolver did not converge in 40 sweeps");
  {
    ProfScope ps_("k_rank", st);
    k_rank<<<(unsigned)cdiv(N0, 256), 256, 0, st>>>(A.p, N, N0, rank.p);
  }
  {
    ProfScope ps_("k_gather_sorted", st);
    k_gather_sorted<<<(unsigned)cdiv(N0 * N0, 256), 256, 0, st>>>(A.p, V.p, N, N0, rank.p, lam, E);
  }
  count_launch(2);
  return check_launch("jacobi sort");
}

// Rank cut on the host from the N0 sorted eigenvalues lam (device):
// r = #{lambda > lambda_max * max(m, n) * 2^-52}; allocates the plan's s64
// (r) and V64 (n x r) and fills s = sqrt(lambda[:r]).
mpq_status cut_and_alloc(mpq_plan_s* p, const double* lam, int64_t N0, int64_t m, int64_t n,
                         cudaStream_t st) {
  std::vector<double> hl(N0);
  MPQ_CUDA(cudaMemcpyAsync(hl.data(), lam, sizeof(double) * N0, cudaMemcpyDeviceToHost, st));
  MPQ_CUDA(cudaStreamSynchronize(st));
  const double tol = (N0 > 0 ? hl[0] : 0.0) * (double)std::max(m, n) * ldexp(1.0, -52);
  int64_t r = 0;
  while (r < N0 && hl[r] > tol) ++r;
  if (r == 0) return fail(MPQ_ERR_RANK, "X has rank 0");
  p->r = r;
  cudaError_t e1 = cudaMalloc((void**)&p->s64, sizeof(double) * r);
  cudaError_t e2 = cudaMalloc((void**)&p->V64, sizeof(double) * n * r);
  if (e1 != cudaSuccess || e2 != cudaSuccess) {
    cudaGetLastError();
    return fail(MPQ_ERR_OOM, "spectrum allocation failed");
  }
  {
    ProfScope ps_("k_sqrt_first", st);
    k_sqrt_first<<<(unsigned)cdiv(r, 256), 256, 0, st>>>(lam, r, p->s64);
  }
  count_launch();
  return check_launch("k_sqrt_first");
}

}  // namespace

mpq_status setup_spectrum_from_gram(mpq_plan_s* p, const double* G, int64_t m, cudaStream_t st) {
  const int64_t n = p->n;
  DevBuf<double> lam, E;
  MPQ_TRY(lam.alloc(n));
  MPQ_TRY(E.alloc(n * n));
  MPQ_TRY(jacobi_eig(G, n, lam.p, E.p, st));
  MPQ_TRY(cut_and_alloc(p, lam.p, n, m, n, st));
  {
    ProfScope ps_("k_take_cols", st);
    k_take_cols<<<(unsigned)cdiv(n * p->r, 256), 256, 0, st>>>(E.p, n, p->r, p->V64);
  }
  count_launch();
  MPQ_TRY(check_launch("setup gather"));
  MPQ_CUDA(cudaStreamSynchronize(st));
  return MPQ_OK;
}

mpq_status gram_accumulate(double* G, int64_t n, const float* X, int64_t rows, cudaStream_t st) {
  if (rows == 0) return MPQ_OK;
  DevBuf<double> Xt;
  MPQ_TRY(Xt.alloc(rows * n));
  {
    ProfScope ps_("k_x_to_f64", st);
    k_x_to_f64<<<g1(rows * n), 256, 0, st>>>(X, rows, n, 1, Xt.p);
  }
  count_launch();
  MPQ_TRY(check_launch("k_x_to_f64"));
  MPQ_TRY(gemm_nt_f64(Xt.p, rows, Xt.p, rows, G, n, n, n, rows, st, /*accumulate=*/true));
  MPQ_CUDA(cudaStreamSynchronize(st));  // Xt is released on return
  return MPQ_OK;
}

mpq_status setup_spectrum_from_x(mpq_plan_s* p, const float* X, int64_t m, int64_t n,
                                 cudaStream_t st) {
  const bool right = n <= m;  // Gram X^T X (n x n); else X X^T (m x m)
  const int64_t N0 = right ? n : m;
  DevBuf<double> Xd, G, lam, E;
  MPQ_TRY(G.alloc(N0 * N0));
  if (right) {
    MPQ_CUDA(cudaMemsetAsync(G.p, 0, sizeof(double) * N0 * N0, st));
    MPQ_TRY(gram_accumulate(G.p, n, X, m, st));
    return setup_spectrum_from_gram(p, G.p, m, st);
  }
  MPQ_TRY(Xd.alloc(m * n));
  MPQ_TRY(lam.alloc(N0));
  MPQ_TRY(E.alloc(N0 * N0));
  {
    ProfScope ps_("k_x_to_f64", st);
    k_x_to_f64<<<g1(m * n), 256, 0, st>>>(X, m, n, 0, Xd.p);
  }
  count_launch();
  MPQ_TRY(check_launch("k_x_to_f64"));
  MPQ_TRY(gemm_nt_f64(Xd.p, n, Xd.p, n, G.p, m, m, m, n, st));  // X X^T
  MPQ_TRY(jacobi_eig(G.p, N0, lam.p, E.p, st));
  MPQ_TRY(cut_and_alloc(p, lam.p, N0, m, n, st));
  const int64_t r = p->r;
  // V = X^T U diag(1/s): (n x r) = Xt (n x m) * Ut (r x m)^T
  DevBuf<double> Xt, Ut;
  MPQ_TRY(Xt.alloc(n * m));
  MPQ_TRY(Ut.alloc(r * m));
  {
    ProfScope ps_("k_x_to_f64", st);
    k_x_to_f64<<<g1(m * n), 256, 0, st>>>(X, m, n, 1, Xt.p);
  }
  {
    ProfScope ps_("k_take_cols_t", st);
    k_take_cols_t<<<(unsigned)cdiv(N0 * r, 256), 256, 0, st>>>(E.p, N0, r, Ut.p);
  }
  count_launch(2);
  MPQ_TRY(check_launch("setup transposes"));
  MPQ_TRY(gemm_nt_f64(Xt.p, m, Ut.p, m, p->V64, r, n, r, m, st));
  {
    ProfScope ps_("k_div_cols", st);
    k_div_cols<<<g1(n * r), 256, 0, st>>>(p->V64, n, r, p->s64);
  }
  count_launch();
  MPQ_TRY(check_launch("k_div_cols"));
  MPQ_CUDA(cudaStreamSynchronize(st));
  return MPQ_OK;
}

// ------------------------------------------- random Hadamard rotation ---
// Incoherence preprocessing (the ai.info page on MPQ, findings: a random
// Hadamard rotation leaves E_lin unchanged because E_lin sees the Hessian
// only through its eigenvalues).  Every row x of X becomes x Q^T with
// Q = H_n diag(signs) / sqrt(n), H_n the Sylvester-Hadamard matrix
// (H_1 = [1], H_2k = [[H_k, H_k], [H_k, -H_k]]; symmetric), so that
// x Q^T = (x .* signs) H_n / sqrt(n): log2(n) butterfly stages, the stage of
// half-width h taking every pair (lo, lo + h) with bit log2(h) of lo clear to
// (a + b, a - b).  Both kernels run the stages in the order h = 1, 2, 4, ...,
// so they give the same bits.
namespace {

// Any n (a power of two up to 32768; used outside 512..8192): one CTA per row, the row in shared
// memory, one pass over it per stage.
__global__ void __launch_bounds__(512)
    k_rht(float* __restrict__ X, int64_t rows, int n, const float* __restrict__ signs,
          float inv_sqrt_n) {
  extern __shared__ float sx[];
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    float* x = X + row * n;
    for (int j = threadIdx.x; j < n; j += blockDim.x) sx[j] = x[j] * signs[j];
    __syncthreads();
    for (int h = 1; h < n; h <<= 1) {
      for (int i = threadIdx.x; i < n / 2; i += blockDim.x) {
        const int lo = ((i & ~(h - 1)) << 1) | (i & (h - 1));
        const float a = sx[lo], b = sx[lo + h];
        sx[lo] = a + b;
        sx[lo + h] = a - b;
      }
      __syncthreads();
    }
    for (int j = threadIdx.x; j < n; j += blockDim.x) x[j] = sx[j] * inv_sqrt_n;
    __syncthreads();
  }
}

// 512 <= n <= 8192: n / 16 threads per row, 16 values each in registers.
// The log2(n) index bits are taken in passes of up to four: in the pass over
// bits [b0, b0 + nb) value v = (vh << nb) | vl of thread t is element
//   j = (r mod 2^b0) | (vl << b0) | ((r >> b0) << (b0 + nb)),  r = vh T + t,
// so its nb stages are butterflies between registers.  The first pass
// (b0 = 0, nb = 4) is the thread's 16 consecutive elements (four float4
// loads); between passes the row goes through shared memory once.  The
// shared-memory word of element j is j with its quad bits (2..4) XORed by a
// function of the 32-word line (j >> 5): line mod 8, and 4 more when bit 3 of
// the line is set.  That keeps the float4 stores of the first pass and the
// 32-lane scalar accesses of the later ones free of bank conflicts.
constexpr int RHT_V = 16;
constexpr int RHT_MIN_N = 512, RHT_MAX_N = 8192;

__device__ __forceinline__ int rht_swz(int j) {
  const int line = j >> 5;
  const int g = (line & 7) ^ (((line >> 3) & 1) << 2);
  return j ^ (g << 2);
}

__device__ __forceinline__ int rht_elem(int t, int v, int T, int b0, int nb) {
  const int r = (v >> nb) * T + t;
  return (r & ((1 << b0) - 1)) | ((v & ((1 << nb) - 1)) << b0) | ((r >> b0) << (b0 + nb));
}

template <int NB>
__device__ __forceinline__ void rht_reg_stages(float (&a)[RHT_V]) {
#pragma unroll
  for (int s = 0; s < NB; ++s) {
#pragma unroll
    for (int v = 0; v < RHT_V; ++v) {
      if (((v >> s) & 1) == 0) {
        const float p = a[v], q = a[v + (1 << s)];
        a[v] = p + q;
        a[v + (1 << s)] = p - q;
      }
    }
  }
}

// One pass over bits [B0, B0 + NB) after the previous pass over [PB0, B0):
// hand the row over through shared memory, then NB register stages.
template <int L, int PB0, int B0>
__device__ __forceinline__ void rht_pass(float (&a)[RHT_V], float* sx, int t) {
  constexpr int T = (1 << L) / RHT_V;
  constexpr int NB = (L - B0) < 4 ? (L - B0) : 4;
  if constexpr (B0 > 4) {
#pragma unroll
    for (int v = 0; v < RHT_V; ++v) sx[rht_swz(rht_elem(t, v, T, PB0, B0 - PB0))] = a[v];
  }
  __syncthreads();
#pragma unroll
  for (int v = 0; v < RHT_V; ++v) a[v] = sx[rht_swz(rht_elem(t, v, T, B0, NB))];
  __syncthreads();  // every read done before the next hand-over or row
  rht_reg_stages<NB>(a);
  if constexpr (B0 + NB < L) rht_pass<L, B0, B0 + NB>(a, sx, t);
}

// At n = 4096 the register bound of 80 (three CTAs per SM) holds the 16
// values and their addresses without spilling.
template <int L>
__global__ void __launch_bounds__((1 << L) / RHT_V, L == 12 ? 3 : 1)
    k_rht_reg(float* __restrict__ X, int64_t rows, const float* __restrict__ signs,
              float inv_sqrt_n) {
  extern __shared__ float sx[];
  constexpr int n = 1 << L;
  constexpr int T = n / RHT_V;
  constexpr int LB0 = 4 * ((L - 1) / 4), LNB = L - LB0;  // the last pass
  const int t = threadIdx.x;
  float a[RHT_V];
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    float* x = X + row * (int64_t)n;
#pragma unroll
    for (int q = 0; q < RHT_V / 4; ++q) {
      const float4 x4 = __ldcs(reinterpret_cast<const float4*>(x + RHT_V * t) + q);
      const float4 s4 = __ldg(reinterpret_cast<const float4*>(signs + RHT_V * t) + q);
      a[4 * q] = x4.x * s4.x;
      a[4 * q + 1] = x4.y * s4.y;
      a[4 * q + 2] = x4.z * s4.z;
      a[4 * q + 3] = x4.w * s4.w;
    }
    rht_reg_stages<4>(a);
    // first hand-over: the 16 consecutive elements as four float4 stores
#pragma unroll
    for (int q = 0; q < RHT_V / 4; ++q)
      *reinterpret_cast<float4*>(sx + rht_swz(RHT_V * t + 4 * q)) =
          make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
    rht_pass<L, 0, 4>(a, sx, t);
    // last pass: its bits start at 8 or above, so a warp's 32 lanes store 32
    // consecutive floats
#pragma unroll
    for (int v = 0; v < RHT_V; ++v) __stcs(x + rht_elem(t, v, T, LB0, LNB), a[v] * inv_sqrt_n);
  }
}

template <int L>
mpq_status launch_rht_reg(float* X, int64_t rows, const float* signs, float inv_sqrt_n, int sms,
                          cudaStream_t st) {
  constexpr int threads = (1 << L) / RHT_V;
  constexpr size_t smem = sizeof(float) << L;
  MPQ_CUDA(cudaFuncSetAttribute(k_rht_reg<L>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  int per_sm = 0;
  MPQ_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_rht_reg<L>, threads, smem));
  const unsigned grid = (unsigned)std::min<int64_t>(rows, (int64_t)sms * std::max(1, per_sm));
  {
    ProfScope ps_("k_rht", st);
    k_rht_reg<L><<<grid, threads, smem, st>>>(X, rows, signs, inv_sqrt_n);
  }
  count_launch();
  return check_launch("k_rht_reg");
}

}  // namespace

mpq_status launch_rht(float* X, int64_t rows, int64_t n, const float* signs, cudaStream_t st) {
  if (rows == 0) return MPQ_OK;
  const float inv_sqrt_n = (float)(1.0 / sqrt((double)n));
  int dev = 0, sms = 0;
  MPQ_CUDA(cudaGetDevice(&dev));
  MPQ_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const size_t smem = sizeof(float) * (size_t)n;
  if (n >= RHT_MIN_N && n <= RHT_MAX_N && (reinterpret_cast<uintptr_t>(X) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(signs) & 15) == 0) {
    switch (n) {
      case 512: return launch_rht_reg<9>(X, rows, signs, inv_sqrt_n, sms, st);
      case 1024: return launch_rht_reg<10>(X, rows, signs, inv_sqrt_n, sms, st);
      case 2048: return launch_rht_reg<11>(X, rows, signs, inv_sqrt_n, sms, st);
      case 4096: return launch_rht_reg<12>(X, rows, signs, inv_sqrt_n, sms, st);
      case 8192: return launch_rht_reg<13>(X, rows, signs, inv_sqrt_n, sms, st);
      default: break;
    }
  }
  const int threads = (int)std::min<int64_t>(512, std::max<int64_t>(32, n / 2));
  MPQ_CUDA(cudaFuncSetAttribute(k_rht, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const unsigned grid = (unsigned)std::min<int64_t>(rows, (int64_t)sms * 8);
  {
    ProfScope ps_("k_rht", st);
    k_rht<<<grid, threads, smem, st>>>(X, rows, (int)n, signs, inv_sqrt_n);
  }
  count_launch();
  return check_launch("k_rht");
}

}  // namespace mpq
