// Plain SIMT GEMMs:  C[M x N] = A[M x K] * B[N x K]^T  (row-major, both
// operands K-contiguous).  fp32 is used for the small and ragged shapes of
// the solve; fp64 for the Gram matrices of the setup.
#include "mpq_internal.cuh"

namespace mpq {
namespace {

template <typename T, int BM, int BN, int BK>
struct GemmCfg {
  static constexpr int THREADS = 256;
  static constexpr int SPLIT_M = BM / 64;  // 4-row groups per thread, spaced BM/SPLIT apart
  static constexpr int SPLIT_N = BN / 64;
  static constexpr int TM = 4 * SPLIT_M;
  static constexpr int TN = 4 * SPLIT_N;
  static constexpr int EA = BM * BK / THREADS;  // A elements loaded per thread per tile
  static constexpr int EB = BN * BK / THREADS;
  static constexpr int PAD = 4;
};

template <typename T, int BM, int BN, int BK>
__global__ void __launch_bounds__(256)
    k_gemm_nt(const T* __restrict__ A, int64_t lda, const T* __restrict__ B, int64_t ldb,
              T* __restrict__ C, int64_t ldc, int64_t M, int64_t N, int64_t K, bool accumulate) {
  using Cfg = GemmCfg<T, BM, BN, BK>;
  constexpr int TM = Cfg::TM, TN = Cfg::TN, EA = Cfg::EA, EB = Cfg::EB;
  __shared__ __align__(16) T As[2][BK][BM + Cfg::PAD];
  __shared__ __align__(16) T Bs[2][BK][BN + Cfg::PAD];

  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int64_t bm = (int64_t)blockIdx.y * BM;
  const int64_t bn = (int64_t)blockIdx.x * BN;

  // load mapping: each thread reads EA consecutive k of one A row (same for B)
  const int a_row = tid / (BK / EA), a_k = (tid % (BK / EA)) * EA;
  const int b_row = tid / (BK / EB), b_k = (tid % (BK / EB)) * EB;

  T ra[EA], rb[EB];
  T acc[TM][TN];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = T(0);

  auto load_tile = [&](int64_t k0) {
    const int64_t gr = bm + a_row;
#pragma unroll
    for (int e = 0; e < EA; ++e) {
      const int64_t gk = k0 + a_k + e;
      ra[e] = (gr < M && gk < K) ? A[gr * lda + gk] : T(0);
    }
    const int64_t gc = bn + b_row;
#pragma unroll
    for (int e = 0; e < EB; ++e) {
      const int64_t gk = k0 + b_k + e;
      rb[e] = (gc < N && gk < K) ? B[gc * ldb + gk] : T(0);
    }
  };
  auto store_tile = [&](int buf) {
#pragma unroll
    for (int e = 0; e < EA; ++e) As[buf][a_k + e][a_row] = ra[e];
#pragma unroll
    for (int e = 0; e < EB; ++e) Bs[buf][b_k + e][b_row] = rb[e];
  };

  const int64_t ntiles = (K + BK - 1) / BK;
  load_tile(0);
  store_tile(0);
  __syncthreads();
  for (int64_t t = 0; t < ntiles; ++t) {
    const int buf = (int)(t & 1);
    if (t + 1 < ntiles) load_tile((t + 1) * BK);
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      T a[TM], b[TN];
#pragma unroll
      for (int h = 0; h < Cfg::SPLIT_M; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) a[h * 4 + i] = As[buf][kk][h * (BM / Cfg::SPLIT_M) + ty * 4 + i];
#pragma unroll
      for (int h = 0; h < Cfg::SPLIT_N; ++h)
#pragma unroll
        for (int j = 0; j < 4; ++j) b[h * 4 + j] = Bs[buf][kk][h * (BN / Cfg::SPLIT_N) + tx * 4 + j];
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    if (t + 1 < ntiles) store_tile(buf ^ 1);
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int64_t gr = bm + (i / 4) * (BM / Cfg::SPLIT_M) + ty * 4 + (i % 4);
    if (gr >= M) continue;
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      const int64_t gc = bn + (j / 4) * (BN / Cfg::SPLIT_N) + tx * 4 + (j % 4);
      if (gc < N) C[gr * ldc + gc] = accumulate ? C[gr * ldc + gc] + acc[i][j] : acc[i][j];
    }
  }
}

}  // namespace

mpq_status gemm_nt_f32(const float* A, int64_t lda, const float* B, int64_t ldb, float* C,
                       int64_t ldc, int64_t M, int64_t N, int64_t K, cudaStream_t st,
                       const char* tag) {
  if (M <= 0 || N <= 0) return MPQ_OK;
  constexpr int BM = 128, BN = 128, BK = 16;
  dim3 grid((unsigned)cdiv(N, BN), (unsigned)cdiv(M, BM));
  if (grid.y > 65535) return fail(MPQ_ERR_INVALID_ARG, "gemm: too many row tiles");
  {
    ProfScope ps_(tag, st);
    k_gemm_nt<float, BM, BN, BK><<<grid, 256, 0, st>>>(A, lda, B, ldb, C, ldc, M, N, K, false);
  }
  count_launch();
  return check_launch("k_gemm_nt<f32>");
}

mpq_status gemm_nt_f64(const double* A, int64_t lda, const double* B, int64_t ldb, double* C,
                       int64_t ldc, int64_t M, int64_t N, int64_t K, cudaStream_t st,
                       bool accumulate) {
  if (M <= 0 || N <= 0) return MPQ_OK;
  constexpr int BM = 64, BN = 64, BK = 16;
  dim3 grid((unsigned)cdiv(N, BN), (unsigned)cdiv(M, BM));
  if (grid.y > 65535) return fail(MPQ_ERR_INVALID_ARG, "gemm: too many row tiles");
  {
    ProfScope ps_("k_gemm_nt_f64", st);
    k_gemm_nt<double, BM, BN, BK><<<grid, 256, 0, st>>>(A, lda, B, ldb, C, ldc, M, N, K,
                                                         accumulate);
  }
  count_launch();
  return check_launch("k_gemm_nt<f64>");
}

}  // namespace mpq
