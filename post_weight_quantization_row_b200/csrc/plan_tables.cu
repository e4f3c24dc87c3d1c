// Plan-time tables: H = V diag(s^2) V^T (fp64 product, stored fp32), its
// diagonal, fp32 copies of the spectrum in both layouts, and for vector
// codebooks |c|^2 and the per-block quadratic forms 1/2 c^T H_bb c used by
// the CD step of the MPQ note's key design 3.
#include "mpq_internal.cuh"

namespace mpq {
namespace {

__global__ void k_scale_cols(const double* __restrict__ V, const double* __restrict__ s,
                             int64_t n, int64_t r, double* __restrict__ out) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * r;
       e += (int64_t)gridDim.x * blockDim.x)
    out[e] = V[e] * s[e % r];
}

__global__ void k_to_f32(const double* __restrict__ x, int64_t count, float* __restrict__ y) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < count;
       e += (int64_t)gridDim.x * blockDim.x)
    y[e] = (float)x[e];
}

// y (cols x rows) = x^T, x rows x cols, fp64 -> fp32
__global__ void k_transpose_f32(const double* __restrict__ x, int64_t rows, int64_t cols,
                                float* __restrict__ y) {
  __shared__ double t[32][33];
  const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) t[i][threadIdx.x] = x[r * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) y[c * rows + r] = (float)t[threadIdx.x][i];
  }
}

__global__ void k_diag_f64_to_f32(const double* __restrict__ H, int64_t n, float* __restrict__ Hs,
                                  float* __restrict__ d) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * n;
       e += (int64_t)gridDim.x * blockDim.x) {
    Hs[e] = (float)H[e];
    if (e / n == e % n) d[e / n] = (float)H[e];
  }
}

__global__ void k_codebook_norms(const float* __restrict__ cb, int K, float* __restrict__ nrm) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= K) return;
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s = fmaf(cb[c * 8 + i], cb[c * 8 + i], s);
  nrm[c] = s;
}

// qtab[b][c] = 1/2 c^T H_bb c (fp64 arithmetic, stored fp32)
__global__ void k_block_quad(const float* __restrict__ cb, int K, const float* __restrict__ H,
                             int64_t n, float* __restrict__ qtab) {
  __shared__ double G[8][8];
  const int64_t b = blockIdx.y;
  if (threadIdx.x < 64) G[threadIdx.x / 8][threadIdx.x % 8] = H[(8 * b + threadIdx.x / 8) * n + 8 * b + threadIdx.x % 8];
  __syncthreads();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= K) return;
  double x[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = cb[c * 8 + i];
  double q = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    double gi = 0.0;
#pragma unroll
    for (int j = 0; j < 8; ++j) gi += G[i][j] * x[j];
    q += x[i] * gi;
  }
  qtab[b * K + c] = (float)(0.5 * q);
}

unsigned grid_for(int64_t count) {
  return (unsigned)std::min<int64_t>(cdiv(count, 256), 148 * 16);
}

}  // namespace

mpq_status build_hessian(mpq_plan_s* p, cudaStream_t st) {
  const int64_t n = p->n, r = p->r;
  double* Vs = nullptr;
  double* H64 = nullptr;
  MPQ_CUDA(cudaMallocAsync(&Vs, sizeof(double) * n * r, st));
  MPQ_CUDA(cudaMallocAsync(&H64, sizeof(double) * n * n, st));
  {
    ProfScope ps_("k_scale_cols", st);
    k_scale_cols<<<grid_for(n * r), 256, 0, st>>>(p->V64, p->s64, n, r, Vs);
  }
  count_launch();
  MPQ_TRY(check_launch("k_scale_cols"));
  MPQ_TRY(gemm_nt_f64(Vs, r, Vs, r, H64, n, n, n, r, st));
  {
    ProfScope ps_("k_diag_f64_to_f32", st);
    k_diag_f64_to_f32<<<grid_for(n * n), 256, 0, st>>>(H64, n, p->H32, p->Hdiag);
  }
  count_launch();
  MPQ_TRY(check_launch("k_diag_f64_to_f32"));
  {
    ProfScope ps_("k_to_f32", st);
    k_to_f32<<<grid_for(n * r), 256, 0, st>>>(p->V64, n * r, p->V32);
  }
  {
    ProfScope ps_("k_to_f32", st);
    k_to_f32<<<grid_for(r), 256, 0, st>>>(p->s64, r, p->s32);
  }
  dim3 tg((unsigned)cdiv(r, 32), (unsigned)cdiv(n, 32));
  {
    ProfScope ps_("k_transpose_f32", st);
    k_transpose_f32<<<tg, dim3(32, 8), 0, st>>>(p->V64, n, r, p->Vt32);
  }
  count_launch(3);
  MPQ_TRY(check_launch("plan tables"));
  cudaFreeAsync(Vs, st);
  cudaFreeAsync(H64, st);
  return MPQ_OK;
}

// 1/2 |c|^2, exact in fp32 (the greedy scan's score table)
__global__ void k_half_norms(const float* __restrict__ nrm, int K, float* __restrict__ out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c < K) out[c] = 0.5f * nrm[c];
}

mpq_status build_codebook_tables(mpq_plan_s* p, cudaStream_t st) {
  if (p->d != 8) return MPQ_OK;
  {
    ProfScope ps_("k_codebook_norms", st);
    k_codebook_norms<<<(unsigned)cdiv(p->K, 256), 256, 0, st>>>(p->cb, p->K, p->cb_norm);
  }
  count_launch();
  MPQ_TRY(check_launch("k_codebook_norms"));
  {
    ProfScope ps_("k_half_norms", st);
    k_half_norms<<<(unsigned)cdiv(p->K, 256), 256, 0, st>>>(p->cb_norm, p->K, p->cb_hnorm);
  }
  count_launch();
  MPQ_TRY(check_launch("k_half_norms"));
  dim3 g((unsigned)cdiv(p->K, 256), (unsigned)p->B);
  {
    ProfScope ps_("k_block_quad", st);
    k_block_quad<<<g, 256, 0, st>>>(p->cb, p->K, p->H32, p->n, p->qtab);
  }
  count_launch();
  return check_launch("k_block_quad");
}

}  // namespace mpq
