// Internal declarations shared by the libmpq translation units.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "../../include/mpq.h"

namespace mpq {

// ---------------------------------------------------------------- errors ---
void set_error(const std::string& msg);
mpq_status fail(mpq_status st, const std::string& msg);
mpq_status cuda_fail(cudaError_t e, const char* what);

#define MPQ_CUDA(call)                                              \
  do {                                                              \
    cudaError_t e_ = (call);                                        \
    if (e_ != cudaSuccess) return ::mpq::cuda_fail(e_, #call);      \
  } while (0)

#define MPQ_TRY(call)                                               \
  do {                                                              \
    mpq_status s_ = (call);                                         \
    if (s_ != MPQ_OK) return s_;                                    \
  } while (0)

// Event pair around one kernel launch when profiling is on (mpq_profile_*).
struct ProfScope {
  int slot = -1;
  cudaStream_t st = nullptr;
  ProfScope(const char* name, cudaStream_t stream);
  ~ProfScope();
};

// Every kernel launch goes through this counter (see mpq_kernel_launch_count).
void count_launch(int n = 1);
mpq_status check_launch(const char* name);

// Device status word bits (set by kernels, read by mpq_plan_status).
enum : int { STATUS_NONFINITE = 1, STATUS_TIMEOUT = 2, STATUS_BADINDEX = 4 };

// A fp32 matrix stored for the tensor-core GEMM as fp16 hi/lo pairs of its
// power-of-two-scaled values: x = (hi + lo) * unscale, rows padded to a
// multiple of 256 and K to a multiple of 64 (zero padding), K contiguous.
struct SplitOperand {
  __half* hi = nullptr;
  __half* lo = nullptr;
  int64_t rows = 0, rows_pad = 0, K = 0, ld = 0;
  float* row_unscale = nullptr;  // per-row 2^e (A operands), rows_pad floats
  float* unscale = nullptr;      // device scalar 2^e (B operands)
  float unscale_host = 1.0f;     // host copy of *unscale
};

inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// Largest row count an entry point accepts: rows map to the grid's x
// dimension, whose limit is 2^31 - 1.
constexpr int64_t MAX_ROWS = 2147483647LL;

// --------------------------------------------------------------- workspace --
struct Workspace {
  int64_t rows = 0;       // rows the buffers are sized for
  int64_t bytes = 0;
  // m x n fp32
  float* R1 = nullptr;
  float* X1 = nullptr;
  float* R2 = nullptr;
  // A operand of the tensor-core GEMMs (w - r2, the GEMM2 operand, residuals)
  SplitOperand As;
  CUtensorMap tm_an_hi, tm_an_lo;  // K = n view
  CUtensorMap tm_ar_hi, tm_ar_lo;  // K = r view
  // A operand of the linear module's second GEMM (D u, K = r), written by
  // the first GEMM's epilogue (a buffer of its own: other tiles of that GEMM
  // still read As), and the epilogue's per-(row, column tile) M-step sums
  SplitOperand Aq;
  CUtensorMap tm_aq_hi, tm_aq_lo;
  float2* lin_part = nullptr;      // cdiv(r, 128) x rows
  int* tile_count = nullptr;       // CD: changes per (sweep, tile)
  // CD gradient h = H (w - x), rows x ldh (ldh = n rounded up to 32)
  float* Hg = nullptr;
  int64_t ldh = 0;
  CUtensorMap tm_hg;               // reduce-add target of the CD updates
  float* Hl = nullptr;             // d = 8 CD: rows x CD_TILE tile-local gradient
  float* sref = nullptr;           // grouped CD: per-row reference scale of Delta
  int32_t* cd_skip = nullptr;      // adaptive CD: rows that keep the marginal MAP
  // m x r fp32
  float* P = nullptr;
  // m x B
  uint16_t* idx = nullptr;
  // per-row
  float* scale = nullptr;
  float* offset = nullptr;
  double* gamma1 = nullptr;
  double* gamma1_0 = nullptr;
  double* gamma2 = nullptr;
  double* beta = nullptr;
  double* vsum = nullptr;
  double* coef = nullptr;   // 1/(1 - alpha2) of the last linear step
  double* kappa = nullptr;  // alpha2/(1 - alpha2)
  int32_t* clamps = nullptr;
  // host-buffer solve staging (m x n W, outputs)
  float* W = nullptr;
  float* w_hat = nullptr;
  float* energy = nullptr;
  uint16_t* idx_stage = nullptr;
};

}  // namespace mpq

struct mpq_plan_s {
  int device = 0;
  int64_t n = 0, r = 0;
  int32_t d = 1, K = 2;
  int64_t B = 0;
  int G = 0;        // scalar grid group size (columns); 0: one grid per row
  int64_t ng = 1;   // grids per row
  mpq_params params{};
  // spectrum
  double* s64 = nullptr;   // r
  double* V64 = nullptr;   // n x r
  float* s32 = nullptr;    // r
  float* V32 = nullptr;    // n x r  (operand of x2 = r2 + V u')
  float* Vt32 = nullptr;   // r x n  (operand of p = V^T (w - r2))
  float* H32 = nullptr;    // n x n  H = V diag(s^2) V^T
  float* Hdiag = nullptr;  // n
  // B operands of the tensor-core GEMMs
  mpq::SplitOperand Vt_s, V_s, H_s;
  CUtensorMap tm_vt_hi, tm_vt_lo, tm_v_hi, tm_v_lo, tm_h_hi, tm_h_lo;
  // greedy baseline (LDLQ), built when params.greedy_init is set (d = 1)
  float* ldlq_diag = nullptr;  // per tile of CD_TILE columns: its diagonal block of B^T
  mpq::SplitOperand Lq_s;      // B = L diag(L)^-1 (n x n), (H + lambda I)^-1 = L L^T
  CUtensorMap tm_lq_hi, tm_lq_lo;
  // vector codebook (d = 8)
  float* cb = nullptr;       // K x 8
  float* cb_norm = nullptr;  // K  |c|^2
  float* cb_hnorm = nullptr; // K  1/2 |c|^2 (the greedy scan's score table)
  float* qtab = nullptr;     // B x K  1/2 c^T H_bb c
  bool vec_tc = false;       // the denoiser runs on the tensor cores
  int vec_tc_F = 0;          // grid bits of its exact split of t - c*
  int vec_tc_Fmin = 0;       //   (finest, coarsest)
  int vec_tc_rk = 0;         // extra scale bits of its remainder operand
  void* cb_tc = nullptr;     // (K / 128) x 4 KiB codebook operand images
  // status
  int* status = nullptr;     // device word
  int64_t ws_cap = 0;
  mpq::Workspace ws;
  uint64_t ws_gen = 0;       // bumped whenever the workspace is reallocated
  // captured solves: mpq_solve replays the graph of its launches when it is
  // called again with the same buffers, sizes and options
  static constexpr int N_GRAPHS = 4;
  static constexpr int GRAPH_KEY = 16;
  struct SolveGraph {
    uint64_t key[GRAPH_KEY] = {};
    cudaGraphExec_t exec = nullptr;
    int64_t launches = 0;
    uint64_t last_use = 0;  // 0: empty slot
  };
  SolveGraph graphs[N_GRAPHS];
  uint64_t graph_clock = 0;
  cudaStream_t capture_stream = nullptr;
};

namespace mpq {

// ------------------------------------------------------------- launchers ---
// GEMM  C[M x N] = A[M x K] * B[N x K]^T  (row-major, K contiguous), fp32.
// `tag` names the launch in the profiler (one name per GEMM role).
mpq_status gemm_nt_f32(const float* A, int64_t lda, const float* B, int64_t ldb, float* C,
                       int64_t ldc, int64_t M, int64_t N, int64_t K, cudaStream_t st,
                       const char* tag = "gemm_f32");
// Same with fp64 operands and accumulation (setup); `accumulate` adds the
// product to C instead of overwriting it.
mpq_status gemm_nt_f64(const double* A, int64_t lda, const double* B, int64_t ldb, double* C,
                       int64_t ldc, int64_t M, int64_t N, int64_t K, cudaStream_t st,
                       bool accumulate = false);

mpq_status launch_init(const mpq_plan_s* p, const float* W, int64_t m, int given, float* scale,
                       float* offset, uint16_t* idx, double* gamma1_0, cudaStream_t st,
                       bool rtn = true);
mpq_status launch_denoise(const mpq_plan_s* p, const float* R1, const double* gamma1,
                          const float* scale, const float* offset, int64_t m, const float* W,
                          const double* gamma1_0, float* xhat1, float* vblock, double* vsum,
                          uint16_t* idx, cudaStream_t st, bool map_only = false);
// (map_only: only idx, the posterior's argmax, is wanted; the tensor-core
// vector denoiser then skips its second pass and writes nothing else)
// writes r2 and the A operand w - r2 (split, K = n)
mpq_status launch_extrinsic_d2l(const mpq_plan_s* p, const float* W, int64_t m, const float* R1,
                                const double* gamma1, const float* xhat1, const double* vsum,
                                const double* gamma1_0, float* R2, SplitOperand* As,
                                double* gamma2, int32_t* clamps, cudaStream_t st);
// reads p' from P, writes the GEMM2 A operand (split, K = r)
// M-step finisher after the projection GEMM's linear epilogue: per row, the
// column tiles' sums in a fixed order, then alpha2, beta_hat, the damped
// beta, gamma1', the l2d coefficients and the second GEMM's row scale.  Its
// inputs and outputs (the fused row kernel can run it in its prologue):
struct LinFinish {
  const float2* part;
  int ntiles, e_bound;
  int64_t m, n, r;
  const float* a_unscale;
  float* q_unscale;  // NULL: the expand GEMM takes its row scale from a_unscale
  const double* gamma2;
  const double* gamma1_0;
  double* beta;
  double damping, glo, ghi, amin, amax;
  double* gamma1_out;
  double* coef;
  double* kappa;
  double* alpha2_out;
  double* beta_hat_out;
  int32_t* clamps;
};
LinFinish make_lin_finish(const mpq_plan_s* p, int64_t m, const float2* part, int ntiles,
                          int e_bound, const float* a_unscale, float* q_unscale,
                          const double* gamma2, const double* gamma1_0, double* beta,
                          double* gamma1_out, double* coef, double* kappa, double* alpha2,
                          double* beta_hat, int32_t* clamps);
mpq_status launch_linear_finish(const mpq_plan_s* p, int64_t m, const float2* part, int ntiles,
                                int e_bound, const float* a_unscale, float* q_unscale,
                                const double* gamma2, const double* gamma1_0, double* beta,
                                double* gamma1_out, double* coef, double* kappa, double* alpha2,
                                double* beta_hat, int32_t* clamps, cudaStream_t st);
int vamp_row_threads(int64_t n, int G);  // 0: the fused scalar row kernel does not apply
mpq_status launch_vamp_row_scalar(const mpq_plan_s* p, const float* W, int64_t m, int first,
                                  int map, const float* G, float* R2, const double* coef,
                                  const double* kappa, const double* gamma1, const float* scale,
                                  const float* offset, const double* gamma1_0, SplitOperand* As,
                                  double* gamma2, int32_t* clamps, uint16_t* idx, cudaStream_t st,
                                  float* R1o = nullptr, const LinFinish* fin = nullptr);
// (fin: the previous linear step's M-step finish, run per row by the kernel
// before it reads gamma1, coef and kappa)
mpq_status launch_extrinsic_l2d(const mpq_plan_s* p, const float* W, int64_t m, const float* R2,
                                const float* G, const double* coef, const double* kappa,
                                float* R1_out, float* xhat2, cudaStream_t st);
// residual w - w_hat as the split A operand (K = n); w_hat optional
mpq_status launch_residual_split(const mpq_plan_s* p, const float* W, int64_t m,
                                 const float* scale, const float* offset, const uint16_t* idx,
                                 SplitOperand* As, float* w_hat, cudaStream_t st);
mpq_status launch_residual(const mpq_plan_s* p, const float* W, int64_t m, const float* scale,
                           const float* offset, const uint16_t* idx, float* E, float* w_hat,
                           cudaStream_t st);
// Clamp caller-supplied codeword indices into [0, K) in place, flagging any
// that were out of range in the status word (STATUS_BADINDEX).
mpq_status launch_sanitize_idx(const mpq_plan_s* p, uint16_t* idx, int64_t count, cudaStream_t st);
mpq_status launch_energy_rows(const mpq_plan_s* p, int64_t m, const float* P, float* energy,
                              cudaStream_t st);
// CD sweeps; h (m x ldh) holds H (w - x) on entry and is updated in place
// (rows with skip[row] != 0 run no CD; skip may be null)
mpq_status launch_cd(mpq_plan_s* p, const float* W, int64_t m, const float* scale,
                     const float* offset, uint16_t* idx, float* h, int64_t ldh, int32_t sweeps,
                     int32_t* changes, cudaStream_t st, const int32_t* skip = nullptr);
mpq_status launch_cd_skip(const double* gamma1, const float* scale, int64_t m, int64_t ng,
                          double threshold, int32_t* skip, cudaStream_t st);
// ceil(y) for |y| < 2^22 with one directed-rounding add: y + 1.5 2^23 rounded
// up lands on the integer grid of [2^23, 2^24) (full-rate adds instead of a
// rounding instruction).  Larger |y| keeps its sign, which is all the callers
// need: they clamp the result to a grid of at most 65536 levels.
__device__ __forceinline__ float ceil_small(float y) {
  return __fsub_rn(__fadd_ru(y, 12582912.0f), 12582912.0f);
}

constexpr int CD_TILE = 128;  // columns per scalar CD tile (multiple of 64)
constexpr int CD_GROUP = 4;   // CD tiles per group of eager gradient updates
constexpr int64_t CD_PANEL_BYTES = 32ll << 20;  // L2-resident slab of the CD gradient
constexpr int64_t CD_PANEL_MIN = 512;           // narrowest CD panel (columns)
int64_t cd_panel_cols(int64_t m, int64_t n);
mpq_status launch_row_max(const float* scale, int64_t m, int64_t ng, float* out, cudaStream_t st);

// greedy baseline (greedy.cu): the factors of (H + lambda I)^-1, lambda =
// damp * mean(diag H), into Bl (n x n fp32) and Ud (tiles x CD_TILE^2 fp32,
// zeroed by the caller); and the LDLQ pass of m rows into idx
mpq_status ldlq_factor(const mpq_plan_s* p, double damp, float* Bl, float* Ud, cudaStream_t st);
mpq_status launch_ldlq(mpq_plan_s* p, const float* W, int64_t m, const float* scale,
                       const float* offset, uint16_t* idx, cudaStream_t st);
mpq_status launch_check_finite(const float* x, int64_t count, int* status, cudaStream_t st);

// tensor-core GEMM (gemm_tc.cu): C = diag(A.row_unscale) (A B^T) * b_scale
mpq_status make_tmap_f16(CUtensorMap* tm, const void* base, int64_t inner, int64_t rows,
                         int64_t ld_elems, int box_rows);
mpq_status split_global(const float* src, int64_t rows, int64_t K, SplitOperand* dst,
                        cudaStream_t st);
// The linear module's epilogue of the projection GEMM (p' = V^T (w - r2),
// one output element per (row, rank component l)): with F = gamma2 / (beta
// s_l^2 + gamma2) and u = s_l p', it accumulates per row and column tile
// sum F and sum F^2 u^2 + s_l^2 / (beta s_l^2 + gamma2) (the M-step's two
// traces), and writes the second GEMM's operand q = -F p' (full rank) or
// (1 - F) p' = D u as a fp16 hi/lo pair scaled by 2^-(e_row + e_bound):
// |p'| <= |w - r2|_2 <= sqrt(n) max|w - r2| (V has orthonormal columns), so
// with 2^e_bound >= sqrt(n) the scaled pair stays below 2^14 without a row
// reduction first.
struct LinEpi {
  const float* s32 = nullptr;      // r singular values
  const double* beta = nullptr;    // per row (before the M-step)
  const double* gamma2 = nullptr;  // per row
  int full_rank = 0;
  int e_bound = 0;
  __half* q_hi = nullptr;
  __half* q_lo = nullptr;
  int64_t ldq = 0;
  float2* part = nullptr;          // ntiles x rows (column tile major)
  int ntiles = 0;
  float* Uprime = nullptr;         // optional: (1 - F) p' (rows x r, fp32)
};

struct GemmOpts {
  int64_t b_k0 = 0;         // K offset into B (a multiple of 64)
  int64_t a_k0 = 0;         // K offset into A (a multiple of 64)
  int64_t n0 = 0;           // first output column (= first row of B)
  bool accumulate = false;  // C += result instead of C = result
  bool a_exact = false;     // A_lo is zero: skip its load and product
  const int* gate = nullptr;  // device int; 0 -> the launch does nothing
  // accumulate through TMA reduce-add into the fp32 matrix this map
  // describes (box 32 x 32, 128B swizzle) instead of a read-modify-write
  const CUtensorMap* c_reduce = nullptr;
  // the linear module's epilogue instead of storing C (C is not written)
  const LinEpi* lin = nullptr;
};
mpq_status make_tmap_f32_out(CUtensorMap* tm, const float* base, int64_t cols, int64_t rows,
                             int64_t ld_elems);
mpq_status gemm_tc(const SplitOperand& A, const CUtensorMap& ta_hi, const CUtensorMap& ta_lo,
                   const SplitOperand& B, const CUtensorMap& tb_hi, const CUtensorMap& tb_lo,
                   float* C, int64_t ldc, int64_t M, int64_t N, int64_t K, float b_scale_host,
                   int* status, cudaStream_t st, const char* tag, const GemmOpts& o = GemmOpts());

// tensor-core vector denoiser (denoise_tc.cu)
int vec_tc_grid_bits(const float* cb_host, int K, int* e_out, int* rk_out);  // -1: not eligible
mpq_status build_vec_tc_tables(mpq_plan_s* p, const float* cb_host);
mpq_status launch_denoise_vec_tc(const mpq_plan_s* p, const float* R1, const double* gamma1,
                                 const float* scale, const float* offset, int64_t m,
                                 const float* W, const double* gamma1_0, double inv_tau2,
                                 float* xhat1, float* vblock, uint16_t* idx, int mode,
                                 cudaStream_t st);  // mode: 0 full, 1 nearest, 2 MAP index only

// tensor-core candidate scan of the vector CD step (cd_scan_tc.cu)
int cd_scan_slices(int64_t m, int K);
// the greedy baseline's nearest-codeword scan on the tensor cores (block b,
// t = Wk[row, 8b..8b+7] / scale), partial minima as the CD scan's
mpq_status launch_ldlq_vec_scan(const mpq_plan_s* p, int64_t m, int64_t b, const float* scale,
                                const float* Wk, int64_t ldw, float* part_val, int* part_idx,
                                int nslices, cudaStream_t st);
mpq_status launch_cd_vec_scan(const mpq_plan_s* p, int64_t m, int64_t b, int64_t t0,
                              const float* scale, const uint16_t* idx, const float* h,
                              int64_t ldh, const float* hl, float* part_val, int* part_idx,
                              int nslices, cudaStream_t st);

// plan-time builders
mpq_status build_hessian(mpq_plan_s* p, cudaStream_t st);
mpq_status build_codebook_tables(mpq_plan_s* p, cudaStream_t st);
mpq_status setup_spectrum_from_x(mpq_plan_s* p, const float* X, int64_t m, int64_t n,
                                 cudaStream_t st);
// Spectrum from an accumulated Gram G = X^T X (n x n fp64, device, n = p->n)
// of m calibration rows: Jacobi eigenpairs, the same rank cut as from X.
mpq_status setup_spectrum_from_gram(mpq_plan_s* p, const double* G, int64_t m, cudaStream_t st);
// G (n x n fp64) += X^T X for X (rows x n fp32, device), fp64 products.
mpq_status gram_accumulate(double* G, int64_t n, const float* X, int64_t rows, cudaStream_t st);
// In place: every row x of X (rows x n) becomes (x .* signs) H_n / sqrt(n).
mpq_status launch_rht(float* X, int64_t rows, int64_t n, const float* signs, cudaStream_t st);

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace mpq
