// C ABI of libmpq: plans, workspace, the solve pipeline and the stage entry
// points.  The order of the pipeline follows the flowchart of "MPQ: A
// Message-Passing View of Post-Training Quantization" (papernotes.org note):
// init -> T_vamp x (denoiser, extrinsic update, rank-space linear module,
// beta M-step) -> marginal-MAP argmax -> exact block CD -> energies.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "mpq_internal.cuh"

namespace mpq {

static thread_local std::string g_last_error = "no error";
static std::atomic<int64_t> g_launches{0};

void set_error(const std::string& msg) { g_last_error = msg; }

mpq_status fail(mpq_status st, const std::string& msg) {
  set_error(msg);
  return st;
}

mpq_status cuda_fail(cudaError_t e, const char* what) {
  set_error(std::string(what) + ": " + cudaGetErrorString(e));
  return e == cudaErrorMemoryAllocation ? MPQ_ERR_OOM : MPQ_ERR_CUDA;
}

void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

mpq_status check_launch(const char* name) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, name);
  return MPQ_OK;
}

// ------------------------------------------------------------- profiling --
namespace {
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return e;
}
}  // namespace

bool profiling_on() {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  return g_prof_on;
}

ProfScope::ProfScope(const char* name, cudaStream_t stream) : st(stream) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on) return;
  ProfRec r{name, pool_event(), pool_event()};
  if (!r.a || !r.b) return;
  cudaEventRecord(r.a, st);
  slot = (int)g_prof.size();
  g_prof.push_back(r);
}

ProfScope::~ProfScope() {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (slot < (int)g_prof.size()) cudaEventRecord(g_prof[slot].b, st);
}

namespace {

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

__global__ void k_fill_f64(double* x, int64_t count, double v) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x)
    x[i] = v;
}

mpq_status fill_f64(double* x, int64_t count, double v, cudaStream_t st) {
  if (count <= 0) return MPQ_OK;
  {
    ProfScope ps_("k_fill_f64", st);
    k_fill_f64<<<(unsigned)std::min<int64_t>(cdiv(count, 256), 1024), 256, 0, st>>>(x, count, v);
  }
  count_launch();
  return check_launch("k_fill_f64");
}

mpq_status validate_params(const mpq_params* q, int64_t n) {
  if (!q) return fail(MPQ_ERR_INVALID_ARG, "params is NULL");
  if (q->d == 1) {
    if (q->K < 2 || q->K > 256) return fail(MPQ_ERR_INVALID_ARG, "d=1 needs 2 <= K <= 256");
    if (q->codebook) return fail(MPQ_ERR_INVALID_ARG, "d=1 takes no codebook (levels 0..K-1)");
  } else if (q->d == 8) {
    if (q->K < 1 || q->K > 65536) return fail(MPQ_ERR_INVALID_ARG, "d=8 needs 1 <= K <= 65536");
    if (!q->codebook) return fail(MPQ_ERR_INVALID_ARG, "d=8 needs a codebook");
  } else {
    return fail(MPQ_ERR_INVALID_ARG, "d must be 1 or 8");
  }
  if (n <= 0 || n % q->d != 0) return fail(MPQ_ERR_INVALID_ARG, "n must be a positive multiple of d");
  if (q->vec_engine < 0 || q->vec_engine > 2) return fail(MPQ_ERR_INVALID_ARG, "vec_engine must be 0, 1 or 2");
  if (q->cd_panel < 0 || q->cd_panel % 128)
    return fail(MPQ_ERR_INVALID_ARG, "cd_panel must be 0 or a positive multiple of 128");
  if (q->solve_graphs != 0 && q->solve_graphs != 1)
    return fail(MPQ_ERR_INVALID_ARG, "solve_graphs must be 0 or 1");
  if (!(q->cd_skip_precision >= 0.0))
    return fail(MPQ_ERR_INVALID_ARG, "cd_skip_precision must be >= 0 (0: never skip)");
  if (q->greedy_init != 0 && q->greedy_init != 1)
    return fail(MPQ_ERR_INVALID_ARG, "greedy_init must be 0 or 1");
  if (!(q->greedy_damp >= 0.0) || !std::isfinite(q->greedy_damp))
    return fail(MPQ_ERR_INVALID_ARG, "greedy_damp must be finite and >= 0");
  if (q->group_size < 0 || (q->group_size > 0 && (q->d != 1 || q->group_size % 128 ||
                                                   n % q->group_size)))
    return fail(MPQ_ERR_INVALID_ARG,
                "group_size must be 0, or for d = 1 a multiple of 128 that divides n");
  if (!(q->beta0 > 0.0) || !isfinite(q->beta0)) return fail(MPQ_ERR_INVALID_ARG, "beta0 must be > 0");
  if (!(q->damping >= 0.0 && q->damping <= 1.0)) return fail(MPQ_ERR_INVALID_ARG, "damping must be in [0,1]");
  if (!(q->tau > 0.0)) return fail(MPQ_ERR_INVALID_ARG, "tau must be > 0 (INFINITY = uniform prior)");
  if (!(q->gamma_lo_rel > 0.0 && q->gamma_lo_rel < q->gamma_hi_rel && isfinite(q->gamma_hi_rel)))
    return fail(MPQ_ERR_INVALID_ARG, "need 0 < gamma_lo_rel < gamma_hi_rel < inf");
  if (!(q->alpha_min > 0.0 && q->alpha_min < q->alpha_max && q->alpha_max < 1.0))
    return fail(MPQ_ERR_INVALID_ARG, "need 0 < alpha_min < alpha_max < 1");
  return MPQ_OK;
}

template <typename T>
mpq_status dalloc(T** p, int64_t count) {
  *p = nullptr;
  if (count <= 0) return MPQ_OK;
  cudaError_t e = cudaMalloc((void**)p, sizeof(T) * (size_t)count);
  if (e != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return fail(MPQ_ERR_OOM, std::string("cudaMalloc of ") + std::to_string(sizeof(T) * count) +
                                 " bytes failed: " + cudaGetErrorString(e));
  }
  return MPQ_OK;
}

template <typename T>
void dfree(T*& p) {
  if (p) cudaFree(p);
  p = nullptr;
}

void free_split(SplitOperand& s) {
  dfree(s.hi); dfree(s.lo); dfree(s.row_unscale); dfree(s.unscale);
  s = SplitOperand();
}

// fp16 hi/lo buffers: rows padded to 256, K to 64, zero-filled
mpq_status alloc_split(SplitOperand& s, int64_t rows, int64_t K, bool per_row) {
  s.rows = rows;
  s.rows_pad = round_up(std::max<int64_t>(rows, 1), 256);
  s.K = K;
  s.ld = round_up(K, 64);
  mpq_status st = dalloc(&s.hi, s.rows_pad * s.ld);
  if (st == MPQ_OK) st = dalloc(&s.lo, s.rows_pad * s.ld);
  if (st == MPQ_OK && per_row) st = dalloc(&s.row_unscale, s.rows_pad);
  if (st == MPQ_OK && !per_row) st = dalloc(&s.unscale, 1);
  if (st != MPQ_OK) return st;
  MPQ_CUDA(cudaMemset(s.hi, 0, sizeof(__half) * s.rows_pad * s.ld));
  MPQ_CUDA(cudaMemset(s.lo, 0, sizeof(__half) * s.rows_pad * s.ld));
  if (per_row) MPQ_CUDA(cudaMemset(s.row_unscale, 0, sizeof(float) * s.rows_pad));
  return MPQ_OK;
}

void free_workspace(Workspace& w) {
  dfree(w.R1); dfree(w.X1); dfree(w.R2); dfree(w.P); dfree(w.idx);
  free_split(w.As);
  free_split(w.Aq);
  dfree(w.lin_part);
  dfree(w.tile_count);
  dfree(w.Hg);
  dfree(w.Hl);
  dfree(w.scale); dfree(w.offset); dfree(w.sref); dfree(w.cd_skip); dfree(w.gamma1); dfree(w.gamma1_0); dfree(w.gamma2);
  dfree(w.beta); dfree(w.vsum); dfree(w.coef); dfree(w.kappa); dfree(w.clamps); dfree(w.W); dfree(w.w_hat);
  dfree(w.energy); dfree(w.idx_stage);
  w.rows = 0;
  w.bytes = 0;
}

constexpr int MAX_SWEEPS = 64;

int64_t ws_bytes_per_row(const mpq_plan_s* p) {
  return 3 * p->n * 4 + round_up(p->n, 32) * 4 + p->r * 4 +
         4 * round_up(std::max(p->n, p->r), CD_TILE) + 4 * round_up(p->r, CD_TILE) +
         8 * cdiv(p->r, CD_TILE) + p->B * 2 + 3 * 4 +
         8 * 8 + 4 + MAX_SWEEPS * 4 + (p->d == 8 ? CD_TILE * 4 : 0) + 8 * (p->ng - 1) + 8;
}

// changes buffer rides in the tail of `clamps`: rows x (1 + MAX_SWEEPS) ints
void drop_graphs(mpq_plan_s* p);

mpq_status ensure_workspace(mpq_plan_s* p, int64_t rows) {
  if (rows <= p->ws.rows) return MPQ_OK;
  const int64_t need = rows * ws_bytes_per_row(p);
  if (p->ws_cap > 0 && need > p->ws_cap)
    return fail(MPQ_ERR_OOM, "workspace of " + std::to_string(need) + " bytes exceeds the cap");
  MPQ_CUDA(cudaDeviceSynchronize());
  drop_graphs(p);  // they hold the old workspace's addresses
  ++p->ws_gen;
  free_workspace(p->ws);
  Workspace& w = p->ws;
  const int64_t mn = rows * p->n;
  mpq_status st = MPQ_OK;
  auto chk = [&](mpq_status s) { if (st == MPQ_OK) st = s; };
  chk(dalloc(&w.R1, mn)); chk(dalloc(&w.X1, mn)); chk(dalloc(&w.R2, mn));
  if (st == MPQ_OK)
    chk(alloc_split(w.As, rows, round_up(std::max(p->n, p->r), CD_TILE), true));
  if (st == MPQ_OK) chk(alloc_split(w.Aq, rows, round_up(p->r, CD_TILE), true));
  chk(dalloc(&w.lin_part, rows * cdiv(p->r, CD_TILE)));
  chk(dalloc(&w.tile_count, (int64_t)MAX_SWEEPS * 2 * cdiv(p->n, CD_TILE)));  // tiles + panels
  w.ldh = round_up(p->n, 32);
  chk(dalloc(&w.Hg, round_up(std::max<int64_t>(rows, 32), 32) * w.ldh));
  if (p->d == 8) chk(dalloc(&w.Hl, rows * CD_TILE));
  if (st == MPQ_OK)
    chk(make_tmap_f32_out(&w.tm_hg, w.Hg, std::max<int64_t>(p->n, 32),
                          round_up(std::max<int64_t>(rows, 32), 32), w.ldh));
  if (st == MPQ_OK)
    chk(make_tmap_f16(&w.tm_an_hi, w.As.hi, round_up(p->n, 64), w.As.rows_pad, w.As.ld, 128));
  if (st == MPQ_OK)
    chk(make_tmap_f16(&w.tm_an_lo, w.As.lo, round_up(p->n, 64), w.As.rows_pad, w.As.ld, 128));
  if (st == MPQ_OK)
    chk(make_tmap_f16(&w.tm_ar_hi, w.As.hi, round_up(p->r, 64), w.As.rows_pad, w.As.ld, 128));
  if (st == MPQ_OK)
    chk(make_tmap_f16(&w.tm_ar_lo, w.As.lo, round_up(p->r, 64), w.As.rows_pad, w.As.ld, 128));
  if (st == MPQ_OK)
    chk(make_tmap_f16(&w.tm_aq_hi, w.Aq.hi, round_up(p->r, 64), w.Aq.rows_pad, w.Aq.ld, 128));
  if (st == MPQ_OK)
    chk(make_tmap_f16(&w.tm_aq_lo, w.Aq.lo, round_up(p->r, 64), w.Aq.rows_pad, w.Aq.ld, 128));
  chk(dalloc(&w.P, rows * p->r)); chk(dalloc(&w.idx, rows * p->B));
  chk(dalloc(&w.scale, rows * p->ng)); chk(dalloc(&w.offset, rows * p->ng));
  chk(dalloc(&w.sref, rows));
  chk(dalloc(&w.cd_skip, rows));
  chk(dalloc(&w.gamma1, rows)); chk(dalloc(&w.gamma1_0, rows)); chk(dalloc(&w.gamma2, rows));
  chk(dalloc(&w.beta, rows)); chk(dalloc(&w.vsum, rows)); chk(dalloc(&w.coef, rows));
  chk(dalloc(&w.kappa, rows));
  chk(dalloc(&w.clamps, rows * (1 + MAX_SWEEPS)));
  if (st != MPQ_OK) {
    free_workspace(w);
    return st;
  }
  w.rows = rows;
  w.bytes = need;
  return MPQ_OK;
}

mpq_status ensure_host_staging(mpq_plan_s* p, int64_t rows) {
  Workspace& w = p->ws;
  // staging buffers follow the workspace row count
  if (w.W) return MPQ_OK;
  mpq_status st = MPQ_OK;
  auto chk = [&](mpq_status s) { if (st == MPQ_OK) st = s; };
  chk(dalloc(&w.W, rows * p->n));
  chk(dalloc(&w.w_hat, rows * p->n));
  chk(dalloc(&w.energy, rows));
  chk(dalloc(&w.idx_stage, rows * p->B));
  return st;
}

// --------------------------------------------------------- pipeline ------

struct SolveIO {
  const float* W;
  int64_t m;
  const float* row_scale;
  const float* row_offset;
  int T_vamp;
  int sweeps;
  uint16_t* idx;
  float* w_hat;
  float* energy;
  const mpq_row_stats* stats;
};

mpq_status run_linear_core(mpq_plan_s* p, int64_t m, double* gamma2, const double* gamma1_0,
                           double* beta, double* gamma1_out, float* Uprime, double* alpha2,
                           double* beta_hat, int32_t* clamps, cudaStream_t st,
                           LinFinish* defer_finish = nullptr);

// linear half-iteration on workspace state (R1 may alias W on the first call)
mpq_status run_linear(mpq_plan_s* p, const float* W, int64_t m, const float* R1,
                      const double* gamma1, const float* X1, const double* vsum,
                      const double* gamma1_0, double* beta, float* R1_out, double* gamma1_out,
                      float* R2, double* gamma2, float* Uprime, float* xhat2, double* alpha2,
                      double* beta_hat, int32_t* clamps, cudaStream_t st) {
  MPQ_TRY(launch_extrinsic_d2l(p, W, m, R1, gamma1, X1, vsum, gamma1_0, R2, &p->ws.As, gamma2,
                               clamps, st));
  MPQ_TRY(run_linear_core(p, m, gamma2, gamma1_0, beta, gamma1_out, Uprime, alpha2, beta_hat,
                          clamps, st));
  return launch_extrinsic_l2d(p, W, m, R2, p->ws.X1, p->ws.coef, p->ws.kappa, R1_out, xhat2, st);
}

// 2^e >= 2 sqrt(n): the linear epilogue's bound on |p'| over max|w - r2|
// (one bit of headroom over sqrt(n))
int linear_e_bound(int64_t n) {
  int e = 0;
  while ((double)(1ll << e) * (double)(1ll << e) < (double)n) ++e;
  return e + 1;
}

// the linear module on the split operand w - r2 already in As: p' = V^T
// (w - r2) with its epilogue (the diagonal scaling D, the M-step's trace
// sums, the second GEMM's operand D u), the M-step finisher, and G = V (D u)
// into X1
// defer_finish: the M-step finish is left to the caller's next fused row
// kernel (its arguments returned here), and the second GEMM takes its row
// scale as the first operand's times 2^e_bound (what the finish would write)
mpq_status run_linear_core(mpq_plan_s* p, int64_t m, double* gamma2, const double* gamma1_0,
                           double* beta, double* gamma1_out, float* Uprime, double* alpha2,
                           double* beta_hat, int32_t* clamps, cudaStream_t st,
                           LinFinish* defer_finish) {
  Workspace& w = p->ws;
  const int64_t n = p->n, r = p->r;
  LinEpi le;
  le.s32 = p->s32;
  le.beta = beta;
  le.gamma2 = gamma2;
  le.full_rank = (r == n) ? 1 : 0;
  le.e_bound = linear_e_bound(n);
  le.q_hi = w.Aq.hi;
  le.q_lo = w.Aq.lo;
  le.ldq = w.Aq.ld;
  le.part = w.lin_part;
  le.ntiles = (int)cdiv(r, CD_TILE);
  le.Uprime = Uprime;
  GemmOpts o;
  o.lin = &le;
  MPQ_TRY(gemm_tc(w.As, w.tm_an_hi, w.tm_an_lo, p->Vt_s, p->tm_vt_hi, p->tm_vt_lo, w.P, r, m, r, n,
                  p->Vt_s.unscale_host, p->status, st, "gemm_project", o));
  if (defer_finish) {
    *defer_finish = make_lin_finish(p, m, w.lin_part, le.ntiles, le.e_bound, w.As.row_unscale,
                                    nullptr, gamma2, gamma1_0, beta, gamma1_out, w.coef, w.kappa,
                                    alpha2, beta_hat, clamps);
    SplitOperand aq = w.Aq;
    aq.row_unscale = w.As.row_unscale;  // times 2^e_bound, folded into b_scale (exact)
    return gemm_tc(aq, w.tm_aq_hi, w.tm_aq_lo, p->V_s, p->tm_v_hi, p->tm_v_lo, w.X1, n, m, n, r,
                   ldexpf(p->V_s.unscale_host, le.e_bound), p->status, st, "gemm_expand");
  }
  MPQ_TRY(launch_linear_finish(p, m, w.lin_part, le.ntiles, le.e_bound, w.As.row_unscale,
                               w.Aq.row_unscale, gamma2, gamma1_0, beta, gamma1_out, w.coef,
                               w.kappa, alpha2, beta_hat, clamps, st));
  // G into X1: the denoiser output is consumed by now
  return gemm_tc(w.Aq, w.tm_aq_hi, w.tm_aq_lo, p->V_s, p->tm_v_hi, p->tm_v_lo, w.X1, n, m, n, r,
                 p->V_s.unscale_host, p->status, st, "gemm_expand");
}

mpq_status run_cd(mpq_plan_s* p, const float* W, int64_t m, const float* scale,
                  const float* offset, uint16_t* idx, int sweeps, int32_t* changes,
                  cudaStream_t st, const double* gamma1 = nullptr) {
  Workspace& w = p->ws;
  const int64_t n = p->n;
  MPQ_TRY(launch_residual_split(p, W, m, scale, offset, idx, &w.As, nullptr, st));
  // h = H (w - x), in its own padded buffer (the CD updates reduce into it)
  MPQ_TRY(gemm_tc(w.As, w.tm_an_hi, w.tm_an_lo, p->H_s, p->tm_h_hi, p->tm_h_lo, w.Hg, w.ldh, m, n,
                  n, p->H_s.unscale_host, p->status, st, "gemm_hessian"));
  // adaptive CD (solve only: it needs the terminal precision)
  const int32_t* skip = nullptr;
  if (gamma1 && p->params.cd_skip_precision > 0.0) {
    MPQ_TRY(launch_cd_skip(gamma1, scale, m, p->ng, p->params.cd_skip_precision, w.cd_skip, st));
    skip = w.cd_skip;
  }
  return launch_cd(p, W, m, scale, offset, idx, w.Hg, w.ldh, sweeps, changes, st, skip);
}

mpq_status run_energy(mpq_plan_s* p, const float* W, int64_t m, const float* scale,
                      const float* offset, const uint16_t* idx, float* w_hat, float* energy,
                      cudaStream_t st) {
  Workspace& w = p->ws;
  const int64_t n = p->n, r = p->r;
  MPQ_TRY(launch_residual_split(p, W, m, scale, offset, idx, &w.As, w_hat, st));
  if (!energy) return MPQ_OK;
  MPQ_TRY(gemm_tc(w.As, w.tm_an_hi, w.tm_an_lo, p->Vt_s, p->tm_vt_hi, p->tm_vt_lo, w.P, r, m, r, n,
                  p->Vt_s.unscale_host, p->status, st, "gemm_energy"));
  return launch_energy_rows(p, m, w.P, energy, st);
}

// one batch of rows, all device pointers
mpq_status solve_batch(mpq_plan_s* p, const SolveIO& io, int64_t row0, int64_t mb,
                       cudaStream_t st) {
  Workspace& w = p->ws;
  const int64_t n = p->n, B = p->B;
  const float* W = io.W + row0 * n;
  uint16_t* idx = io.idx + row0 * B;
  const int given = io.row_scale != nullptr;
  if (given) {
    const int64_t ng = p->ng;
    MPQ_CUDA(cudaMemcpyAsync(w.scale, io.row_scale + row0 * ng, sizeof(float) * mb * ng,
                             cudaMemcpyDeviceToDevice, st));
    MPQ_CUDA(cudaMemcpyAsync(w.offset, io.row_offset + row0 * ng, sizeof(float) * mb * ng,
                             cudaMemcpyDeviceToDevice, st));
  }
  int32_t* clamps = w.clamps;
  int32_t* changes = w.clamps + w.rows;  // rows x MAX_SWEEPS
  MPQ_CUDA(cudaMemsetAsync(clamps, 0, sizeof(int32_t) * mb, st));
  // init: scale/offset, round-to-nearest (into idx), gamma1_0.  A greedy
  // vector solve overwrites idx with the greedy pass and reads gamma1_0 only
  // for adaptive CD or the row statistics: without those it skips the
  // round-to-nearest pass
  const bool rtn = !(io.T_vamp == 0 && p->params.greedy_init && p->d == 8 &&
                     !(p->params.cd_skip_precision > 0.0) && io.stats == nullptr);
  MPQ_TRY(launch_init(p, W, mb, given, w.scale, w.offset, idx, w.gamma1_0, st, rtn));
  if (!rtn) MPQ_TRY(fill_f64(w.gamma1_0, mb, 0.0, st));
  MPQ_CUDA(cudaMemcpyAsync(w.gamma1, w.gamma1_0, sizeof(double) * mb, cudaMemcpyDeviceToDevice, st));
  MPQ_TRY(fill_f64(w.beta, mb, p->params.beta0, st));
  if (p->d == 1 && vamp_row_threads(n, p->G) > 0) {
    // scalar rows: l2d, denoiser and d2l of an iteration in one fused row
    // kernel (r1 never leaves the chip), then the linear module
    // (each linear step's M-step finish runs in the next row kernel's prologue)
    LinFinish fin{};
    for (int t = 0; t < io.T_vamp; ++t) {
      MPQ_TRY(launch_vamp_row_scalar(p, W, mb, t == 0, 0, w.X1, w.R2, w.coef, w.kappa, w.gamma1,
                                     w.scale, w.offset, w.gamma1_0, &w.As, w.gamma2, clamps,
                                     nullptr, st, nullptr, t > 0 ? &fin : nullptr));
      MPQ_TRY(run_linear_core(p, mb, w.gamma2, w.gamma1_0, w.beta, w.gamma1, nullptr, nullptr,
                              nullptr, clamps, st, &fin));
    }
    // marginal MAP: argmax of the denoiser at the last cavity
    if (io.T_vamp > 0)
      MPQ_TRY(launch_vamp_row_scalar(p, W, mb, 0, 1, w.X1, w.R2, w.coef, w.kappa, w.gamma1,
                                     w.scale, w.offset, w.gamma1_0, nullptr, nullptr, nullptr, idx,
                                     st, nullptr, &fin));
  } else {
    const float* R1 = W;  // cavity r1_0 = w
    float* vblock = (p->d == 8) ? w.R2 : nullptr;  // R2 is free while the denoiser runs
    for (int t = 0; t < io.T_vamp; ++t) {
      MPQ_TRY(launch_denoise(p, R1, w.gamma1, w.scale, w.offset, mb, W, w.gamma1_0, w.X1, vblock,
                             w.vsum, nullptr, st));
      MPQ_TRY(run_linear(p, W, mb, R1, w.gamma1, w.X1, w.vsum, w.gamma1_0, w.beta, w.R1,
                         w.gamma1, w.R2, w.gamma2, nullptr, nullptr, nullptr, nullptr, clamps, st));
      R1 = w.R1;
    }
    // marginal MAP: argmax of one more denoiser call (only the index is used)
    if (io.T_vamp > 0)
      MPQ_TRY(launch_denoise(p, R1, w.gamma1, w.scale, w.offset, mb, W, w.gamma1_0, w.X1, vblock,
                             w.vsum, idx, st, /*map_only=*/true));
  }
  // the greedy baseline replaces round-to-nearest as the hard init
  if (io.T_vamp == 0 && p->params.greedy_init)
    MPQ_TRY(launch_ldlq(p, W, mb, w.scale, w.offset, idx, st));
  if (io.sweeps > 0)
    MPQ_TRY(run_cd(p, W, mb, w.scale, w.offset, idx, io.sweeps, changes, st, w.gamma1));
  MPQ_TRY(run_energy(p, W, mb, w.scale, w.offset, idx, io.w_hat ? io.w_hat + row0 * n : nullptr,
                     io.energy ? io.energy + row0 : nullptr, st));
  if (io.stats) {
    const mpq_row_stats* s = io.stats;
    if (s->gamma1) MPQ_CUDA(cudaMemcpyAsync(s->gamma1 + row0, w.gamma1, sizeof(double) * mb, cudaMemcpyDeviceToDevice, st));
    if (s->beta) MPQ_CUDA(cudaMemcpyAsync(s->beta + row0, w.beta, sizeof(double) * mb, cudaMemcpyDeviceToDevice, st));
    if (s->clamps) MPQ_CUDA(cudaMemcpyAsync(s->clamps + row0, clamps, sizeof(int32_t) * mb, cudaMemcpyDeviceToDevice, st));
    if (s->cd_changes && io.sweeps > 0)
      MPQ_CUDA(cudaMemcpyAsync(s->cd_changes + row0 * io.sweeps, changes, sizeof(int32_t) * mb * io.sweeps, cudaMemcpyDeviceToDevice, st));
  }
  return MPQ_OK;
}

mpq_status solve_device(mpq_plan_s* p, const SolveIO& io, cudaStream_t st) {
  if (io.m <= 0) return MPQ_OK;
  int64_t rows = io.m;
  if (p->ws_cap > 0) {
    const int64_t fit = p->ws_cap / ws_bytes_per_row(p);
    if (fit < 1) return fail(MPQ_ERR_OOM, "workspace cap is below one row");
    rows = std::min(rows, fit);
  }
  MPQ_TRY(ensure_workspace(p, rows));
  auto run = [&](cudaStream_t s) -> mpq_status {
    for (int64_t r0 = 0; r0 < io.m; r0 += rows)
      MPQ_TRY(solve_batch(p, io, r0, std::min(rows, io.m - r0), s));
    return MPQ_OK;
  };
  if (!p->params.solve_graphs || profiling_on()) return run(st);
  // the call's identity: buffers, sizes, options and the workspace generation
  uint64_t key[mpq_plan_s::GRAPH_KEY] = {
      (uint64_t)(uintptr_t)io.W, (uint64_t)io.m, (uint64_t)(uintptr_t)io.row_scale,
      (uint64_t)(uintptr_t)io.row_offset, (uint64_t)io.T_vamp, (uint64_t)io.sweeps,
      (uint64_t)(uintptr_t)io.idx, (uint64_t)(uintptr_t)io.w_hat,
      (uint64_t)(uintptr_t)io.energy, 0, 0, 0, 0, (uint64_t)rows, p->ws_gen, 1};
  if (io.stats) {
    key[9] = (uint64_t)(uintptr_t)io.stats->gamma1;
    key[10] = (uint64_t)(uintptr_t)io.stats->beta;
    key[11] = (uint64_t)(uintptr_t)io.stats->clamps;
    key[12] = (uint64_t)(uintptr_t)io.stats->cd_changes;
  }
  mpq_plan_s::SolveGraph* seen = nullptr;
  for (auto& gr : p->graphs) {
    if (gr.last_use && std::equal(key, key + mpq_plan_s::GRAPH_KEY, gr.key)) {
      gr.last_use = ++p->graph_clock;
      if (!gr.exec) {
        seen = &gr;
        break;
      }
      MPQ_CUDA(cudaGraphLaunch(gr.exec, st));
      count_launch((int)gr.launches);
      return MPQ_OK;
    }
  }
  auto lru = [&]() {
    mpq_plan_s::SolveGraph* s = &p->graphs[0];
    for (auto& gr : p->graphs)
      if (gr.last_use < s->last_use) s = &gr;
    return s;
  };
  if (!seen) {
    // a call seen for the first time runs directly; the second one captures
    mpq_plan_s::SolveGraph* s = lru();
    if (s->exec) cudaGraphExecDestroy(s->exec);
    *s = mpq_plan_s::SolveGraph{};
    std::copy(key, key + mpq_plan_s::GRAPH_KEY, s->key);
    s->last_use = ++p->graph_clock;
    return run(st);
  }
  // capture the launches on a private stream (the caller's may be the legacy
  // default stream, which cannot be captured); anything that fails to
  // capture runs directly instead
  if (!p->capture_stream)
    MPQ_CUDA(cudaStreamCreateWithFlags(&p->capture_stream, cudaStreamNonBlocking));
  if (cudaStreamBeginCapture(p->capture_stream, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaGetLastError();
    return run(st);
  }
  const int64_t l0 = mpq_kernel_launch_count();
  const mpq_status rc = run(p->capture_stream);
  cudaGraph_t graph = nullptr;
  const cudaError_t ce = cudaStreamEndCapture(p->capture_stream, &graph);
  const int64_t nl = mpq_kernel_launch_count() - l0;
  count_launch((int)-nl);  // nothing ran yet
  cudaGraphExec_t exec = nullptr;
  const bool ok = rc == MPQ_OK && ce == cudaSuccess && graph &&
                  cudaGraphInstantiate(&exec, graph, 0) == cudaSuccess;
  if (graph) cudaGraphDestroy(graph);
  if (!ok) {
    cudaGetLastError();
    return run(st);
  }
  seen->exec = exec;
  seen->launches = nl;
  MPQ_CUDA(cudaGraphLaunch(exec, st));
  count_launch((int)nl);
  return MPQ_OK;
}

mpq_status finish_plan(mpq_plan_s* p, cudaStream_t st) {
  const int64_t n = p->n, r = p->r;
  MPQ_TRY(dalloc(&p->s32, r));
  MPQ_TRY(dalloc(&p->V32, n * r));
  MPQ_TRY(dalloc(&p->Vt32, r * n));
  MPQ_TRY(dalloc(&p->H32, n * n));
  MPQ_TRY(dalloc(&p->Hdiag, n));
  MPQ_TRY(dalloc(&p->status, 1));
  MPQ_CUDA(cudaMemsetAsync(p->status, 0, sizeof(int), st));
  MPQ_TRY(build_hessian(p, st));
  MPQ_TRY(alloc_split(p->Vt_s, r, n, false));
  MPQ_TRY(alloc_split(p->V_s, n, r, false));
  MPQ_TRY(alloc_split(p->H_s, n, n, false));
  MPQ_TRY(split_global(p->Vt32, r, n, &p->Vt_s, st));
  MPQ_TRY(split_global(p->V32, n, r, &p->V_s, st));
  MPQ_TRY(split_global(p->H32, n, n, &p->H_s, st));
  MPQ_CUDA(cudaMemcpyAsync(&p->Vt_s.unscale_host, p->Vt_s.unscale, sizeof(float), cudaMemcpyDeviceToHost, st));
  MPQ_CUDA(cudaMemcpyAsync(&p->V_s.unscale_host, p->V_s.unscale, sizeof(float), cudaMemcpyDeviceToHost, st));
  MPQ_CUDA(cudaMemcpyAsync(&p->H_s.unscale_host, p->H_s.unscale, sizeof(float), cudaMemcpyDeviceToHost, st));
  MPQ_TRY(make_tmap_f16(&p->tm_vt_hi, p->Vt_s.hi, p->Vt_s.ld, p->Vt_s.rows_pad, p->Vt_s.ld, 128));
  MPQ_TRY(make_tmap_f16(&p->tm_vt_lo, p->Vt_s.lo, p->Vt_s.ld, p->Vt_s.rows_pad, p->Vt_s.ld, 128));
  MPQ_TRY(make_tmap_f16(&p->tm_v_hi, p->V_s.hi, p->V_s.ld, p->V_s.rows_pad, p->V_s.ld, 128));
  MPQ_TRY(make_tmap_f16(&p->tm_v_lo, p->V_s.lo, p->V_s.ld, p->V_s.rows_pad, p->V_s.ld, 128));
  MPQ_TRY(make_tmap_f16(&p->tm_h_hi, p->H_s.hi, p->H_s.ld, p->H_s.rows_pad, p->H_s.ld, 128));
  MPQ_TRY(make_tmap_f16(&p->tm_h_lo, p->H_s.lo, p->H_s.ld, p->H_s.rows_pad, p->H_s.ld, 128));
  if (p->params.greedy_init) {
    const int64_t nt = cdiv(n, CD_TILE);
    MPQ_TRY(dalloc(&p->ldlq_diag, nt * CD_TILE * CD_TILE));
    MPQ_CUDA(cudaMemsetAsync(p->ldlq_diag, 0, sizeof(float) * nt * CD_TILE * CD_TILE, st));
    float* Bl = nullptr;
    MPQ_TRY(dalloc(&Bl, n * n));
    mpq_status rc = ldlq_factor(p, p->params.greedy_damp, Bl, p->ldlq_diag, st);
    if (rc == MPQ_OK) rc = alloc_split(p->Lq_s, n, n, false);
    if (rc == MPQ_OK) rc = split_global(Bl, n, n, &p->Lq_s, st);
    if (rc == MPQ_OK) {
      cudaError_t e = cudaMemcpyAsync(&p->Lq_s.unscale_host, p->Lq_s.unscale, sizeof(float),
                                      cudaMemcpyDeviceToHost, st);
      if (e == cudaSuccess) e = cudaStreamSynchronize(st);
      if (e != cudaSuccess) rc = cuda_fail(e, "greedy factor");
    }
    dfree(Bl);
    MPQ_TRY(rc);
    MPQ_TRY(make_tmap_f16(&p->tm_lq_hi, p->Lq_s.hi, p->Lq_s.ld, p->Lq_s.rows_pad, p->Lq_s.ld, 128));
    MPQ_TRY(make_tmap_f16(&p->tm_lq_lo, p->Lq_s.lo, p->Lq_s.ld, p->Lq_s.rows_pad, p->Lq_s.ld, 128));
  }
  if (p->d == 8) {
    MPQ_TRY(dalloc(&p->cb_norm, p->K));
    MPQ_TRY(dalloc(&p->cb_hnorm, p->K));
    MPQ_TRY(dalloc(&p->qtab, p->B * (int64_t)p->K));
    MPQ_TRY(build_codebook_tables(p, st));
  }
  MPQ_CUDA(cudaStreamSynchronize(st));
  return MPQ_OK;
}

void drop_graphs(mpq_plan_s* p) {
  for (auto& gr : p->graphs) {
    if (gr.exec) cudaGraphExecDestroy(gr.exec);
    gr = mpq_plan_s::SolveGraph{};
  }
}

void destroy_plan(mpq_plan_s* p) {
  if (!p) return;
  DeviceGuard g(p->device);
  drop_graphs(p);
  if (p->capture_stream) cudaStreamDestroy(p->capture_stream);
  free_workspace(p->ws);
  dfree(p->s64); dfree(p->V64); dfree(p->s32); dfree(p->V32); dfree(p->Vt32); dfree(p->H32);
  dfree(p->Hdiag); dfree(p->cb); dfree(p->cb_norm); dfree(p->cb_hnorm); dfree(p->qtab); dfree(p->status);
  if (p->cb_tc) cudaFree(p->cb_tc);
  free_split(p->Vt_s); free_split(p->V_s); free_split(p->H_s); free_split(p->Lq_s);
  dfree(p->ldlq_diag);
  delete p;
}

mpq_status new_plan(const mpq_params* params, int64_t n, mpq_plan_s** out) {
  MPQ_TRY(validate_params(params, n));
  mpq_plan_s* p = new mpq_plan_s();
  MPQ_CUDA(cudaGetDevice(&p->device));
  p->params = *params;
  p->params.codebook = nullptr;
  p->n = n;
  p->d = params->d;
  p->K = params->K;
  p->B = n / params->d;
  p->G = params->group_size;
  p->ng = p->G ? n / p->G : 1;
  if (p->d == 8) {
    mpq_status st = dalloc(&p->cb, (int64_t)p->K * 8);
    if (st == MPQ_OK) {
      cudaError_t e = cudaMemcpy(p->cb, params->codebook, sizeof(float) * p->K * 8, cudaMemcpyHostToDevice);
      if (e != cudaSuccess) st = cuda_fail(e, "codebook copy");
    }
    if (st == MPQ_OK && params->vec_engine != 1) {
      int e = 0;
      p->vec_tc_F = vec_tc_grid_bits(params->codebook, p->K, &e, &p->vec_tc_rk);
      p->vec_tc_Fmin = e + 1;
      p->vec_tc = p->vec_tc_F > 0;
      if (!p->vec_tc && params->vec_engine == 2)
        st = fail(MPQ_ERR_UNSUPPORTED, "codebook does not qualify for the tensor-core denoiser");
      if (st == MPQ_OK && p->vec_tc) st = build_vec_tc_tables(p, params->codebook);
    }
    if (st != MPQ_OK) {
      destroy_plan(p);
      return st;
    }
  }
  *out = p;
  return MPQ_OK;
}

#define PLAN_CHECK(p)                                                      \
  do {                                                                     \
    if (!(p)) return ::mpq::fail(MPQ_ERR_INVALID_ARG, "plan is NULL");     \
  } while (0)

// row counts index the grid's x dimension (one CTA or warp group per row)
#define ROWS_CHECK(m)                                                      \
  do {                                                                     \
    if ((m) > ::mpq::MAX_ROWS)                                             \
      return ::mpq::fail(MPQ_ERR_INVALID_ARG, "row count above 2^31 - 1"); \
  } while (0)

}  // namespace
}  // namespace mpq

using namespace mpq;

extern "C" {

void mpq_params_default(mpq_params* p, int32_t d, int32_t K) {
  if (!p) return;
  memset(p, 0, sizeof(*p));
  p->d = d;
  p->K = K;
  p->codebook = nullptr;
  p->beta0 = 1.0;
  p->damping = 0.5;
  p->tau = 0.2;
  p->gamma_lo_rel = 1e-10;
  p->gamma_hi_rel = 1e10;
  p->alpha_min = 1e-10;
  p->alpha_max = 0.99;
  p->vec_engine = 0;
  p->cd_panel = 0;
  p->group_size = 0;
  p->solve_graphs = 1;
  p->cd_skip_precision = 0.0;
  p->greedy_init = 0;
  p->greedy_damp = 0.01;
}

mpq_status mpq_plan_create_from_spectrum(const double* s, const double* V, int64_t n, int64_t r,
                                         const mpq_params* params, mpq_stream_t stream,
                                         mpq_plan_t* plan) {
  if (!plan) return fail(MPQ_ERR_INVALID_ARG, "plan out-pointer is NULL");
  *plan = nullptr;
  if (!s || !V) return fail(MPQ_ERR_INVALID_ARG, "s and V must be device pointers");
  if (r < 1 || r > n) return fail(MPQ_ERR_INVALID_ARG, "need 1 <= r <= n");
  cudaStream_t st = (cudaStream_t)stream;
  mpq_plan_s* p = nullptr;
  MPQ_TRY(new_plan(params, n, &p));
  p->r = r;
  mpq_status rc = dalloc(&p->s64, r);
  if (rc == MPQ_OK) rc = dalloc(&p->V64, n * r);
  if (rc == MPQ_OK) {
    cudaError_t e = cudaMemcpyAsync(p->s64, s, sizeof(double) * r, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(p->V64, V, sizeof(double) * n * r, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) rc = cuda_fail(e, "spectrum copy");
  }
  if (rc == MPQ_OK) {
    std::vector<double> hs(r);
    cudaError_t e = cudaMemcpyAsync(hs.data(), p->s64, sizeof(double) * r, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) rc = cuda_fail(e, "spectrum read-back");
    for (int64_t l = 0; rc == MPQ_OK && l < r; ++l)
      if (!(hs[l] > 0.0) || !isfinite(hs[l]))
        rc = fail(MPQ_ERR_INVALID_ARG, "singular values must be finite and > 0");
  }
  if (rc == MPQ_OK) rc = finish_plan(p, st);
  if (rc != MPQ_OK) {
    destroy_plan(p);
    return rc;
  }
  *plan = p;
  return MPQ_OK;
}

mpq_status mpq_plan_create_from_x(const float* X, int64_t m, int64_t n, const mpq_params* params,
                                  mpq_stream_t stream, mpq_plan_t* plan) {
  if (!plan) return fail(MPQ_ERR_INVALID_ARG, "plan out-pointer is NULL");
  *plan = nullptr;
  if (!X || m < 1 || n < 1) return fail(MPQ_ERR_INVALID_ARG, "X must be a device m x n matrix");
  cudaStream_t st = (cudaStream_t)stream;
  mpq_plan_s* p = nullptr;
  MPQ_TRY(new_plan(params, n, &p));
  mpq_status rc = setup_spectrum_from_x(p, X, m, n, st);
  if (rc == MPQ_OK) rc = finish_plan(p, st);
  if (rc != MPQ_OK) {
    destroy_plan(p);
    return rc;
  }
  *plan = p;
  return MPQ_OK;
}

// ------------------------------------------------ streamed calibration ---
struct mpq_gram_s {
  int device = 0;
  int64_t n = 0;
  int64_t rows = 0;
  double* G = nullptr;  // n x n, fp64, device
};

mpq_status mpq_gram_create(int64_t n, mpq_stream_t stream, mpq_gram_t* gram) {
  if (!gram) return fail(MPQ_ERR_INVALID_ARG, "gram out-pointer is NULL");
  *gram = nullptr;
  if (n < 1 || n > (int64_t)1 << 17) return fail(MPQ_ERR_INVALID_ARG, "gram: n must be in [1, 131072]");
  cudaStream_t st = (cudaStream_t)stream;
  mpq_gram_s* g = new mpq_gram_s();
  g->n = n;
  mpq_status rc = MPQ_OK;
  cudaError_t e = cudaGetDevice(&g->device);
  if (e == cudaSuccess) e = cudaMalloc((void**)&g->G, sizeof(double) * n * n);
  if (e == cudaSuccess) e = cudaMemsetAsync(g->G, 0, sizeof(double) * n * n, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) rc = cuda_fail(e, "gram allocation");
  if (rc != MPQ_OK) {
    mpq_gram_destroy(g);
    return rc;
  }
  *gram = g;
  return MPQ_OK;
}

mpq_status mpq_gram_accumulate(mpq_gram_t g, const float* X, int64_t rows, mpq_stream_t stream) {
  if (!g) return fail(MPQ_ERR_INVALID_ARG, "gram is NULL");
  if (rows < 0 || (rows > 0 && !X)) return fail(MPQ_ERR_INVALID_ARG, "X must be a device rows x n matrix");
  DeviceGuard dg(g->device);
  MPQ_TRY(gram_accumulate(g->G, g->n, X, rows, (cudaStream_t)stream));
  g->rows += rows;
  return MPQ_OK;
}

mpq_status mpq_gram_info(mpq_gram_t g, int64_t* n, int64_t* rows) {
  if (!g) return fail(MPQ_ERR_INVALID_ARG, "gram is NULL");
  if (n) *n = g->n;
  if (rows) *rows = g->rows;
  return MPQ_OK;
}

mpq_status mpq_gram_get(mpq_gram_t g, double* G, mpq_stream_t stream) {
  if (!g || !G) return fail(MPQ_ERR_INVALID_ARG, "gram and G must be non-NULL");
  DeviceGuard dg(g->device);
  MPQ_CUDA(cudaMemcpyAsync(G, g->G, sizeof(double) * g->n * g->n, cudaMemcpyDeviceToDevice,
                           (cudaStream_t)stream));
  return MPQ_OK;
}

mpq_status mpq_gram_destroy(mpq_gram_t g) {
  if (!g) return MPQ_OK;
  if (g->G) cudaFree(g->G);
  delete g;
  return MPQ_OK;
}

mpq_status mpq_plan_create_from_gram(mpq_gram_t g, const mpq_params* params, mpq_stream_t stream,
                                     mpq_plan_t* plan) {
  if (!plan) return fail(MPQ_ERR_INVALID_ARG, "plan out-pointer is NULL");
  *plan = nullptr;
  if (!g) return fail(MPQ_ERR_INVALID_ARG, "gram is NULL");
  if (g->rows < 1) return fail(MPQ_ERR_RANK, "gram holds no calibration rows");
  DeviceGuard dg(g->device);
  cudaStream_t st = (cudaStream_t)stream;
  mpq_plan_s* p = nullptr;
  MPQ_TRY(new_plan(params, g->n, &p));
  mpq_status rc = setup_spectrum_from_gram(p, g->G, g->rows, st);
  if (rc == MPQ_OK) rc = finish_plan(p, st);
  if (rc != MPQ_OK) {
    destroy_plan(p);
    return rc;
  }
  *plan = p;
  return MPQ_OK;
}

mpq_status mpq_rht(float* X, int64_t rows, int64_t n, const float* signs, mpq_stream_t stream) {
  if (n < 1 || n > MPQ_RHT_MAX_N || (n & (n - 1)))
    return fail(MPQ_ERR_INVALID_ARG, "rht: n must be a power of two in [1, 32768]");
  if (rows < 0 || (rows > 0 && (!X || !signs)))
    return fail(MPQ_ERR_INVALID_ARG, "rht: X (rows x n) and signs (n) must be device buffers");
  return launch_rht(X, rows, n, signs, (cudaStream_t)stream);
}

mpq_status mpq_plan_destroy(mpq_plan_t plan) {
  destroy_plan(plan);
  return MPQ_OK;
}

mpq_status mpq_plan_info(mpq_plan_t p, int64_t* n, int64_t* r, int32_t* d, int32_t* K) {
  PLAN_CHECK(p);
  if (n) *n = p->n;
  if (r) *r = p->r;
  if (d) *d = p->d;
  if (K) *K = p->K;
  return MPQ_OK;
}

mpq_status mpq_plan_get_spectrum(mpq_plan_t p, double* s, double* V, mpq_stream_t stream) {
  PLAN_CHECK(p);
  DeviceGuard g(p->device);
  cudaStream_t st = (cudaStream_t)stream;
  if (s) MPQ_CUDA(cudaMemcpyAsync(s, p->s64, sizeof(double) * p->r, cudaMemcpyDeviceToDevice, st));
  if (V) MPQ_CUDA(cudaMemcpyAsync(V, p->V64, sizeof(double) * p->n * p->r, cudaMemcpyDeviceToDevice, st));
  return MPQ_OK;
}

mpq_status mpq_plan_status(mpq_plan_t p, mpq_stream_t stream) {
  PLAN_CHECK(p);
  DeviceGuard g(p->device);
  MPQ_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
  int word = 0;
  MPQ_CUDA(cudaMemcpy(&word, p->status, sizeof(int), cudaMemcpyDeviceToHost));
  MPQ_CUDA(cudaMemset(p->status, 0, sizeof(int)));
  if (word & STATUS_NONFINITE) return fail(MPQ_ERR_NONFINITE, "non-finite value in an input row");
  if (word & STATUS_TIMEOUT) return fail(MPQ_ERR_TIMEOUT, "a bounded device loop reached its cap");
  if (word & STATUS_BADINDEX) return fail(MPQ_ERR_INVALID_ARG, "a codeword index was >= K (clamped)");
  return MPQ_OK;
}

int64_t mpq_plan_workspace_bytes(mpq_plan_t p, int64_t m_out) {
  if (!p || m_out < 0) return -1;
  return m_out * ws_bytes_per_row(p);
}

mpq_status mpq_plan_set_workspace_cap(mpq_plan_t p, int64_t cap_bytes) {
  PLAN_CHECK(p);
  if (cap_bytes < 0) return fail(MPQ_ERR_INVALID_ARG, "cap must be >= 0");
  p->ws_cap = cap_bytes;
  return MPQ_OK;
}

mpq_status mpq_solve(mpq_plan_t p, const float* W, int64_t m_out, const float* row_scale,
                     const float* row_offset, int32_t T_vamp, int32_t cd_sweeps, uint16_t* idx,
                     float* w_hat, float* energy, const mpq_row_stats* stats,
                     mpq_stream_t stream) {
  PLAN_CHECK(p);
  if (m_out < 0) return fail(MPQ_ERR_INVALID_ARG, "m_out must be >= 0");
  if (m_out > 0 && (!W || !idx)) return fail(MPQ_ERR_INVALID_ARG, "W and idx are required");
  if ((row_scale == nullptr) != (row_offset == nullptr))
    return fail(MPQ_ERR_INVALID_ARG, "row_scale and row_offset go together");
  if (T_vamp < 0) return fail(MPQ_ERR_INVALID_ARG, "T_vamp must be >= 0");
  if (cd_sweeps < 0 || cd_sweeps > MAX_SWEEPS) return fail(MPQ_ERR_INVALID_ARG, "cd_sweeps must be in [0, 64]");
  ROWS_CHECK(m_out);
  DeviceGuard g(p->device);
  SolveIO io{W, m_out, row_scale, row_offset, T_vamp, cd_sweeps, idx, w_hat, energy, stats};
  return solve_device(p, io, (cudaStream_t)stream);
}

mpq_status mpq_solve_host(mpq_plan_t p, const float* W_host, int64_t m_out, int32_t T_vamp,
                          int32_t cd_sweeps, uint16_t* idx_host, float* w_hat_host,
                          float* energy_host, mpq_stream_t stream) {
  PLAN_CHECK(p);
  if (m_out < 0) return fail(MPQ_ERR_INVALID_ARG, "m_out must be >= 0");
  if (m_out == 0) return MPQ_OK;
  ROWS_CHECK(m_out);
  if (!W_host || !idx_host) return fail(MPQ_ERR_INVALID_ARG, "W and idx are required");
  if (T_vamp < 0 || cd_sweeps < 0 || cd_sweeps > MAX_SWEEPS)
    return fail(MPQ_ERR_INVALID_ARG, "bad T_vamp / cd_sweeps");
  if (p->ws_cap > 0) return fail(MPQ_ERR_UNSUPPORTED, "host solve does not batch under a cap");
  DeviceGuard g(p->device);
  cudaStream_t st = (cudaStream_t)stream;
  if (p->ws.rows < m_out) MPQ_TRY(ensure_workspace(p, m_out));
  MPQ_TRY(ensure_host_staging(p, p->ws.rows));
  Workspace& w = p->ws;
  const int64_t n = p->n, B = p->B;
  MPQ_CUDA(cudaMemcpyAsync(w.W, W_host, sizeof(float) * m_out * n, cudaMemcpyHostToDevice, st));
  SolveIO io{w.W, m_out, nullptr, nullptr, T_vamp, cd_sweeps, w.idx_stage,
             w_hat_host ? w.w_hat : nullptr, energy_host ? w.energy : nullptr, nullptr};
  MPQ_TRY(solve_device(p, io, st));
  MPQ_CUDA(cudaMemcpyAsync(idx_host, w.idx_stage, sizeof(uint16_t) * m_out * B, cudaMemcpyDeviceToHost, st));
  if (w_hat_host)
    MPQ_CUDA(cudaMemcpyAsync(w_hat_host, w.w_hat, sizeof(float) * m_out * n, cudaMemcpyDeviceToHost, st));
  if (energy_host)
    MPQ_CUDA(cudaMemcpyAsync(energy_host, w.energy, sizeof(float) * m_out, cudaMemcpyDeviceToHost, st));
  return mpq_plan_status(p, stream);
}

mpq_status mpq_stage_init(mpq_plan_t p, const float* W, int64_t m, int32_t given, float* scale,
                          float* offset, uint16_t* idx_rtn, double* gamma1_0,
                          mpq_stream_t stream) {
  PLAN_CHECK(p);
  if (m < 0 || (m > 0 && (!W || !scale || !offset || !idx_rtn || !gamma1_0)))
    return fail(MPQ_ERR_INVALID_ARG, "init: missing buffer");
  ROWS_CHECK(m);
  DeviceGuard g(p->device);
  return launch_init(p, W, m, given ? 1 : 0, scale, offset, idx_rtn, gamma1_0, (cudaStream_t)stream);
}

mpq_status mpq_stage_denoise(mpq_plan_t p, const float* R1, const double* gamma1,
                             const float* scale, const float* offset, int64_t m, const float* W,
                             const double* gamma1_0, float* xhat1, float* vblock, double* vsum,
                             uint16_t* idx, mpq_stream_t stream) {
  PLAN_CHECK(p);
  if (m < 0 || (m > 0 && (!R1 || !gamma1 || !scale || !offset || !xhat1 || !vsum)))
    return fail(MPQ_ERR_INVALID_ARG, "denoise: missing buffer");
  ROWS_CHECK(m);
  if (isfinite(p->params.tau) && m > 0 && !W)
    return fail(MPQ_ERR_INVALID_ARG, "denoise: an anchored plan needs W");
  DeviceGuard g(p->device);
  cudaStream_t st = (cudaStream_t)stream;
  if (p->d == 8 && vblock == nullptr) {
    MPQ_TRY(ensure_workspace(p, m));
    vblock = p->ws.R2;
  }
  return launch_denoise(p, R1, gamma1, scale, offset, m, W, gamma1_0, xhat1, vblock, vsum, idx, st);
}

mpq_status mpq_stage_linear(mpq_plan_t p, const float* W, int64_t m, const float* R1,
                            const double* gamma1, const float* xhat1, const double* vsum,
                            const double* gamma1_0, double* beta, float* R1_out,
                            double* gamma1_out, float* R2, double* gamma2, float* Uprime,
                            float* xhat2, double* alpha2, double* beta_hat, int32_t* clamps,
                            mpq_stream_t stream) {
  PLAN_CHECK(p);
  if (m < 0 || (m > 0 && (!W || !R1 || !gamma1 || !xhat1 || !vsum || !gamma1_0 || !beta ||
                          !R1_out || !gamma1_out)))
    return fail(MPQ_ERR_INVALID_ARG, "linear: missing buffer");
  ROWS_CHECK(m);
  if (m == 0) return MPQ_OK;
  DeviceGuard g(p->device);
  MPQ_TRY(ensure_workspace(p, m));
  Workspace& w = p->ws;
  cudaStream_t st = (cudaStream_t)stream;
  if (!R2) R2 = w.R2;
  if (!gamma2) gamma2 = w.gamma2;
  return run_linear(p, W, m, R1, gamma1, xhat1, vsum, gamma1_0, beta, R1_out, gamma1_out, R2,
                    gamma2, Uprime, xhat2, alpha2, beta_hat, clamps, st);
}

mpq_status mpq_stage_vamp_scalar(mpq_plan_t p, const float* W, int64_t m, const float* scale,
                                 const float* offset, const float* R1, const double* gamma1,
                                 const double* gamma1_0, double* beta, float* R2, double* gamma2,
                                 float* R1_out, double* gamma1_out, uint16_t* idx_map,
                                 float* R2_next, double* gamma2_next, int32_t* clamps,
                                 mpq_stream_t stream) {
  PLAN_CHECK(p);
  if (m < 0 || (m > 0 && (!W || !scale || !offset || !R1 || !gamma1 || !gamma1_0 || !beta ||
                          !gamma1_out)))
    return fail(MPQ_ERR_INVALID_ARG, "vamp_scalar: missing buffer");
  ROWS_CHECK(m);
  if (p->d != 1 || vamp_row_threads(p->n, p->G) == 0)
    return fail(MPQ_ERR_UNSUPPORTED,
                "vamp_scalar: the fused row kernel runs d = 1 rows that fit its shared memory");
  if (m == 0) return MPQ_OK;
  DeviceGuard g(p->device);
  MPQ_TRY(ensure_workspace(p, m));
  Workspace& w = p->ws;
  cudaStream_t st = (cudaStream_t)stream;
  // the order of one iteration of mpq_solve: fused denoiser + d2l on the
  // injected cavity, the linear module, then the next fused pass (l2d,
  // denoiser, d2l); the MAP pass reads the same G and r2 before that pass
  // overwrites r2
  MPQ_TRY(launch_vamp_row_scalar(p, W, m, 2, 0, R1, w.R2, w.coef, w.kappa, gamma1, scale, offset,
                                 gamma1_0, &w.As, w.gamma2, clamps, nullptr, st));
  if (R2) MPQ_CUDA(cudaMemcpyAsync(R2, w.R2, sizeof(float) * m * p->n, cudaMemcpyDeviceToDevice, st));
  if (gamma2) MPQ_CUDA(cudaMemcpyAsync(gamma2, w.gamma2, sizeof(double) * m, cudaMemcpyDeviceToDevice, st));
  MPQ_TRY(run_linear_core(p, m, w.gamma2, gamma1_0, beta, gamma1_out, nullptr, nullptr, nullptr,
                          clamps, st));
  if (idx_map)
    MPQ_TRY(launch_vamp_row_scalar(p, W, m, 0, 1, w.X1, w.R2, w.coef, w.kappa, gamma1_out, scale,
                                   offset, gamma1_0, nullptr, nullptr, nullptr, idx_map, st));
  if (R1_out || R2_next || gamma2_next) {
    MPQ_TRY(launch_vamp_row_scalar(p, W, m, 0, 0, w.X1, w.R2, w.coef, w.kappa, gamma1_out, scale,
                                   offset, gamma1_0, &w.As, w.gamma2, clamps, nullptr, st, R1_out));
    if (R2_next)
      MPQ_CUDA(cudaMemcpyAsync(R2_next, w.R2, sizeof(float) * m * p->n, cudaMemcpyDeviceToDevice, st));
    if (gamma2_next)
      MPQ_CUDA(cudaMemcpyAsync(gamma2_next, w.gamma2, sizeof(double) * m, cudaMemcpyDeviceToDevice, st));
  }
  return MPQ_OK;
}

mpq_status mpq_stage_cd(mpq_plan_t p, const float* W, int64_t m, const float* scale,
                        const float* offset, uint16_t* idx, int32_t sweeps, int32_t* changes,
                        mpq_stream_t stream) {
  PLAN_CHECK(p);
  if (m < 0 || (m > 0 && (!W || !scale || !offset || !idx)))
    return fail(MPQ_ERR_INVALID_ARG, "cd: missing buffer");
  ROWS_CHECK(m);
  if (sweeps < 0 || sweeps > MAX_SWEEPS) return fail(MPQ_ERR_INVALID_ARG, "sweeps must be in [0, 64]");
  if (m == 0 || sweeps == 0) return MPQ_OK;
  DeviceGuard g(p->device);
  MPQ_TRY(ensure_workspace(p, m));
  if (!changes) changes = p->ws.clamps + p->ws.rows;
  MPQ_TRY(launch_sanitize_idx(p, idx, m * p->B, (cudaStream_t)stream));
  return run_cd(p, W, m, scale, offset, idx, sweeps, changes, (cudaStream_t)stream);
}

mpq_status mpq_stage_energy(mpq_plan_t p, const float* W, int64_t m, const float* scale,
                            const float* offset, const uint16_t* idx, float* w_hat, float* energy,
                            mpq_stream_t stream) {
  PLAN_CHECK(p);
  if (m < 0 || (m > 0 && (!W || !scale || !offset || !idx || !energy)))
    return fail(MPQ_ERR_INVALID_ARG, "energy: missing buffer");
  ROWS_CHECK(m);
  if (m == 0) return MPQ_OK;
  DeviceGuard g(p->device);
  MPQ_TRY(ensure_workspace(p, m));
  // the caller's indices are copied and sanitised before any codebook lookup
  uint16_t* safe = p->ws.idx;
  MPQ_CUDA(cudaMemcpyAsync(safe, idx, sizeof(uint16_t) * m * p->B, cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
  MPQ_TRY(launch_sanitize_idx(p, safe, m * p->B, (cudaStream_t)stream));
  return run_energy(p, W, m, scale, offset, safe, w_hat, energy, (cudaStream_t)stream);
}

mpq_status mpq_profile_start(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof) {
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_prof.clear();
  g_prof_on = true;
  return MPQ_OK;
}

mpq_status mpq_profile_stop(char* buf, int64_t buflen) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = false;
  std::map<std::string, std::pair<int64_t, double>> agg;
  for (auto& r : g_prof) {
    MPQ_CUDA(cudaEventSynchronize(r.b));
    float ms = 0.0f;
    MPQ_CUDA(cudaEventElapsedTime(&ms, r.a, r.b));
    auto& e = agg[r.name];
    e.first += 1;
    e.second += ms;
  }
  std::string out;
  for (auto& kv : agg) {
    char line[256];
    snprintf(line, sizeof(line), "%s %lld %.6f\n", kv.first.c_str(), (long long)kv.second.first,
             kv.second.second);
    out += line;
  }
  if (!buf || (int64_t)out.size() + 1 > buflen) return fail(MPQ_ERR_INVALID_ARG, "profile buffer too small");
  memcpy(buf, out.c_str(), out.size() + 1);
  return MPQ_OK;
}

const char* mpq_last_error(void) { return g_last_error.c_str(); }

int64_t mpq_kernel_launch_count(void) { return g_launches.load(); }

}  // extern "C"
