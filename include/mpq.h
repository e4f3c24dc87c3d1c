/*
 * mpq.h -- C ABI of libmpq, a B200 (sm_100a) implementation of the MPQ
 * row-batched post-training-quantisation solver.
 *
 * Source of every operation: "MPQ: A Message-Passing View of Post-Training
 * Quantization" (papernotes.org NeurIPS 2026 note).  Sections cited below:
 *   [Overall framework]  row objective 1/2 |Xw - X w_hat|^2 over the product
 *                        of block codebooks C_1 x ... x C_B, B = n/d;
 *   [Flowchart]          A = X, y = Xw -> compact SVD (T = Sigma V^T,
 *                        y~ = U^T y) -> T_vamp x (VAMP soft messages, beta
 *                        M-step) -> marginal MAP -> Mahalanobis CD;
 *   [Key design 1]       blockwise denoiser q_b(c) ~ rho_b(c) exp(-gamma1/2
 *                        |c - r1_b|^2), extrinsic updates, Gaussian linear
 *                        module solved in rank space;
 *   [Key design 2]       empirical-Bayes M-step for beta, damped;
 *   [Key design 3]       marginal-MAP argmax and exact block CD in the metric
 *                        G_b = T_b^T T_b;
 *   [Hyper-parameters]   (loss / training strategy section) T_vamp = 16,
 *                        rho_damp = 0.5, tau, S_CD = 3 with early stop,
 *                        gamma1_0 = 1/MSE(w, w_rtn), E8 d = 8, M_b = 2^16;
 *   [Main experiments]   (key experimental data) calibration on 128 C4
 *                        sequences of length 2048;
 *   [Motivation]         (research background) GPTQ, LDLQ and block CD as
 *                        hard-decision solvers;
 *   [Ablation]           (ablation table) T_vamp / CD-sweep settings,
 *                        including the LDLQ and LDLQ + CD3 rows.
 * [ai.info findings] is the ai.info page on the same paper, its list of
 * findings (random Hadamard transforms and E_lin).
 * The min-max scalar grid follows the NeUQI note ("Near-Optimal Uniform
 * Quantization Parameter Initialization for Low-Bit LLMs"), existing pain
 * points section: s = (max - min)/(2^k - 1), z = -round(min/s).
 *
 * Conventions for every entry point:
 *  - Pointers are DEVICE pointers (memory the caller allocated on the
 *    plan's device) unless the argument says HOST.  The caller owns every
 *    buffer it passes and keeps it alive until the stream has finished the
 *    call.  Row-major layouts throughout.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and the call returns without synchronising, except where noted.
 *  - Arguments are validated before anything is launched; a rejected call
 *    launches nothing and returns MPQ_ERR_INVALID_ARG.  Kernels that meet a
 *    non-finite input or hit an iteration cap set a device status word that
 *    mpq_plan_status() reads.  Outputs are defined only when both the call
 *    and the following mpq_plan_status() return MPQ_OK.
 *  - mpq_last_error() gives a thread-local message for the last failure.
 *  - No entry point throws; all are thread-compatible per plan (one thread
 *    at a time per plan).
 */
#ifndef MPQ_H_
#define MPQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MPQ_API __attribute__((visibility("default")))
#else
#define MPQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct mpq_plan_s* mpq_plan_t;
typedef struct mpq_gram_s* mpq_gram_t;
typedef void* mpq_stream_t; /* cudaStream_t */

typedef enum {
  MPQ_OK = 0,
  MPQ_ERR_INVALID_ARG = 1, /* bad size, NULL pointer, unsupported parameter */
  MPQ_ERR_CUDA = 2,        /* a CUDA runtime call failed (message has it)   */
  MPQ_ERR_OOM = 3,         /* device allocation failed / over the cap       */
  MPQ_ERR_NONFINITE = 4,   /* NaN/Inf met in an input on the device         */
  MPQ_ERR_RANK = 5,        /* setup found rank 0                            */
  MPQ_ERR_TIMEOUT = 6,     /* a bounded device loop reached its cap         */
  MPQ_ERR_UNSUPPORTED = 7
} mpq_status;

/* Solver parameters ([Hyper-parameters]).  Fill with mpq_params_default. */
typedef struct {
  int32_t d;              /* block size: 1 (scalar grid) or 8 (vector codebook) */
  int32_t K;              /* d = 1: grid levels L, 2..256; d = 8: codebook size 1..65536 */
  const float* codebook;  /* d = 8: HOST pointer, K x 8 row-major, copied at plan
                             creation; d = 1: must be NULL (levels are 0..L-1,
                             mapped per row by scale * k + offset) */
  double beta0;           /* initial inverse temperature, default 1 */
  double damping;         /* rho_damp: beta <- (1-rho) beta + rho beta_hat, default 0.5 */
  double tau;             /* prior anchor scale ([Hyper-parameters]: tau = 0.2,
                             the default; [Key design 1]: the denoiser works "under
                             the prior anchor").  The anchor pins each block to its
                             own weights w_b with a width of tau codebook units
                             (grid steps for d = 1, lattice units for d = 8):
                             rho_b(c) = exp(-|c - w_b|^2 / (2 tau^2 scale^2)) with c
                             in weight units and scale the row's (or group's)
                             scale.  INFINITY = uniform rho_b, the unanchored
                             limit of the pages' analysis. */
  double gamma_lo_rel;    /* extrinsic precisions are clipped into        */
  double gamma_hi_rel;    /*   [lo, hi] * gamma1_0 (defaults 1e-10, 1e10) */
  double alpha_min;       /* mean divergences are clipped into            */
  double alpha_max;       /*   [alpha_min, alpha_max] (1e-10, 0.99)       */
  int32_t vec_engine;     /* d = 8 denoiser: 0 (default) tensor cores when the
                             codebook qualifies, else SIMT; 1 SIMT always;
                             2 tensor cores (plan creation fails with
                             MPQ_ERR_UNSUPPORTED when the codebook does not
                             qualify).  Qualifies: K a multiple of 128, all
                             coordinates integer multiples of 2^-e (e <= 8)
                             with |c_i| 2^e <= 127, and |c|^2 < 2^14, so that
                             fp16 holds them and the distance terms of the
                             scores are exact in fp32 (lattice codebooks such
                             as the offset E8 set).  Ignored for d = 1. */
  int32_t cd_panel;       /* block CD visits the columns in panels: a change
                             updates the gradient of its own panel at once and
                             of all other columns when the panel ends (same
                             result, less memory traffic).  0 (default):
                             automatic, the widest multiple of 128 columns
                             whose slice of the gradient (rows x panel x 4
                             bytes) fits in 32 MiB, at least 512; else the
                             panel width in columns, a positive multiple of
                             128 (a panel as wide as n is one panel). */
  int32_t group_size;     /* d = 1: 0 (default) one min-max grid per row; G > 0
                             (a multiple of 128 dividing n) one grid per group
                             of G consecutive columns of a row, the pages'
                             group-wise setting ("group 128").  Then every
                             scale/offset array of the API (row_scale,
                             row_offset, the stage hooks' scale/offset) holds
                             m x n/G values, row-major.  Must be 0 for d = 8. */
  int32_t solve_graphs;   /* 1 (default): when mpq_solve or mpq_solve_host is
                             called a second time with the same buffers, sizes
                             and options (the buffers' contents may change), it
                             captures its kernel launches into a CUDA graph, and
                             later such calls replay it, which removes most
                             inter-launch gaps; 4 calls are remembered per plan.
                             0: every call launches its kernels directly.  Calls
                             made while the per-kernel profiler runs always
                             launch directly. */
  double cd_skip_precision;  /* adaptive CD: 0 (default) every row runs CD; > 0:
                             in mpq_solve / mpq_solve_host, rows whose terminal
                             VAMP precision gamma1 s^2 exceeds this (s the row's
                             scale, its largest group scale with group-wise
                             grids) skip CD and keep the marginal MAP; their
                             cd_changes are 0.  The stage hook mpq_stage_cd
                             always runs CD. */
  int32_t greedy_init;    /* the greedy baseline ([Motivation]: GPTQ / LDLQ
                             commit each block to one codeword and pass its
                             error on; [Ablation] rows "LDLQ" and "LDLQ +
                             CD3").  0 (default): a solve with T_vamp = 0
                             starts CD from round-to-nearest.  1: it starts
                             from LDLQ instead -- blocks in order, each
                             committed to its nearest level (d = 1) or
                             nearest codeword in the Euclidean metric
                             (d = 8), its error fed to the later columns
                             through the Cholesky factor of
                             (H + lambda I)^-1, built at plan creation (fp64
                             on the device; n x n fp32 and fp16 copies kept).
                             T_vamp > 0 is unaffected. */
  double greedy_damp;     /* lambda = greedy_damp * mean(diag H), default 0.01;
                             0 needs a full-rank H (else plan creation fails
                             with MPQ_ERR_RANK). */
} mpq_params;

/* Fill `p` with the defaults above for block size d and codebook size K. */
MPQ_API void mpq_params_default(mpq_params* p, int32_t d, int32_t K);

/* ---------------------------------------------------------------- plans --- */

/* Create a plan from a precomputed spectrum ([Flowchart]: T = diag(s) V^T).
 *   s: r doubles, descending, > 0.   V: n x r doubles, orthonormal columns.
 *   n must be a multiple of params->d; 1 <= r <= n.
 * The plan copies s and V (fp32 + fp64 copies, both layouts), builds
 * H = V diag(s^2) V^T and, for d = 8, the per-block tables 1/2 c^T H_bb c.
 * Synchronises `stream` before returning. */
MPQ_API mpq_status mpq_plan_create_from_spectrum(const double* s, const double* V, int64_t n, int64_t r,
                                         const mpq_params* params, mpq_stream_t stream,
                                         mpq_plan_t* plan);

/* Create a plan from calibration activations X (m x n fp32, device):
 * the compact SVD of X through the smaller Gram matrix (X^T X if n <= m,
 * else X X^T), computed on the device in fp64 by cyclic Jacobi; rank cut at
 * lambda > lambda_max * max(m, n) * 2^-52 ([Key design 1]: T in the rank
 * space r = rank(X)).  Synchronises `stream`.  MPQ_ERR_RANK if X == 0. */
MPQ_API mpq_status mpq_plan_create_from_x(const float* X, int64_t m, int64_t n, const mpq_params* params,
                                  mpq_stream_t stream, mpq_plan_t* plan);

/* ------------------------------------------------ streamed calibration --- */
/* Calibration at scale ([Main experiments]: 128 sequences x 2048 tokens, so
 * m = 262144 activation rows) does not fit one X matrix: stream it.  A gram
 * handle owns G = sum_c X_c^T X_c (n x n, fp64, device); each chunk X_c
 * (rows x n fp32, device, row-major) adds its products in fp64.  The plan
 * built from it has the spectrum of X = [X_1; X_2; ...] through the right
 * Gram (Jacobi eigenpairs of G, s = sqrt(lambda), V = eigenvectors) and the
 * same rank cut as mpq_plan_create_from_x with m = the total row count.
 *   create:     n in [1, 131072]; G = 0.  Synchronises `stream`.
 *   accumulate: rows >= 0 (0 is a no-op); X is read, never kept; the call
 *               synchronises `stream` before returning (it frees a fp64
 *               rows x n staging copy).  Chunks may differ in row count.
 *   info:       HOST outputs (either may be NULL): n and the rows so far.
 *   get:        copy G out (device, n x n doubles, row-major).
 *   create_from_gram: MPQ_ERR_RANK with no rows or G == 0; the gram stays
 *               owned by the caller and may keep accumulating.
 *   destroy:    NULL is a no-op. */
MPQ_API mpq_status mpq_gram_create(int64_t n, mpq_stream_t stream, mpq_gram_t* gram);
MPQ_API mpq_status mpq_gram_accumulate(mpq_gram_t gram, const float* X, int64_t rows, mpq_stream_t stream);
MPQ_API mpq_status mpq_gram_info(mpq_gram_t gram, int64_t* n, int64_t* rows);
MPQ_API mpq_status mpq_gram_get(mpq_gram_t gram, double* G, mpq_stream_t stream);
MPQ_API mpq_status mpq_gram_destroy(mpq_gram_t gram);
MPQ_API mpq_status mpq_plan_create_from_gram(mpq_gram_t gram, const mpq_params* params,
                                             mpq_stream_t stream, mpq_plan_t* plan);

/* Random Hadamard rotation, in place, on the device (incoherence
 * preprocessing; [ai.info findings]: the rotation leaves E_lin unchanged, as
 * E_lin sees the Hessian only through its eigenvalues).  Every row x of X
 * (rows x n fp32, row-major, device) becomes x Q^T, Q = H_n diag(signs) /
 * sqrt(n) with H_n the Sylvester-Hadamard matrix; apply it to both W and X
 * and the objective ||(W - W_hat) X^T||^2 is unchanged.  signs: n floats,
 * each +1 or -1 (device).  n a power of two in [1, MPQ_RHT_MAX_N].  Any
 * alignment is accepted; with X and signs 16-byte aligned and 512 <= n <=
 * 8192 the rotation takes four butterfly stages per pass in registers, else
 * one shared-memory pass per stage, with the same result bits either way.
 * Asynchronous on `stream`. */
#define MPQ_RHT_MAX_N 32768
MPQ_API mpq_status mpq_rht(float* X, int64_t rows, int64_t n, const float* signs, mpq_stream_t stream);

/* Release every device buffer the plan owns.  NULL is a no-op. */
MPQ_API mpq_status mpq_plan_destroy(mpq_plan_t plan);

/* HOST outputs (any may be NULL): n, rank r, d, K. */
MPQ_API mpq_status mpq_plan_info(mpq_plan_t plan, int64_t* n, int64_t* r, int32_t* d, int32_t* K);

/* Copy the plan's spectrum out: s (r doubles) and V (n x r doubles), device. */
MPQ_API mpq_status mpq_plan_get_spectrum(mpq_plan_t plan, double* s, double* V, mpq_stream_t stream);

/* Synchronise `stream`, read and clear the plan's device status word.
 * Returns MPQ_OK, MPQ_ERR_NONFINITE or MPQ_ERR_TIMEOUT. */
MPQ_API mpq_status mpq_plan_status(mpq_plan_t plan, mpq_stream_t stream);

/* Upper bound on the workspace (bytes) that a solve of m_out rows allocates
 * inside the plan, and an optional cap: a solve that would need more than
 * `cap_bytes` fails with MPQ_ERR_OOM before launching (0 = no cap). */
MPQ_API int64_t mpq_plan_workspace_bytes(mpq_plan_t plan, int64_t m_out);
MPQ_API mpq_status mpq_plan_set_workspace_cap(mpq_plan_t plan, int64_t cap_bytes);

/* --------------------------------------------------------------- solve --- */

/* Optional per-row outputs of a solve (device pointers, each may be NULL). */
typedef struct {
  double* gamma1;     /* m_out: terminal denoiser precision gamma1^T          */
  double* beta;       /* m_out: terminal inverse temperature                  */
  int32_t* clamps;    /* m_out: number of clips applied over the VAMP loop    */
  int32_t* cd_changes;/* m_out x cd_sweeps: blocks changed in each CD sweep   */
} mpq_row_stats;

/* The whole MPQ solve of every row of W ([Flowchart]):
 * init (per-row scale/offset, round-to-nearest, gamma1_0 = 1/MSE, r1 = w,
 * beta = beta0) -> T_vamp iterations of {denoiser, extrinsic update, rank-
 * space linear module, beta M-step} -> marginal-MAP argmax -> at most
 * cd_sweeps sweeps of exact block CD (stop after a sweep without change)
 * -> w_hat and energies E = 1/2 |T (w - w_hat)|^2.
 *   W: m_out x n fp32.
 *   row_scale/row_offset: m_out floats each, or both NULL for the built-in
 *     choice (d = 1: per-row min-max grid; d = 8: scale = RMS(w), offset 0).
 *   T_vamp >= 0, 0 <= cd_sweeps <= 64.
 *   idx: m_out x B uint16 codeword indices (out).  w_hat: m_out x n fp32
 *   (out, may be NULL).  energy: m_out fp32 (out, may be NULL).
 *   stats: HOST struct of optional device outputs, may be NULL.
 * Asynchronous; may allocate plan workspace on first use for a row count
 * (which synchronises the device). */
MPQ_API mpq_status mpq_solve(mpq_plan_t plan, const float* W, int64_t m_out, const float* row_scale,
                     const float* row_offset, int32_t T_vamp, int32_t cd_sweeps, uint16_t* idx,
                     float* w_hat, float* energy, const mpq_row_stats* stats,
                     mpq_stream_t stream);

/* Same as mpq_solve with HOST buffers for W, idx, w_hat and energy (pinned
 * memory gives the fastest copies).  Copies W to plan-owned device memory,
 * solves, copies the results back, synchronises `stream` and returns the
 * device status (as mpq_plan_status). */
MPQ_API mpq_status mpq_solve_host(mpq_plan_t plan, const float* W_host, int64_t m_out, int32_t T_vamp,
                          int32_t cd_sweeps, uint16_t* idx_host, float* w_hat_host,
                          float* energy_host, mpq_stream_t stream);

/* -------------------------------------------------- stage entry points --- */
/* Each runs one stage on state the caller injects, so that every stage can
 * be compared on identical inputs.  B = n/d.  Per-row scalars are fp64,
 * vectors fp32.  The init, CD and energy hooks, the linear hook and (for
 * d = 8, and for d = 1 rows too wide for the fused kernel) the denoiser hook
 * run the kernels mpq_solve runs.  mpq_solve runs the denoiser and the
 * extrinsic updates of d = 1 rows that fit in shared memory in one fused row
 * kernel; mpq_stage_denoise and mpq_stage_linear run the separate kernels
 * for them (same arithmetic, shared device functions), and
 * mpq_stage_vamp_scalar runs the fused kernel itself. */

/* Init ([Hyper-parameters]): if `given` == 0, compute scale/offset (built-in
 * rule) into scale/offset; else read them.  idx_rtn: m x B nearest codeword
 * (lowest index on ties); gamma1_0: m doubles, 1/max(MSE(w, w_rtn), 1e-30). */
MPQ_API mpq_status mpq_stage_init(mpq_plan_t plan, const float* W, int64_t m, int32_t given, float* scale,
                          float* offset, uint16_t* idx_rtn, double* gamma1_0, mpq_stream_t stream);

/* Denoiser ([Key design 1]): for every block the posterior over the row's
 * codewords scale*c + offset.  Inputs R1 (m x n), gamma1 (m), scale/offset
 * (m); for a finite-tau plan also W (m x n), the anchor's centre, else NULL.
 * (gamma1_0 is not read by the denoiser and may be NULL.)
 * Outputs xhat1 (m x n posterior means), vblock (m x B traces of the
 * posterior covariances, may be NULL), vsum (m, fp64 sums of vblock),
 * idx (m x B argmax, lowest index on ties, may be NULL). */
MPQ_API mpq_status mpq_stage_denoise(mpq_plan_t plan, const float* R1, const double* gamma1,
                             const float* scale, const float* offset, int64_t m, const float* W,
                             const double* gamma1_0, float* xhat1, float* vblock, double* vsum,
                             uint16_t* idx, mpq_stream_t stream);

/* Extrinsic update, linear module and M-step ([Key design 1], [Key design
 * 2]).  Inputs W, R1, xhat1 (m x n), gamma1, vsum, gamma1_0 (m); beta (m)
 * is read and overwritten with the damped update.  Outputs R1_out (m x n),
 * gamma1_out (m).  Diagnostics (each may be NULL): R2 (m x n), gamma2 (m),
 * Uprime (m x r, D*u), xhat2 (m x n), alpha2 (m, before clipping),
 * beta_hat (m), clamps (m, added to). */
MPQ_API mpq_status mpq_stage_linear(mpq_plan_t plan, const float* W, int64_t m, const float* R1,
                            const double* gamma1, const float* xhat1, const double* vsum,
                            const double* gamma1_0, double* beta, float* R1_out,
                            double* gamma1_out, float* R2, double* gamma2, float* Uprime,
                            float* xhat2, double* alpha2, double* beta_hat, int32_t* clamps,
                            mpq_stream_t stream);

/* One VAMP iteration of scalar (d = 1) rows as mpq_solve runs it, on an
 * injected cavity ([Key design 1] denoiser and extrinsic updates, [Key
 * design 2] M-step).  mpq_solve runs these rows through one fused row kernel
 * per iteration, which forms the cavity r1 from the linear module's output
 * (extrinsic update linear -> denoiser), runs the denoiser and the extrinsic
 * update denoiser -> linear; this hook runs that same kernel:
 *   1. fused pass on the cavity (R1, gamma1): denoiser, then r2 and gamma2;
 *   2. the linear module and beta M-step (as mpq_stage_linear): beta is read
 *      and overwritten with the damped update, gamma1_out receives gamma1';
 *   3. if idx_map: the fused MAP pass on the next cavity r1' (argmax);
 *   4. if R1_out, R2_next or gamma2_next: the next fused pass, which forms
 *      r1' (written to R1_out) and runs the denoiser and the d2l step on it
 *      (r2' to R2_next, gamma2' to gamma2_next).
 *   W, R1: m x n; scale/offset: as mpq_stage_denoise; gamma1, gamma1_0, beta:
 *   m doubles.  Outputs R2, R1_out, R2_next (m x n floats), gamma2,
 *   gamma2_next (m doubles), idx_map (m x n) may each be NULL; clamps (m
 *   ints, added to) may be NULL.  A finite-tau plan anchors the denoiser at W.
 * MPQ_ERR_UNSUPPORTED unless d = 1 and a row fits the fused kernel's shared
 * memory (8 bytes per weight; the same rows mpq_solve runs fused). */
MPQ_API mpq_status mpq_stage_vamp_scalar(mpq_plan_t plan, const float* W, int64_t m,
                                         const float* scale, const float* offset, const float* R1,
                                         const double* gamma1, const double* gamma1_0,
                                         double* beta, float* R2, double* gamma2, float* R1_out,
                                         double* gamma1_out, uint16_t* idx_map, float* R2_next,
                                         double* gamma2_next, int32_t* clamps,
                                         mpq_stream_t stream);

/* Exact block CD ([Key design 3]) from the codewords in idx (m x B, read
 * and overwritten): h = H (w - x), then at most `sweeps` sweeps over the
 * blocks in order; each block takes the codeword of least energy (lowest
 * index on ties) when that lowers the energy; a row stops after a sweep
 * without change.  changes: m x sweeps ints (may be NULL). */
MPQ_API mpq_status mpq_stage_cd(mpq_plan_t plan, const float* W, int64_t m, const float* scale,
                        const float* offset, uint16_t* idx, int32_t sweeps, int32_t* changes,
                        mpq_stream_t stream);

/* Output ([Overall framework]): w_hat = scale * C[idx] + offset (m x n, may
 * be NULL) and E = 1/2 |diag(s) V^T (w - w_hat)|^2 (m floats). */
MPQ_API mpq_status mpq_stage_energy(mpq_plan_t plan, const float* W, int64_t m, const float* scale,
                            const float* offset, const uint16_t* idx, float* w_hat, float* energy,
                            mpq_stream_t stream);

/* Allocation-free variant of mpq_stage_energy (the paper has no counterpart;
 * this exists for integration).  Some callers cannot let a library allocate
 * device memory: a framework whose allocator owns all of the GPU's memory, a
 * serving loop that must never stall on the device-wide synchronisation an
 * allocation or free can cause, or a process whose memory budget is fixed at
 * start-up.  This entry point uses no plan workspace and calls no allocator:
 * its intermediates (the residual w - w_hat, its projection V^T (w - w_hat)
 * and a sanitised copy of idx) live in one static device array of
 * MPQ_NOALLOC_SCRATCH_BYTES bytes that every GPU loading the library holds
 * until the process exits.
 *   Same arguments, layouts and results as mpq_stage_energy.
 *   Limit: m * (4 n + 4 r + 2 B) bytes (each part rounded up to 256) must
 *   fit in MPQ_NOALLOC_SCRATCH_BYTES; larger calls return
 *   MPQ_ERR_INVALID_ARG without launching -- split the rows.
 *   The plan's device must be current.  The first call on a device looks
 *   up the array's device address (cudaGetSymbolAddress) and caches it;
 *   make that first call before any stream capture.
 *   All calls on a device share the one array and it keeps the last call's
 *   contents; two calls whose work overlaps on the GPU (different streams,
 *   no ordering between them) race on it, so order them on one stream. */
#define MPQ_NOALLOC_SCRATCH_BYTES (16u << 20)
MPQ_API mpq_status mpq_stage_energy_noalloc(mpq_plan_t plan, const float* W, int64_t m,
                                            const float* scale, const float* offset,
                                            const uint16_t* idx, float* w_hat, float* energy,
                                            mpq_stream_t stream);

/* ----------------------------------------------------------- profiling --- */
/* Per-kernel timing with CUDA events recorded on the launching stream around
 * every kernel the library launches while profiling is on.  start clears
 * earlier records; stop synchronises on the recorded events and writes one
 * line per kernel name into the HOST buffer `buf` (NUL-terminated):
 *   "<name> <launches> <total milliseconds>\n"
 * Returns MPQ_ERR_INVALID_ARG if the text does not fit in `buflen`. */
MPQ_API mpq_status mpq_profile_start(void);
MPQ_API mpq_status mpq_profile_stop(char* buf, int64_t buflen);

/* Thread-local text of the last error (never NULL). */
MPQ_API const char* mpq_last_error(void);

/* Number of kernels this library has launched in the calling process. */
MPQ_API int64_t mpq_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* MPQ_H_ */
