// Tensor-core blockwise denoiser for vector codebooks (d = 8).
//
// For every block b of 8 weights the denoiser needs the posterior
// q_b(c) ~ exp(-g/2 |c - t_b|^2) over all K codewords (the blockwise
// denoiser of the MPQ page, section "VAMP in rank space"; g = gamma1 s^2 and
// t = r1 / s in codebook units), its mean, its total variance and its argmax.
// The brute-force cost is K exponentials per block; everything else runs on
// the tensor cores:
//
//   pass 1  s(c) = t.c - |c|^2/2 in fp32                     -> argmax c*
//   pass 2  logit(c) - logit(c*) = g [ (t - c*).(c - c*) - |c - c*|^2/2 ]
//           q(c) = 2^(log2e logit + 8),  S0 = sum q,  S1 = sum q c  (c != c*)
//
// Logits.  t - c* = q + r with q on the grid 2^-F (exact in fp16) and a small
// remainder r (|r| <= 2^-(F+1), scaled up on the way in so that its fp16 pair
// stays clear of subnormals).  Three accumulators, each one MMA (K = 16) over
// the codebook operand [c | |c|^2 (fp16 pair), 1, 1]:
//
//   Q(c) = q.c - q.c*                 exact (integers in units 2^-(F+e))
//   X(c) = c*.c - |c|^2/2 - |c*|^2/2  = -|c - c*|^2/2, exact
//   R(c) = r.c - r.c*                 small; the only rounded one
//
// The per-row constants q.c*, |c*|^2/2 and r.c* ride in the spare K columns
// against the 1s of the codebook operand.  This needs a codebook whose
// coordinates are multiples of 2^-e with |c_i| 2^e <= 127 (lattice codebooks
// such as the offset E8 set).  Q + X is then exact and the logit carries
// rounding only from R, 2^-(F+1) smaller than t - c*.
//
// Moments.  The weights (c* excluded: its weight 2^8 is added back at the
// end, which leaves the first moment centred on c* without cancellation) go
// to shared memory as fp16 hi/lo pairs and one more MMA (N = 16) against the
// transposed codebook [c_0 .. c_7, 1] accumulates S1 and S0 in TMEM over a
// chunk of MOM_CHUNK codebook tiles (two accumulators take turns); the
// epilogue adds the chunks' partial sums in fp32, so that no accumulator
// sums more than a chunk's worth of MMAs (a broad posterior over the whole
// 65536-word codebook would otherwise lose ~1e-4 to accumulation in one
// fp32 register); only S2 = sum q X (the centred second moment, -1/2
// |c - c*|^2 per codeword) and the exponential stay on the ALU.  A weight
// more than 2^8 times c*'s (the argmax pass's fp32 scores misjudged a
// near-tie at an enormous g) would overflow the fp16 weights: that block
// falls back to the point mass on c*.
//
// Pipeline.  One tile is 128 blocks x 128 codewords.  The block operands are
// written by the epilogue threads into shared memory in the no-swizzle
// K-major layout; the codebook operands (8 KiB per 128 codewords: scores
// and transposed) are prepared at plan time in the same layout and streamed
// by bulk copies through a 6-stage ring.  Pass 1 is two MMAs (N = 128, t as
// an fp16 hi/lo pair); pass 2 is, per half of 64 codewords, four score MMAs
// (N = 64, three accumulators) and eight moment MMAs (N = 16, K = 64 as hi
// and lo).  TMEM holds two score buffers so that the MMAs of the next half
// overlap the exponentials of this one, plus the moment accumulator.  The
// kernel is persistent: one CTA per SM walks the 128-block tiles.  Warps 0-15
// are the epilogue (warp w reads TMEM lanes 32 (w % 4) .. +31; warpgroup
// w / 4 takes one quarter of the columns of each MMA), warp 16 owns TMEM and
// issues the MMAs, warp 17 issues the loads.
#include <cuda.h>
#include <cuda_fp16.h>

#include <cmath>
#include <vector>

#include "f32x2.cuh"
#include "mpq_internal.cuh"
#include "tc_ptx.cuh"

namespace mpq {
namespace {
using namespace tcx;

constexpr int DT_M = 128;                  // blocks per tile (MMA M)
constexpr int DT_N = 128;                  // codewords per tile (pass 1 MMA N)
constexpr int DT_N2 = 64;                  // pass 2 score MMA N (two halves per tile)
constexpr int DT_STAGES = 6;
constexpr int DT_EPI_WARPS = 16;
constexpr int DT_WGS = DT_EPI_WARPS / 4;   // column quarters
constexpr int DT_THREADS = (DT_EPI_WARPS + 2) * 32;
constexpr int MMA_WARP = DT_EPI_WARPS, LOAD_WARP = DT_EPI_WARPS + 1;
constexpr int OPER_BYTES = 128 * 32;       // 128 rows x 16 fp16
constexpr int CBT_BYTES = 16 * 128 * 2;    // transposed codebook tile: 16 x 128 fp16
constexpr int STAGE_BYTES = OPER_BYTES + CBT_BYTES;
constexpr int QW_BYTES = 128 * 64 * 2;     // weights of one half: 128 x 64 fp16
// TMEM: pass 1 cycles through 4 score buffers of 128 columns; pass 2 through
// 2 buffers of 192 (Q | X | R, 64 each) and keeps the moments at 384.  The
// passes reuse the same columns: every pass starts after the epilogue has
// read all of the previous one.
constexpr uint32_t DT_TMEM_COLS = 512;
constexpr int T1_BUFS = 4, T2_BUFS = 2;
// weight tiles in shared memory: more than the TMEM score buffers, so that
// the epilogue can run ahead of the moment MMAs that still read older halves
constexpr int QW_BUFS = 4;
constexpr uint32_t T1_COLS = 128, T2_COLS = 192, TM_MOM = 384;  // moments: 2 x 16 columns
constexpr int MOM_CHUNK = 16;              // codebook tiles per moment accumulator
constexpr uint32_t IDESC_P1 = idesc_f16(DT_M, DT_N);
constexpr uint32_t IDESC_P2 = idesc_f16(DT_M, DT_N2);
constexpr uint32_t IDESC_MOM = idesc_f16(DT_M, 16);
constexpr float Q_SHIFT = 8.0f;            // weights carry 2^8: c*'s is 256

// shared-memory map (offsets from the 1024-aligned base)
constexpr int N_ATILES = 6;
constexpr int SM_A = 0;                                   // block operand tiles
constexpr int SM_B = SM_A + N_ATILES * OPER_BYTES;        // stage ring
constexpr int SM_QW = SM_B + DT_STAGES * STAGE_BYTES;     // QW_BUFS x (hi | lo) weights
constexpr int SM_T = SM_QW + QW_BUFS * 2 * QW_BYTES;      // t per row (fp64, 128 x 8)
constexpr int SM_ROW = SM_T + DT_M * 8 * 8;               // per-row data
constexpr int SM_BAR = SM_ROW + (3 + 2 * DT_WGS + DT_WGS) * DT_M * 4;
constexpr int N_BARS = 2 * DT_STAGES + 2 * T1_BUFS + 2 * T2_BUFS + 1 + 2 * QW_BUFS + 4;
constexpr int SM_END = SM_BAR + N_BARS * 8 + 16;
constexpr int DT_SMEM_BYTES = 220 * 1024;  // > half of the SM: one CTA (and TMEM owner) per SM
static_assert(SM_END + 1024 <= DT_SMEM_BYTES, "denoiser shared memory");

enum { A1_HI = 0, A1_LO = 1, A2_Q = 2, A2_X = 3, A2_RH = 4, A2_RL = 5 };

struct DenoiseTcArgs {
  const float* R1;        // m x n (blocks of 8 contiguous)
  const double* gamma1;   // per row
  const float* scale;
  const float* offset;
  const float* W;         // anchor (nullable)
  const double* gamma1_0;
  double inv_tau2;
  int64_t nblocks;        // m * B
  int64_t B;              // blocks per row
  int NT;                 // codeword tiles (K / 128)
  int F, Fmin;            // grid bits of the exact part q of t - c* (finest, coarsest)
  int rk;                 // r enters the MMA as r 2^(Fb + 1 + rk)
  const uint8_t* cb_tc;   // NT x STAGE_BYTES operand images
  const float* cb;        // K x 8 fp32
  float* xhat;
  float* vblock;
  uint16_t* idx;
  int mode;  // 0: both passes; 1: nearest codeword to r1 / s (pass 1, no prior); 2: the
             // posterior's argmax only (pass 1 on the cavity / anchor mean): the marginal MAP
  int* status;
};

// Byte offset of element (row r, k) of a no-swizzle K-major fp16 tile whose
// 8-row groups are `sbo` bytes apart: 8 x 16 B core matrices, consecutive K
// chunks of 8 elements 128 B apart (the descriptor's LBO).
__host__ __device__ __forceinline__ int kmaj_off(int r, int k, int sbo) {
  return (r & 7) * 16 + (r >> 3) * sbo + (k >> 3) * 128 + (k & 7) * 2;
}

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(128 >> 4) << 16;   // LBO: next K chunk
  d |= (uint64_t)(sbo >> 4) << 32;   // SBO: next 8-row group
  d |= (uint64_t)1 << 46;            // descriptor version
  return d;                          // layout type 0: no swizzle
}

__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void named_sync_epi() {
  asm volatile("bar.sync 1, %0;" ::"n"(DT_EPI_WARPS * 32) : "memory");
}

// Bounded wait that also gives up when another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag, int* status) {
  for (uint32_t i = 0; i < WAIT_SPIN; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  for (uint32_t i = 0; i < WAIT_TRIES; ++i) {
    if (mbar_try_wait_sleep(bar, parity, WAIT_SLICE_NS)) return true;
    if (*abort_flag) return false;
  }
  atomicOr(status, STATUS_TIMEOUT);
  *abort_flag = 1;
  return false;
}

// Warp-uniform bounded wait (every lane polls; all must see the phase).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* status) {
  return __all_sync(0xffffffffu, wait_or_abort(bar, parity, abort_flag, status));
}

// fp16 pair of x (|x| clamped to 2^14, NaN kept): x ~ hi + lo with ~22
// significand bits
__device__ __forceinline__ void split16(double x, __half& hi, __half& lo) {
  if (fabs(x) > 16384.0) x = copysign(16384.0, x);
  hi = __double2half(x);
  lo = __double2half(x - (double)__half2float(hi));
}

// one 16-element row of a 128 x 16 block operand tile
__device__ __forceinline__ void store_row(uint8_t* tile, int r, const __half (&v)[16]) {
  uint4 c0, c1;
  __half* p0 = reinterpret_cast<__half*>(&c0);
  __half* p1 = reinterpret_cast<__half*>(&c1);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    p0[i] = v[i];
    p1[i] = v[8 + i];
  }
  *reinterpret_cast<uint4*>(tile + kmaj_off(r, 0, 256)) = c0;
  *reinterpret_cast<uint4*>(tile + kmaj_off(r, 8, 256)) = c1;
}

// 18 warps: five share an SM sub-partition's 16K registers, so at most 96 each
__global__ void __launch_bounds__(DT_THREADS, 1) k_denoise_vec_tc(DenoiseTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* At = smem + SM_A;
  double* sm_t = reinterpret_cast<double*>(smem + SM_T);        // [128][8]
  float* sm_g2 = reinterpret_cast<float*>(smem + SM_ROW);
  float* sm_rs = sm_g2 + DT_M;
  float* sm_g = sm_rs + DT_M;
  float* sm_bval = sm_g + DT_M;                                   // [DT_WGS][128]
  int* sm_bidx = reinterpret_cast<int*>(sm_bval + DT_WGS * DT_M);  // [DT_WGS][128]
  float* sm_s2 = reinterpret_cast<float*>(sm_bidx + DT_WGS * DT_M);  // [DT_WGS][128]
  uint64_t* b_full = reinterpret_cast<uint64_t*>(smem + SM_BAR);
  uint64_t* b_empty = b_full + DT_STAGES;
  uint64_t* t1_full = b_empty + DT_STAGES;
  uint64_t* t1_empty = t1_full + T1_BUFS;
  uint64_t* t2_full = t1_empty + T1_BUFS;
  uint64_t* t2_empty = t2_full + T2_BUFS;
  uint64_t* a_full = t2_empty + T2_BUFS;
  uint64_t* q_full = a_full + 1;
  uint64_t* q_free = q_full + QW_BUFS;
  uint64_t* mom_full = q_free + QW_BUFS;  // [2]: a chunk's moment MMAs are done
  uint64_t* mom_free = mom_full + 2;      // [2]: the epilogue has read that accumulator
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mom_free + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t mtiles = (a.nblocks + DT_M - 1) / DT_M;
  const int passes = a.mode ? 1 : 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < DT_STAGES; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int b = 0; b < T1_BUFS; ++b) {
      mbar_init(&t1_full[b], 1);
      mbar_init(&t1_empty[b], DT_EPI_WARPS);
    }
    for (int b = 0; b < T2_BUFS; ++b) {
      mbar_init(&t2_full[b], 1);
      mbar_init(&t2_empty[b], DT_EPI_WARPS / 2);  // the group of eight warps that owns it
    }
    for (int b = 0; b < QW_BUFS; ++b) {
      mbar_init(&q_full[b], DT_EPI_WARPS / 2);
      mbar_init(&q_free[b], 1);
    }
    mbar_init(a_full, DT_M);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&mom_full[b], 1);
      mbar_init(&mom_free[b], 4);  // the four warps of warpgroup 0
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == MMA_WARP) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(DT_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Counters every role keeps in step: `seq` codebook tiles (stage ring),
  // `tu1` pass-1 tiles (4 TMEM buffers), `hq` pass-2 halves (2 TMEM buffers
  // and 2 weights buffers), `mt_n` block tiles done (moment phases).
  if (warp == LOAD_WARP) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      uint32_t seq = 0;
      bool ok = true;
      for (int64_t mt = blockIdx.x; mt < mtiles && ok; mt += gridDim.x)
        for (int pass = 0; pass < passes && ok; ++pass)
          for (int j = 0; j < a.NT; ++j, ++seq) {
            const int s = seq % DT_STAGES;
            const uint32_t use = seq / DT_STAGES;
            if (seq >= DT_STAGES && !wait_or_abort(&b_empty[s], (use - 1) & 1, abort_flag, a.status)) {
              ok = false;
              break;
            }
            const uint32_t bytes = pass ? STAGE_BYTES : OPER_BYTES;
            mbar_expect_tx(&b_full[s], bytes);
            bulk_load_1d(smem + SM_B + s * STAGE_BYTES, a.cb_tc + (size_t)j * STAGE_BYTES, bytes,
                         &b_full[s]);
          }
      // the copies in flight land before the CTA may exit
      const uint32_t last = seq;
      for (uint32_t q = (last > DT_STAGES ? last - DT_STAGES : 0); q < last; ++q) {
        const int s = q % DT_STAGES;
        for (uint32_t i = 0; i < (1u << 25) && !mbar_try_wait(&b_full[s], (q / DT_STAGES) & 1); ++i)
          if (i > 256) __nanosleep(64);
      }
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t seq = 0, tu1 = 0, hq = 0, aphase = 0, cbase = 0;
      bool ok = true;
      const uint32_t nch = (uint32_t)((a.NT + MOM_CHUNK - 1) / MOM_CHUNK);  // chunks per tile
      const uint32_t a_base = smem_u32(At);
      const uint32_t qw_base = smem_u32(smem + SM_QW);
      for (int64_t mt = blockIdx.x; mt < mtiles && ok; mt += gridDim.x) {
        // ------------------------------------------ pass 1: scores
        if (!(ok = wait_or_abort(a_full, aphase++ & 1, abort_flag, a.status))) break;
        tc_fence_after();
        for (int j = 0; j < a.NT; ++j, ++seq, ++tu1) {
          const int s = seq % DT_STAGES, b = tu1 % T1_BUFS;
          if (!(ok = wait_or_abort(&b_full[s], (seq / DT_STAGES) & 1, abort_flag, a.status))) break;
          if (tu1 >= T1_BUFS &&
              !(ok = wait_or_abort(&t1_empty[b], (tu1 / T1_BUFS - 1) & 1, abort_flag, a.status)))
            break;
          tc_fence_after();
          const uint32_t d = tmem + (uint32_t)b * T1_COLS;
          const uint64_t bd = kmajor_desc(smem_u32(smem + SM_B + s * STAGE_BYTES), 256);
          umma_f16(d, kmajor_desc(a_base + A1_HI * OPER_BYTES, 256), bd, IDESC_P1, 0u);
          umma_f16(d, kmajor_desc(a_base + A1_LO * OPER_BYTES, 256), bd, IDESC_P1, 1u);
          umma_commit(&t1_full[b]);
          umma_commit(&b_empty[s]);
        }
        if (!ok || a.mode) continue;
        // ---------------------------------- pass 2: scores and moments
        // A polling scheduler: the score MMAs of a half go out as soon as its
        // TMEM buffer and codebook stage are ready, the moment MMAs of a half
        // as soon as its weights are in shared memory, so neither waits on
        // the other.
        if (!(ok = wait_or_abort(a_full, aphase++ & 1, abort_flag, a.status))) break;
        tc_fence_after();
        const uint32_t total = 2u * (uint32_t)a.NT;
        uint32_t us = 0, um = 0, idle = 0;
        bool staged = false;
        while (um < total) {
          bool prog = false;
          if (us < total) {
            const uint32_t sq = seq + (us >> 1), u = hq + us;
            const int s = sq % DT_STAGES, b = u % T2_BUFS;
            if (!staged) staged = mbar_test_wait(&b_full[s], (sq / DT_STAGES) & 1);
            if (staged && (u < T2_BUFS || mbar_test_wait(&t2_empty[b], (u / T2_BUFS - 1) & 1))) {
              tc_fence_after();
              // codewords 64h .. 64h+63 of the tile: rows from byte 2048 h
              const uint32_t d = tmem + (uint32_t)b * T2_COLS;
              const uint64_t bd = kmajor_desc(smem_u32(smem + SM_B + s * STAGE_BYTES) + (us & 1) * 2048u, 256);
              umma_f16(d, kmajor_desc(a_base + A2_Q * OPER_BYTES, 256), bd, IDESC_P2, 0u);
              umma_f16(d + 64u, kmajor_desc(a_base + A2_X * OPER_BYTES, 256), bd, IDESC_P2, 0u);
              umma_f16(d + 128u, kmajor_desc(a_base + A2_RH * OPER_BYTES, 256), bd, IDESC_P2, 0u);
              umma_f16(d + 128u, kmajor_desc(a_base + A2_RL * OPER_BYTES, 256), bd, IDESC_P2, 1u);
              umma_commit(&t2_full[b]);
              if (++us % 2 == 0) staged = false;
              prog = true;
            }
          }
          if (um < us) {
            const uint32_t u = hq + um, qb = u % QW_BUFS;
            // the chunk of codebook tiles this half belongs to, and its
            // moment accumulator (two take turns; a chunk's first MMA waits
            // until the epilogue has read that accumulator's previous chunk)
            const uint32_t jt = um >> 1, c = cbase + jt / MOM_CHUNK, mb = c & 1;
            const bool cfirst = (um & 1) == 0 && jt % MOM_CHUNK == 0;
            const bool clast = (um & 1) == 1 &&
                               (jt % MOM_CHUNK == MOM_CHUNK - 1 || jt == (uint32_t)a.NT - 1);
            bool ready = mbar_test_wait(&q_full[qb], (u / QW_BUFS) & 1);
            if (ready && cfirst && c >= 2) ready = mbar_test_wait(&mom_free[mb], ((c >> 1) - 1) & 1);
            if (ready) {
              tc_fence_after();
              const int s = (seq + (um >> 1)) % DT_STAGES;
              const uint32_t wq = qw_base + qb * 2u * QW_BYTES;
              const uint32_t bt = smem_u32(smem + SM_B + s * STAGE_BYTES + OPER_BYTES) + (um & 1) * 1024u;
              const uint32_t dm = tmem + TM_MOM + 16u * mb;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {  // weights (hi, lo) x transposed codebook
                const uint64_t bd = kmajor_desc(bt + kk * 256u, 2048);
                umma_f16(dm, kmajor_desc(wq + kk * 256u, 1024), bd, IDESC_MOM,
                         (cfirst && kk == 0) ? 0u : 1u);
                umma_f16(dm, kmajor_desc(wq + QW_BYTES + kk * 256u, 1024), bd, IDESC_MOM, 1u);
              }
              umma_commit(&q_free[qb]);
              if (um & 1) umma_commit(&b_empty[s]);  // both halves of the stage are done
              if (clast) umma_commit(&mom_full[mb]);
              ++um;
              prog = true;
            }
          }
          if (prog) {
            idle = 0;
          } else {
            if (++idle >= (1u << 25)) {
              atomicOr(a.status, STATUS_TIMEOUT);
              *abort_flag = 1;
            }
            if ((idle & 63) == 63 && *abort_flag) break;
            if (idle > 8) __nanosleep(32);
          }
        }
        if (um < total) {
          ok = false;
          break;
        }
        seq += a.NT;
        hq += total;
        cbase += nch;
      }
      // the MMAs in flight finish before TMEM is released
      for (uint32_t q = (tu1 > T1_BUFS ? tu1 - T1_BUFS : 0); q < tu1; ++q)
        for (uint32_t i = 0; i < (1u << 25) && !mbar_try_wait(&t1_full[q % T1_BUFS], (q / T1_BUFS) & 1); ++i)
          if (i > 256) __nanosleep(64);
      for (uint32_t q = (hq > QW_BUFS ? hq - QW_BUFS : 0); q < hq; ++q)
        for (uint32_t i = 0; i < (1u << 25) && !mbar_try_wait(&q_free[q % QW_BUFS], (q / QW_BUFS) & 1); ++i)
          if (i > 256) __nanosleep(64);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    // After a failed wait a warp stops touching TMEM and the pipelines but
    // keeps walking the tiles, so that every epilogue warp still reaches
    // every named barrier (the other roles give up at their next wait).
    const int wg = warp >> 2, qd = warp & 3;
    const int rl = qd * 32 + lane;  // row of the tile this thread owns
    const uint32_t t_lane = tmem + ((uint32_t)(qd * 32) << 16);
    uint8_t* qw = smem + SM_QW;
    const int grp = wg >> 1, sub = wg & 1;  // pass 2: halves hq % 2 == grp, codewords 32 sub ..
    const int w_off = kmaj_off(rl, sub * 32, 1024);  // this thread's 32 weights of a half
    uint32_t tu1 = 0, hq = 0, mt_n = 0;
    bool ok = true;
    const uint32_t nch = (uint32_t)((a.NT + MOM_CHUNK - 1) / MOM_CHUNK);  // chunks per tile
    // warpgroup 0: the moment chunks' running sums of its row (S1 x 8, S0),
    // in the shared slot of t, which pass 2 no longer reads once its
    // operands are built
    float* msum = reinterpret_cast<float*>(sm_t) + rl * 16;
    auto read_chunk = [&](uint32_t cl) {
      const uint32_t c = mt_n * nch + cl, mb = c & 1;
      if (ok) ok = warp_wait(&mom_full[mb], (c >> 1) & 1, abort_flag, a.status);
      if (!ok) return;
      tc_fence_after();
      uint32_t mv[16];
      tmem_ld16_nowait(t_lane + TM_MOM + 16u * mb, mv);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&mom_free[mb]);
#pragma unroll
      for (int i = 0; i < 9; ++i) msum[i] = (cl == 0 ? 0.0f : msum[i]) + __uint_as_float(mv[i]);
    };
    for (int64_t mt = blockIdx.x; mt < mtiles; mt += gridDim.x) {
      const int64_t blk = mt * DT_M + rl;
      const bool active = blk < a.nblocks;
      const int64_t row = active ? blk / a.B : 0;
      if (wg == 0) {
        // t = r1 / s (with the anchor: precision-weighted with w / s); kept in
        // shared memory across pass 1 to spare registers
        double t64[8];
        float g = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) t64[i] = 0.0;
        if (active) {
          const double sc = a.scale[row];
          const double sc2 = sc * sc;
          const float4 r0 = *reinterpret_cast<const float4*>(a.R1 + blk * 8);
          const float4 r1 = *reinterpret_cast<const float4*>(a.R1 + blk * 8 + 4);
          const float rv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
          double gg = 1.0, ga = 0.0;
          if (a.mode != 1) {
            gg = a.gamma1[row] * sc2;
            ga = a.W ? a.inv_tau2 : 0.0;  // anchor: tau codebook units wide
          }
          g = (float)fmin(gg + ga, 1e30);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            double ti = (double)rv[i] / sc;
            if (a.W && a.mode != 1) ti = (gg * ti + ga * ((double)a.W[blk * 8 + i] / sc)) / (gg + ga);
            t64[i] = ti;
          }
        }
        // pass-1 operands [t_hi | -1/2 -1/2 0...] and [t_lo | 0...], scaled
        // by 2^6 (the argmax does not change) so that t_lo stays out of the
        // fp16 subnormal range
        __half hi[16], lo[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) split16(t64[i] * 64.0, hi[i], lo[i]);
#pragma unroll
        for (int i = 8; i < 16; ++i) hi[i] = lo[i] = __float2half(0.0f);
        hi[8] = hi[9] = __float2half(-32.0f);
        store_row(At + A1_HI * OPER_BYTES, rl, hi);
        store_row(At + A1_LO * OPER_BYTES, rl, lo);
#pragma unroll
        for (int i = 0; i < 8; ++i) sm_t[rl * 8 + i] = t64[i];
        sm_g[rl] = g;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(a_full);
      }

      // ---------------------------------------------- pass 1: argmax
      float best = -INFINITY;
      int bidx = 0;
      for (int j = 0; j < a.NT; ++j, ++tu1) {
        const int buf = tu1 % T1_BUFS;
        if (ok) ok = warp_wait(&t1_full[buf], (tu1 / T1_BUFS) & 1, abort_flag, a.status);
        if (!ok) continue;
        tc_fence_after();
        uint32_t v[32];
        tmem_ld32_nowait(t_lane + (uint32_t)buf * T1_COLS + (uint32_t)(wg * 32), v);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&t1_empty[buf]);
        // maximum of the 32 scores as a tree of three-input maxima (depth 4)
        float t1[11];
#pragma unroll
        for (int k = 0; k < 10; ++k)
          t1[k] = fmax3(__uint_as_float(v[3 * k]), __uint_as_float(v[3 * k + 1]), __uint_as_float(v[3 * k + 2]));
        t1[10] = fmaxf(__uint_as_float(v[30]), __uint_as_float(v[31]));
        const float m0 = fmaxf(fmax3(fmax3(t1[0], t1[1], t1[2]), fmax3(t1[3], t1[4], t1[5]),
                                     fmax3(t1[6], t1[7], t1[8])),
                               fmaxf(t1[9], t1[10]));
        if (m0 > best) {  // first index of the chunk maximum
          int kk = 31;
#pragma unroll
          for (int k = 31; k >= 0; --k)
            if (__uint_as_float(v[k]) == m0) kk = k;
          best = m0;
          bidx = j * DT_N + wg * 32 + kk;
        }
      }
      // merge the column quarters: larger score, then the smaller index
      sm_bval[wg * DT_M + rl] = best;
      sm_bidx[wg * DT_M + rl] = bidx;
      named_sync_epi();
      if (wg == 0) {
#pragma unroll
        for (int w = 1; w < DT_WGS; ++w) {
          const float ob = sm_bval[w * DT_M + rl];
          const int oi = sm_bidx[w * DT_M + rl];
          if (ob > best || (ob == best && oi < bidx)) {
            best = ob;
            bidx = oi;
          }
        }
      }
      if (a.mode) {
        if (wg == 0 && active && ok) a.idx[blk] = (uint16_t)bidx;
        continue;
      }

      // ---------------------------------- pass 2 operands (centred on c*)
      if (wg == 0) {
        float cst[8];
        double t64[8];
        const float4 c0 = *reinterpret_cast<const float4*>(a.cb + (int64_t)bidx * 8);
        const float4 c1 = *reinterpret_cast<const float4*>(a.cb + (int64_t)bidx * 8 + 4);
        cst[0] = c0.x; cst[1] = c0.y; cst[2] = c0.z; cst[3] = c0.w;
        cst[4] = c1.x; cst[5] = c1.y; cst[6] = c1.z; cst[7] = c1.w;
#pragma unroll
        for (int i = 0; i < 8; ++i) t64[i] = sm_t[rl * 8 + i];
        const float g = sm_g[rl];
        // t - c* = q + r: q on the grid 2^-Fb with |q_i| 2^Fb <= 2047 (exact
        // fp16), Fb the finest grid up to F that holds this block's largest
        // coordinate, so |r| <= 2^-(Fb+1) stays ~2^-11 of |t - c*|.  r enters
        // the MMA as r 2^(Fb+1+rk), |.| <= 2^rk, an fp16 pair whose low half
        // is subnormal only for tiny r (rk is set at plan time so that
        // r.c* stays within fp16); the epilogue scales R back.
        double mx = 0.0;
#pragma unroll
        for (int i = 0; i < 8; ++i) mx = fmax(mx, fabs(t64[i] - (double)cst[i]));
        int Fb = a.F;
        while (Fb > a.Fmin && ldexp(mx, Fb) > 2047.0) --Fb;
        const double sF = ldexp(1.0, Fb), isF = ldexp(1.0, -Fb), sR = ldexp(1.0, Fb + 1 + a.rk);
        double qc = 0.0, rc = 0.0, nn = 0.0;
        __half q16[16], x16[16], rh[16], rlo[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const double tp = t64[i] - (double)cst[i];
          const double qi = fmin(fmax(rint(tp * sF), -2047.0), 2047.0);
          const double tq = qi * isF;
          q16[i] = __double2half(tq);
          split16((tp - tq) * sR, rh[i], rlo[i]);
          qc += tq * (double)cst[i];  // exact
          rc += ((double)__half2float(rh[i]) + (double)__half2float(rlo[i])) * (double)cst[i];  // x sR
          nn += (double)cst[i] * (double)cst[i];
          x16[i] = __float2half(cst[i]);
        }
#pragma unroll
        for (int i = 8; i < 16; ++i) q16[i] = x16[i] = rh[i] = rlo[i] = __float2half(0.0f);
        // constants against the [.. | n_hi n_lo 1 1 ..] columns of the codebook operand
        split16(-qc, q16[10], q16[11]);
        x16[8] = x16[9] = __float2half(-0.5f);
        split16(-0.5 * nn, x16[10], x16[11]);
        split16(-rc, rh[10], rh[11]);
        store_row(At + A2_Q * OPER_BYTES, rl, q16);
        store_row(At + A2_X * OPER_BYTES, rl, x16);
        store_row(At + A2_RH * OPER_BYTES, rl, rh);
        store_row(At + A2_RL * OPER_BYTES, rl, rlo);
        sm_g2[rl] = g * 1.4426950408889634f;  // logits in log2 units
        sm_rs[rl] = (float)(1.0 / sR);
        sm_bidx[rl] = bidx;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(a_full);
      }
      named_sync_epi();
      const float g2 = sm_g2[rl], rs = sm_rs[rl];
      const int c16 = sm_bidx[rl] >> 4, kst = sm_bidx[rl] & 15;  // c* as (16-chunk, column)

      // ------------------------------------------- pass 2: weights
      float zmax = -INFINITY;
      uint64_t S2p = 0;  // (+0, +0): S2 over even and odd codewords
      const uint64_t rs2 = f2_pack(rs, rs), g22 = f2_pack(g2, g2), sh2 = f2_pack(Q_SHIFT, Q_SHIFT);
      uint32_t rd = 0;  // moment chunks read (warpgroup 0)
      // The two halves of every codebook tile go to the two groups of eight
      // warps (group g takes the halves with hq % 2 == g, so TMEM score
      // buffer g and weights buffers g, g + 2): while one group turns its
      // half's scores into weights the other waits for its MMAs or stores,
      // so the exponentials of one overlap the latencies of the other.  A
      // warp covers 32 of its half's 64 codewords, 16 at a time.
      for (int j = 0; j < a.NT; ++j) {
        // a chunk is read one codebook tile into the next chunk, by when its
        // moment MMAs have long been issued
        if (wg == 0 && j > MOM_CHUNK && (j - 1) % MOM_CHUNK == 0) read_chunk(rd++);
        const uint32_t u = hq + 2u * (uint32_t)j + (uint32_t)grp;  // this group's half of tile j
        const int buf = (int)(u % T2_BUFS), qb = (int)(u % QW_BUFS);
        if (ok) ok = warp_wait(&t2_full[buf], (u / T2_BUFS) & 1, abort_flag, a.status);
        // the moment MMAs of the weights buffer's previous use have read it
        if (ok && u >= QW_BUFS) ok = warp_wait(&q_free[qb], (u / QW_BUFS - 1) & 1, abort_flag, a.status);
        if (!ok) continue;
        tc_fence_after();
        uint8_t* wb = qw + qb * 2 * QW_BYTES + w_off;
#pragma unroll 1
        for (int k = 0; k < 2; ++k) {
          const uint32_t ta = t_lane + (uint32_t)buf * T2_COLS + (uint32_t)(sub * 32 + k * 16);
          uint32_t Q[16], X[16], R[16];
          tmem_ld16_nowait(ta, Q);
          tmem_ld16_nowait(ta + 64u, X);
          tmem_ld16_nowait(ta + 128u, R);
          tmem_wait_ld();
          if (k == 1) {  // the half's scores are read: hand the buffer back
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&t2_empty[buf]);
          }
          // c* needs no special case here: X(c*) = 0 exactly, so it adds
          // nothing to S2, and its weight is zeroed in the moment operand
          // below.  (Its logit is 0 up to R's rounding, so z(c*) reaches the
          // overflow mark only at g > ~5e9, where the point mass on c* that
          // the overflow fallback returns is the answer.)
          // Two codewords per packed f32x2 instruction, each half rounded as
          // the scalar form: z = g2 (R rs + (Q + X)) + 8 (Q + X is exact, R
          // carries the rounding), q = 2^z, S2 += q X (X = -|c - c*|^2 / 2),
          // and the weight as a saturating fp16 pair hi + lo.
          uint32_t hi[8], lo[8];
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const uint64_t xv = f2_pack(__uint_as_float(X[2 * p]), __uint_as_float(X[2 * p + 1]));
            const uint64_t qx = f2_add(f2_pack(__uint_as_float(Q[2 * p]), __uint_as_float(Q[2 * p + 1])), xv);
            const uint64_t rr = f2_pack(__uint_as_float(R[2 * p]), __uint_as_float(R[2 * p + 1]));
            float z0, z1;
            f2_unpack(f2_fma(g22, f2_fma(rr, rs2, qx), sh2), z0, z1);
            zmax = fmax3(zmax, z0, z1);
            const float e0 = ex2_approx(z0), e1 = ex2_approx(z1);
            const uint64_t e = f2_pack(e0, e1);
            S2p = f2_fma(e, xv, S2p);
            asm("cvt.rn.satfinite.f16x2.f32 %0, %2, %1;" : "=r"(hi[p]) : "f"(e0), "f"(e1));
            const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&hi[p]));
            float d0, d1;
            f2_unpack(f2_sub(e, f2_pack(h.x, h.y)), d0, d1);
            asm("cvt.rn.satfinite.f16x2.f32 %0, %2, %1;" : "=r"(lo[p]) : "f"(d0), "f"(d1));
          }
          uint8_t* wk = wb + k * 256;  // codewords 16k .. 16k + 15 of this warp's 32
          *reinterpret_cast<uint4*>(wk) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(wk + 128) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
          *reinterpret_cast<uint4*>(wk + QW_BYTES) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          *reinterpret_cast<uint4*>(wk + QW_BYTES + 128) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
          if (j * 8 + grp * 4 + sub * 2 + k == c16) {  // c*: weight 0 (added back at the end)
            const int o = (kst >> 3) * 128 + (kst & 7) * 2;
            *reinterpret_cast<uint16_t*>(wk + o) = 0;
            *reinterpret_cast<uint16_t*>(wk + QW_BYTES + o) = 0;
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_full[qb]);
      }
      hq += 2u * (uint32_t)a.NT;
      {
        float s2a, s2b;
        f2_unpack(S2p, s2a, s2b);
        sm_s2[wg * DT_M + rl] = s2a + s2b;
      }
      sm_bval[wg * DT_M + rl] = zmax;
      named_sync_epi();
      if (wg == 0) {
        // S0 = sum q, S1 = sum q c over c != c* (weights x 2^8) from the
        // moment accumulator; c* adds 2^8 to S0, 2^8 c* to S1 and 0 to S2:
        // E[c - c*] = (S1 - c* S0) / (2^8 + S0), E|c - c*|^2 = -2 S2 / (2^8 + S0)
        for (; rd < nch; ++rd) read_chunk(rd);
        float mv[9];
#pragma unroll
        for (int i = 0; i < 9; ++i) mv[i] = msum[i];
        if (active && ok) {
          const int bi = sm_bidx[rl];
          const float4 c0 = *reinterpret_cast<const float4*>(a.cb + (int64_t)bi * 8);
          const float4 c1 = *reinterpret_cast<const float4*>(a.cb + (int64_t)bi * 8 + 4);
          const float cst[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          float s2 = 0.0f, zm = -INFINITY;
#pragma unroll
          for (int w = 0; w < DT_WGS; ++w) {
            s2 += sm_s2[w * DT_M + rl];
            zm = fmaxf(zm, sm_bval[w * DT_M + rl]);
          }
          const float S0 = mv[8];
          const float sc = a.scale[row], off = a.offset[row];
          const float inv = 1.0f / (256.0f + S0);
          // a weight past the fp16 range (more than 2^8 times c*'s): point mass
          const bool point = zm >= 15.99f;
          float mm = 0.0f, xo[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float mc = point ? 0.0f : fmaf(-cst[i], S0, mv[i]) * inv;
            mm = fmaf(mc, mc, mm);
            xo[i] = fmaf(sc, cst[i] + mc, off);
          }
          *reinterpret_cast<float4*>(a.xhat + blk * 8) = make_float4(xo[0], xo[1], xo[2], xo[3]);
          *reinterpret_cast<float4*>(a.xhat + blk * 8 + 4) = make_float4(xo[4], xo[5], xo[6], xo[7]);
          // E|c - c*|^2 - |E c - c*|^2
          const float var = point ? 0.0f : fmaxf(-2.0f * s2 * inv - mm, 0.0f);
          a.vblock[blk] = (float)((double)sc * sc * var);
          if (a.idx) a.idx[blk] = (uint16_t)bi;
        }
      }
      ++mt_n;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(DT_TMEM_COLS));
  }
}

}  // namespace

// Plan-time: decide whether the codebook can use the tensor-core denoiser.
// Returns the grid bits F of the exact part of t - c*, or -1.  Qualifies: K a
// multiple of 128, every coordinate an integer multiple of 2^-e (e <= 8) with
// C = max |c_i| 2^e <= 127 and |c|^2 < 2^14.  Then (in units of 2^-(F+e),
// F = e + f) q.c - q.c* stays below 2^14 C and |c - c*|^2 / 2 below
// 2^(3+f) C^2, and f (<= 8) is the largest with the sum below 2^22: every
// partial sum of the MMAs for Q and X is an exact fp32 value.  A block may
// use any coarser grid down to 2^-(e+1) (the bounds only shrink).
int vec_tc_grid_bits(const float* cb_host, int K, int* e_out, int* rk_out) {
  if (K <= 0 || K % DT_N != 0) return -1;
  for (int e = 0; e <= 8; ++e) {
    const double u = std::ldexp(1.0, e);
    bool ok = true;
    double cmax = 0.0, nmax = 0.0;
    for (int64_t c = 0; c < K && ok; ++c) {
      double nn = 0.0;
      for (int i = 0; i < 8; ++i) {
        const double v = (double)cb_host[c * 8 + i];
        const double w = v * u;
        if (!std::isfinite(w) || w != std::nearbyint(w)) {
          ok = false;
          break;
        }
        cmax = std::fmax(cmax, std::fabs(w));
        nn += v * v;
      }
      nmax = std::fmax(nmax, nn);
    }
    if (!ok) continue;
    if (cmax > 127.0 || nmax >= 16384.0) return -1;
    for (int f = 8; f >= 1; --f)
      if (std::ldexp(cmax, 14) + std::ldexp(cmax * cmax, 3 + f) < std::ldexp(1.0, 22)) {
        *e_out = e;
        // r 2^(Fb+1+rk) is at most 2^rk per coordinate: 8 2^rk max|c_i| <= 2^14
        const double cm = std::fmax(std::ldexp(cmax, -e), 1e-30);
        *rk_out = (int)std::fmin(9.0, std::fmax(0.0, std::floor(std::log2(2048.0 / cm))));
        return e + f;
      }
    return -1;
  }
  return -1;
}

// Codebook operand images, 8 KiB per tile of 128 codewords, in the no-swizzle
// K-major layout the kernel's descriptors describe:
//   scores      128 rows (codewords) x 16: [c_0 .. c_7 | n_hi n_lo 1 1 0 0 0 0],
//               |c|^2 = n_hi + n_lo  (8-row groups 256 B apart)
//   moments     16 rows x 128 (codewords): rows 0-7 the coordinates, row 8 ones
//               (8-row groups 2048 B apart)
mpq_status build_vec_tc_tables(mpq_plan_s* p, const float* cb_host) {
  const int NT = p->K / DT_N;
  std::vector<__half> img((size_t)NT * STAGE_BYTES / 2, __float2half(0.0f));
  for (int c = 0; c < p->K; ++c) {
    const int j = c / DT_N, r = c % DT_N;
    __half* sc = img.data() + (size_t)j * STAGE_BYTES / 2;
    __half* mo = sc + OPER_BYTES / 2;
    double nn = 0.0;
    for (int i = 0; i < 8; ++i) {
      const float v = cb_host[(size_t)c * 8 + i];
      sc[kmaj_off(r, i, 256) / 2] = __float2half(v);
      mo[kmaj_off(i, r, 2048) / 2] = __float2half(v);
      nn += (double)v * v;
    }
    const __half nh = __double2half(nn);
    sc[kmaj_off(r, 8, 256) / 2] = nh;
    sc[kmaj_off(r, 9, 256) / 2] = __double2half(nn - (double)__half2float(nh));
    sc[kmaj_off(r, 10, 256) / 2] = sc[kmaj_off(r, 11, 256) / 2] = __float2half(1.0f);
    mo[kmaj_off(8, r, 2048) / 2] = __float2half(1.0f);
  }
  MPQ_CUDA(cudaMalloc(&p->cb_tc, img.size() * sizeof(__half)));
  MPQ_CUDA(cudaMemcpy(p->cb_tc, img.data(), img.size() * sizeof(__half), cudaMemcpyHostToDevice));
  return MPQ_OK;
}

mpq_status launch_denoise_vec_tc(const mpq_plan_s* p, const float* R1, const double* gamma1,
                                 const float* scale, const float* offset, int64_t m,
                                 const float* W, const double* gamma1_0, double inv_tau2,
                                 float* xhat1, float* vblock, uint16_t* idx, int mode,
                                 cudaStream_t st) {
  static bool attr_set[64] = {};
  int dev = 0;
  MPQ_CUDA(cudaGetDevice(&dev));
  if (dev < 64 && !attr_set[dev]) {
    MPQ_CUDA(cudaFuncSetAttribute(k_denoise_vec_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  DT_SMEM_BYTES));
    attr_set[dev] = true;
  }
  int sms = 0;
  MPQ_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  cudaFuncAttributes fa{};
  MPQ_CUDA(cudaFuncGetAttributes(&fa, k_denoise_vec_tc));
  if (fa.maxThreadsPerBlock < DT_THREADS)
    return fail(MPQ_ERR_CUDA, "k_denoise_vec_tc: " + std::to_string(fa.numRegs) +
                                  " registers/thread allow only " +
                                  std::to_string(fa.maxThreadsPerBlock) + " threads per block");
  DenoiseTcArgs a{};
  a.R1 = R1;
  a.gamma1 = gamma1;
  a.scale = scale;
  a.offset = offset;
  a.W = W;
  a.gamma1_0 = gamma1_0;
  a.inv_tau2 = inv_tau2;
  a.B = p->B;
  a.nblocks = m * p->B;
  a.NT = p->K / DT_N;
  a.F = p->vec_tc_F;
  a.Fmin = p->vec_tc_Fmin;
  a.rk = p->vec_tc_rk;
  a.cb_tc = reinterpret_cast<const uint8_t*>(p->cb_tc);
  a.cb = p->cb;
  a.xhat = xhat1;
  a.vblock = vblock;
  a.idx = idx;
  a.mode = mode;
  a.status = p->status;
  const int64_t mtiles = cdiv(a.nblocks, DT_M);
  const unsigned grid = (unsigned)std::min<int64_t>(mtiles, (int64_t)sms);
  {
    ProfScope ps_(mode == 1 ? "k_denoise_vec_tc(nearest)" : mode == 2 ? "k_denoise_vec_tc(map)" : "k_denoise_vec_tc",
                  st);
    k_denoise_vec_tc<<<grid, DT_THREADS, DT_SMEM_BYTES, st>>>(a);
  }
  count_launch();
  return check_launch("k_denoise_vec_tc");
}

}  // namespace mpq
