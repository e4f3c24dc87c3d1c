// Tensor-core candidate scan of the vector CD step (d = 8, lattice codebooks).
//
// One step of exact block CD visits block b of every row: the energy change of
// moving x_b to codeword c is scale^2 (score(c) - score(x_b)) with
// score(c) = qtab_b(c) - c.g',  qtab_b(c) = 1/2 c^T G_b c,  g' = (h_b + G_b x_b)/scale
// (the CD of the MPQ page, section "Key design 3"; block CD in the metric
// H = X^T X).  The scan finds the argmin of score(c) over all K codewords
// for every row, lowest index on ties.  The contraction c.g' runs on the
// tensor cores: A = -2^k g' as an fp16 hi/lo pair (k per row, so that the low
// half stays clear of subnormals) against the plan's codebook operand
// [c | |c|^2 pair, 1, 1] (the extra columns meet zeros), two MMAs
// (M = 128 rows, N = 256 codewords, K = 16) per tile into TMEM; the epilogue
// forms score = qtab + 2^-k D in fp32 and keeps the first minimum.
//
// The same scan serves the greedy baseline (LDLQ with E8 rounding): the
// codeword nearest a block's working values v_b is the argmin of
// 1/2 |c|^2 - c.t with t = v_b / scale, i.e. score(c) with qtab replaced by
// 1/2 |c|^2 and g' by t.
//
// Grid: (slices of the codebook) x (tiles of 128 rows); every CTA writes the
// minimum of its slice per row, and the apply step combines the slices.
// Warps 0-15 read TMEM (warp w: lanes 32 (w % 4) .. +31, columns 64 (w / 4)
// .. +63 of each 256-codeword tile), warp 16 owns TMEM and issues the MMAs,
// warp 17 issues the bulk copies of the codebook operand and the qtab row
// through a 10-stage ring; TMEM holds 2 score buffers.  All waits are bounded.
#include <cuda.h>
#include <cuda_fp16.h>

#include <cmath>

#include "f32x2.cuh"
#include "mpq_internal.cuh"
#include "tc_ptx.cuh"

namespace mpq {
namespace {
using namespace tcx;

// A scan tile is 256 codewords (two of the plan's 128-codeword operand
// images, copied side by side): one MMA pair of N = 256 per tile, so that the
// fixed cost of issuing an MMA and of each pipeline handshake is spread over
// twice the codewords (two TMEM buffers of 256 columns).  The ring holds 10
// tiles of 9 KiB.
constexpr int SC_M = 128, SC_N = 256, SC_TN = SC_N / 128, SC_STAGES = 10, SC_BUFS = 2;
constexpr int SC_EPI_WARPS = 16, SC_WGS = 4;
constexpr int SC_THREADS = (SC_EPI_WARPS + 2) * 32;
constexpr int SC_MMA_WARP = SC_EPI_WARPS, SC_LOAD_WARP = SC_EPI_WARPS + 1;
constexpr int SC_OPER = 128 * 32;           // 128 rows x 16 fp16
constexpr int SC_QT = SC_N * 4;             // qtab of one tile (fp32)
constexpr int SC_STAGE = SC_TN * SC_OPER + SC_QT;
constexpr int SC_IMG_STRIDE = 8192;         // bytes per tile in the plan's operand images
constexpr uint32_t SC_TMEM_COLS = 512;
constexpr uint32_t SC_IDESC = idesc_f16(SC_M, SC_N);
constexpr int SC_A = 0;                                     // A hi, A lo
constexpr int SC_B = SC_A + 2 * SC_OPER;                    // stage ring
constexpr int SC_ROW = SC_B + SC_STAGES * SC_STAGE;         // per-row data
constexpr int SC_BAR = SC_ROW + (1 + 2 * SC_WGS) * SC_M * 4;
constexpr int SC_END = SC_BAR + (2 * SC_STAGES + 2 * SC_BUFS + 1) * 8 + 16;
// more than half of the SM's shared memory: one CTA (and one TMEM owner) per SM
constexpr int SC_SMEM = 120 * 1024;
static_assert(SC_END + 1024 <= SC_SMEM, "scan shared memory");

struct ScanArgs {
  int64_t m, n;
  int K, NT;              // codewords, scan tiles of SC_N (the last one may be partial)
  int64_t b, t0;          // block, first column of its CD tile
  const uint8_t* cb_tc;   // NT x 8 KiB operand images (the first 4 KiB: scores)
  const float* cb;        // K x 8
  const float* qtab_row;  // K: the score table of this scan (qtab_b, or 1/2 |c|^2)
  const float* Wk;        // greedy mode: working rows (t = Wk[row, block] / scale), else NULL
  int64_t ldw;
  const float* H;         // n x n fp32
  const float* scale;
  const uint16_t* idx;
  const float* h;         // gradient (used at the first block of a tile)
  int64_t ldh;
  const float* hl;        // tile-local gradient (other blocks)
  float* part_val;        // m x nslices
  int* part_idx;
  int nslices;
  int* status;
};

__device__ __forceinline__ uint64_t sc_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(128 >> 4) << 16;   // LBO: next K chunk
  d |= (uint64_t)(256 >> 4) << 32;   // SBO: next 8-row group
  d |= (uint64_t)1 << 46;
  return d;
}

__device__ __forceinline__ int sc_off(int r, int h) { return (r & 7) * 16 + (r >> 3) * 256 + h * 128; }

__device__ __forceinline__ void sc_ld32(uint32_t taddr, uint32_t (&v)[32]) {
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
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// bounded wait that gives up when another role has aborted
__device__ __forceinline__ bool sc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                        int* status) {
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

__global__ void __launch_bounds__(SC_THREADS, 1) k_cd_vec_scan(ScanArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  float* sm_rsc = reinterpret_cast<float*>(smem + SC_ROW);       // 2^-k per row
  float* sm_bval = sm_rsc + SC_M;                                // [SC_WGS][128]
  int* sm_bidx = reinterpret_cast<int*>(sm_bval + SC_WGS * SC_M);
  uint64_t* b_full = reinterpret_cast<uint64_t*>(smem + SC_BAR);
  uint64_t* b_empty = b_full + SC_STAGES;
  uint64_t* t_full = b_empty + SC_STAGES;
  uint64_t* t_empty = t_full + SC_BUFS;
  uint64_t* a_full = t_empty + SC_BUFS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(a_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slice = blockIdx.x;
  const int64_t r0 = (int64_t)blockIdx.y * SC_M;
  const int j0 = (int)((int64_t)slice * a.NT / a.nslices);
  const int nt = (int)((int64_t)(slice + 1) * a.NT / a.nslices) - j0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SC_STAGES; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], SC_EPI_WARPS);  // released after the epilogue has read qtab
    }
    for (int b = 0; b < SC_BUFS; ++b) {
      mbar_init(&t_full[b], 1);
      mbar_init(&t_empty[b], SC_EPI_WARPS);
    }
    mbar_init(a_full, SC_M);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == SC_MMA_WARP) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(SC_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == SC_LOAD_WARP) {
    if (lane == 0) {
      int t = 0;
      for (; t < nt; ++t) {
        const int s = t % SC_STAGES;
        if (t >= SC_STAGES && !sc_wait(&b_empty[s], (t / SC_STAGES - 1) & 1, abort_flag, a.status))
          break;
        uint8_t* st = smem + SC_B + s * SC_STAGE;
        // the tile's 128-codeword images present (a partial last tile has
        // fewer; the MMA's columns past them are never read back)
        const int nimg = min(SC_TN, (a.K - (j0 + t) * SC_N) / 128);
        mbar_expect_tx(&b_full[s], (uint32_t)(nimg * (SC_OPER + 128 * 4)));
        for (int i = 0; i < nimg; ++i)
          bulk_load_1d(st + i * SC_OPER, a.cb_tc + (size_t)((j0 + t) * SC_TN + i) * SC_IMG_STRIDE,
                       SC_OPER, &b_full[s]);
        bulk_load_1d(st + SC_TN * SC_OPER, a.qtab_row + (int64_t)(j0 + t) * SC_N,
                     (uint32_t)(nimg * 128 * 4), &b_full[s]);
      }
      for (int q = (t > SC_STAGES ? t - SC_STAGES : 0); q < t; ++q)  // copies land before exit
        for (uint32_t i = 0; i < (1u << 25) && !mbar_try_wait(&b_full[q % SC_STAGES], (q / SC_STAGES) & 1); ++i)
          if (i > 256) __nanosleep(64);
    }
  } else if (warp == SC_MMA_WARP) {
    if (lane == 0) {
      int t = 0;
      if (sc_wait(a_full, 0, abort_flag, a.status)) {
        tc_fence_after();
        const uint32_t ah = smem_u32(smem + SC_A), al = ah + SC_OPER;
        for (; t < nt; ++t) {
          const int s = t % SC_STAGES, buf = t % SC_BUFS;
          if (!sc_wait(&b_full[s], (t / SC_STAGES) & 1, abort_flag, a.status)) break;
          if (t >= SC_BUFS && !sc_wait(&t_empty[buf], (t / SC_BUFS - 1) & 1, abort_flag, a.status)) break;
          tc_fence_after();
          const uint64_t bd = sc_desc(smem_u32(smem + SC_B + s * SC_STAGE));
          const uint32_t d = tmem + (uint32_t)buf * SC_N;
          umma_f16(d, sc_desc(ah), bd, SC_IDESC, 0u);
          umma_f16(d, sc_desc(al), bd, SC_IDESC, 1u);
          umma_commit(&t_full[buf]);
        }
      }
      for (int q = (t > SC_BUFS ? t - SC_BUFS : 0); q < t; ++q)  // MMAs finish before TMEM is freed
        for (uint32_t i = 0; i < (1u << 25) && !mbar_try_wait(&t_full[q % SC_BUFS], (q / SC_BUFS) & 1); ++i)
          if (i > 256) __nanosleep(64);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int wg = warp >> 2, qd = warp & 3;
    const int rl = qd * 32 + lane;
    const int64_t row = r0 + rl;
    const bool active = row < a.m;
    if (wg == 0) {
      // g' = (h_b + G_b x_b) / scale; A = -2^k g' as an fp16 pair
      float g[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (active && a.Wk) {  // greedy: the block's working values in codebook units
        const float inv = 1.0f / a.scale[row];
#pragma unroll
        for (int i = 0; i < 8; ++i) g[i] = a.Wk[row * a.ldw + 8 * a.b + i] * inv;
      } else if (active) {
        const float sc = a.scale[row];
        const int kcur = a.idx[row * (a.n / 8) + a.b];
        const float* hb = (8 * a.b == a.t0) ? a.h + row * a.ldh + 8 * a.b
                                            : a.hl + row * CD_TILE + (8 * a.b - a.t0);
        float x[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = sc * a.cb[(int64_t)kcur * 8 + j];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float gi = hb[i];
          const float* Hi = a.H + (8 * a.b + i) * a.n + 8 * a.b;
#pragma unroll
          for (int j = 0; j < 8; ++j) gi = fmaf(Hi[j], x[j], gi);
          g[i] = gi / sc;
        }
      }
      float mx = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(g[i]));
      const int k = (mx > 0.0f && isfinite(mx)) ? 10 - ilogbf(mx) : 0;
      __half hi[16], lo[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) hi[i] = lo[i] = __float2half(0.0f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float v = ldexpf(-g[i], k);
        hi[i] = __float2half_rn(v);
        lo[i] = __float2half_rn(v - __half2float(hi[i]));
      }
      uint4 c0, c1;
      __half* p0 = reinterpret_cast<__half*>(&c0);
      __half* p1 = reinterpret_cast<__half*>(&c1);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        p0[i] = hi[i];
        p1[i] = hi[8 + i];
      }
      *reinterpret_cast<uint4*>(smem + SC_A + sc_off(rl, 0)) = c0;
      *reinterpret_cast<uint4*>(smem + SC_A + sc_off(rl, 1)) = c1;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        p0[i] = lo[i];
        p1[i] = lo[8 + i];
      }
      *reinterpret_cast<uint4*>(smem + SC_A + SC_OPER + sc_off(rl, 0)) = c0;
      *reinterpret_cast<uint4*>(smem + SC_A + SC_OPER + sc_off(rl, 1)) = c1;
      sm_rsc[rl] = ldexpf(1.0f, -k);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(a_full);
    }
    asm volatile("bar.sync 1, %0;" ::"n"(SC_EPI_WARPS * 32) : "memory");
    const float rsc = sm_rsc[rl];
    const uint64_t rsc2 = f2_pack(rsc, rsc);
    float best = INFINITY;
    int bidx = 0x7fffffff;
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      const int s = t % SC_STAGES, buf = t % SC_BUFS;
      if (ok) ok = __all_sync(0xffffffffu, sc_wait(&t_full[buf], (t / SC_BUFS) & 1, abort_flag, a.status));
      if (!ok) continue;
      tc_fence_after();
      const int nvalid = min(SC_N, a.K - (j0 + t) * SC_N);  // codewords in this tile
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {  // this warp's 64 columns, 32 at a time
        const int cbase = wg * 64 + hh * 32;
        uint32_t v[32];
        sc_ld32(tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)buf * SC_N + (uint32_t)cbase, v);
        if (hh == 1) {  // the tile's scores are read: hand the buffer back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&t_empty[buf]);
        }
        const float4* q4 = reinterpret_cast<const float4*>(smem + SC_B + s * SC_STAGE + SC_TN * SC_OPER) +
                           cbase / 4;
        // score = D rsc + qtab, two codewords per packed f32x2 fma; columns
        // past the codebook's end (a partial last tile) score +inf
        float sv[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float4 q = q4[c];
          f2_unpack(f2_fma(f2_pack(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1])), rsc2,
                           f2_pack(q.x, q.y)),
                    sv[4 * c], sv[4 * c + 1]);
          f2_unpack(f2_fma(f2_pack(__uint_as_float(v[4 * c + 2]), __uint_as_float(v[4 * c + 3])), rsc2,
                           f2_pack(q.z, q.w)),
                    sv[4 * c + 2], sv[4 * c + 3]);
        }
        if (cbase + 32 > nvalid) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (cbase + c >= nvalid) sv[c] = INFINITY;
        }
        // minimum of the 32 scores as a tree of three-input minima (depth 4)
        float t1[11];
#pragma unroll
        for (int c = 0; c < 10; ++c) t1[c] = fmin3(sv[3 * c], sv[3 * c + 1], sv[3 * c + 2]);
        t1[10] = fminf(sv[30], sv[31]);
        const float m0 = fminf(fmin3(fmin3(t1[0], t1[1], t1[2]), fmin3(t1[3], t1[4], t1[5]),
                                     fmin3(t1[6], t1[7], t1[8])),
                               fminf(t1[9], t1[10]));
        if (m0 < best) {  // first index of the chunk minimum
          int kk = 31;
#pragma unroll
          for (int c = 31; c >= 0; --c)
            if (sv[c] == m0) kk = c;
          best = m0;
          bidx = (j0 + t) * SC_N + cbase + kk;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&b_empty[s]);  // qtab of this stage is read
    }
    sm_bval[wg * SC_M + rl] = best;
    sm_bidx[wg * SC_M + rl] = bidx;
    asm volatile("bar.sync 1, %0;" ::"n"(SC_EPI_WARPS * 32) : "memory");
    if (wg == 0 && active && ok) {
#pragma unroll
      for (int w = 1; w < SC_WGS; ++w) {
        const float ob = sm_bval[w * SC_M + rl];
        const int oi = sm_bidx[w * SC_M + rl];
        if (ob < best || (ob == best && oi < bidx)) {
          best = ob;
          bidx = oi;
        }
      }
      a.part_val[row * a.nslices + slice] = best;
      a.part_idx[row * a.nslices + slice] = bidx;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == SC_MMA_WARP) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(SC_TMEM_COLS));
  }
}

}  // namespace

int cd_scan_slices(int64_t m, int K) {
  const int64_t mtiles = cdiv(m, SC_M);
  return (int)std::max<int64_t>(1, std::min<int64_t>((K + SC_N - 1) / SC_N, 148 / std::max<int64_t>(mtiles, 1)));
}

mpq_status launch_cd_vec_scan(const mpq_plan_s* p, int64_t m, int64_t b, int64_t t0,
                              const float* scale, const uint16_t* idx, const float* h,
                              int64_t ldh, const float* hl, float* part_val, int* part_idx,
                              int nslices, cudaStream_t st) {
  static bool attr_set[64] = {};
  int dev = 0;
  MPQ_CUDA(cudaGetDevice(&dev));
  if (dev < 64 && !attr_set[dev]) {
    MPQ_CUDA(cudaFuncSetAttribute(k_cd_vec_scan, cudaFuncAttributeMaxDynamicSharedMemorySize, SC_SMEM));
    attr_set[dev] = true;
  }
  ScanArgs a{};
  a.m = m;
  a.n = p->n;
  a.K = p->K;
  a.NT = (p->K + SC_N - 1) / SC_N;
  a.b = b;
  a.t0 = t0;
  a.cb_tc = reinterpret_cast<const uint8_t*>(p->cb_tc);
  a.cb = p->cb;
  a.qtab_row = p->qtab + b * p->K;
  a.H = p->H32;
  a.scale = scale;
  a.idx = idx;
  a.h = h;
  a.ldh = ldh;
  a.hl = hl;
  a.part_val = part_val;
  a.part_idx = part_idx;
  a.nslices = nslices;
  a.status = p->status;
  dim3 grid((unsigned)nslices, (unsigned)cdiv(m, SC_M));
  {
    ProfScope ps_("k_cd_vec_scan", st);
    k_cd_vec_scan<<<grid, SC_THREADS, SC_SMEM, st>>>(a);
  }
  count_launch();
  return check_launch("k_cd_vec_scan");
}

mpq_status launch_ldlq_vec_scan(const mpq_plan_s* p, int64_t m, int64_t b, const float* scale,
                                const float* Wk, int64_t ldw, float* part_val, int* part_idx,
                                int nslices, cudaStream_t st) {
  static bool attr_set[64] = {};
  int dev = 0;
  MPQ_CUDA(cudaGetDevice(&dev));
  if (dev < 64 && !attr_set[dev]) {
    MPQ_CUDA(cudaFuncSetAttribute(k_cd_vec_scan, cudaFuncAttributeMaxDynamicSharedMemorySize, SC_SMEM));
    attr_set[dev] = true;
  }
  if (!p->cb_hnorm) return fail(MPQ_ERR_INVALID_ARG, "the plan has no half-norm table");
  ScanArgs a{};
  a.m = m;
  a.n = p->n;
  a.K = p->K;
  a.NT = (p->K + SC_N - 1) / SC_N;
  a.b = b;
  a.t0 = 8 * b;
  a.cb_tc = reinterpret_cast<const uint8_t*>(p->cb_tc);
  a.cb = p->cb;
  a.qtab_row = p->cb_hnorm;
  a.Wk = Wk;
  a.ldw = ldw;
  a.scale = scale;
  a.part_val = part_val;
  a.part_idx = part_idx;
  a.nslices = nslices;
  a.status = p->status;
  dim3 grid((unsigned)nslices, (unsigned)cdiv(m, SC_M));
  {
    ProfScope ps_("k_ldlq8_scan", st);
    k_cd_vec_scan<<<grid, SC_THREADS, SC_SMEM, st>>>(a);
  }
  count_launch();
  return check_launch("k_ldlq8_scan");
}

}  // namespace mpq
