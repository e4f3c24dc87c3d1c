// Tensor-core GEMM for the fp32 contractions of the solve (sm_100a tcgen05).
//
//   C[M x N] = diag(row_scale) * (A_hi B_hi^T + A_hi B_lo^T + A_lo B_hi^T) * b_scale
//
// A and B are fp32 matrices stored as power-of-two-scaled fp16 pairs
// (x * 2^-e = hi + lo, hi = fp16(x * 2^-e), lo = fp16(x * 2^-e - hi)), so
// hi + lo carries ~22 significand bits and the three products recover an
// fp32-accurate contraction (the dropped lo*lo term is ~2^-22 relative).
// Both operands are K-major (K contiguous).  Persistent kernel in two forms:
//  - CTA pairs (M > 128, K >= 512): a cluster of two CTAs on two SMs computes each
//    256 x 256 tile with tcgen05.mma.cta_group::2.  Each CTA stages 128 rows
//    of A and its half (128 rows) of the tile's B; the MMAs, issued by the
//    even CTA, read both CTAs' shared memory and leave each CTA's 128 x 256
//    accumulator in its own TMEM.  K steps of 64 with 128-byte swizzle
//    through a 3-stage ring of 64 KiB.  Per MAC an SM moves 2/3 of the
//    operand bytes of a single-CTA 128 x 256 tile, in half as many
//    128-byte requests as 64-byte rows take.
//  - single CTAs (M <= 128, K < 512, or no pair fits): 128 x 256 tiles, K
//    steps of 32 with 64-byte swizzle through a 4-stage ring of 48 KiB.
// fp16 kind::f16 MMAs with the fp32 accumulator in TMEM (two 256-column
// accumulators, so that the epilogue of one tile overlaps the MMAs of the
// next); operands staged by TMA (no multicast) through an mbarrier ring that
// runs across tiles.  Warp 0 issues TMA, warp 1 owns TMEM and issues the MMAs
// from one thread, warps 2-5 read the accumulators back (tcgen05.ld) and
// store C.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <map>
#include <mutex>
#include <tuple>

#include "mpq_internal.cuh"
#include "tc_ptx.cuh"

namespace mpq {
namespace {
using namespace tcx;

constexpr int TC_THREADS = 192;

// Tiles are 128 (single) or 256 (pair) rows by 256 columns (the three MMAs of
// a k-step then read 96 B of shared memory per cycle of tensor work, against
// 128 B, the whole shared-memory bandwidth, at 128 x 128) for as many full
// waves of the grid as the product holds; the 256-column tiles left over for
// a last, partial wave run as two 128-column tiles each, and an odd
// 128-column strip at the right edge as 128-column tiles too.  Wide tiles go
// in groups of 8 M-tiles (M fastest) so that the A and B panels in flight
// stay in L2.
constexpr int PBN = 128, WBN = 256, PGROUP = 8;
constexpr int P_STG_WARP = 8192;  // epilogue staging per warp
constexpr uint32_t P_TMEM_COLS = 2 * WBN;

template <bool PAIR>
struct TcCfg;
template <>
struct TcCfg<false> {
  static constexpr int BK = 32, STAGES = 4, TM = 128;
  static constexpr int B_BOX = 128;                 // rows of B per TMA box
  static constexpr int B_HALF = 256 * BK * 2;       // one split half of up to 256 rows of B
  static constexpr uint32_t IDESC_W = idesc_f16(128, WBN), IDESC_N = idesc_f16(128, PBN);
  __device__ static uint64_t desc(uint32_t a) { return sw64_desc(a); }
};
template <>
struct TcCfg<true> {
  static constexpr int BK = 64, STAGES = 3, TM = 256;
  static constexpr int B_BOX = 64;
  static constexpr int B_HALF = 128 * BK * 2;       // this CTA's half of the tile's B
  static constexpr uint32_t IDESC_W = idesc_f16(256, WBN), IDESC_N = idesc_f16(256, PBN);
  __device__ static uint64_t desc(uint32_t a) { return sw128_desc(a); }
};
template <bool PAIR>
struct TcLayout {
  static constexpr int A_TILE = 128 * TcCfg<PAIR>::BK * 2;  // 128 rows of one split half
  static constexpr int STAGE = 2 * A_TILE + 2 * TcCfg<PAIR>::B_HALF;
  static constexpr int SMEM = TcCfg<PAIR>::STAGES * STAGE + 4 * P_STG_WARP + 1024 + 256;
};
static_assert(TcLayout<true>::SMEM <= 232448, "pair GEMM shared memory");

// The walk over tiles for G workers (CTAs or CTA pairs) and tiles TM rows
// high: T2 wide tiles in all, the first tmain (whole waves) as such, the rest
// split in halves, then the strip.
struct TileWalk {
  int mtiles, np2, tmain, nsplit, total;
};
__device__ __forceinline__ TileWalk tile_walk(int M, int N, int G, int TM) {
  TileWalk tw;
  tw.mtiles = (M + TM - 1) / TM;
  const int n128 = (N + PBN - 1) / PBN;
  tw.np2 = n128 / 2;
  const int t2 = tw.mtiles * tw.np2;
  tw.tmain = t2 / G * G;
  tw.nsplit = 2 * (t2 - tw.tmain);
  tw.total = tw.tmain + tw.nsplit + tw.mtiles * (n128 % 2);
  return tw;
}
__device__ __forceinline__ void wide_tile(int t, int mtiles, int np2, int TM, int& m0, int& n0) {
  const int per_group = PGROUP * np2;
  const int g = t / per_group, w = t % per_group;
  const int gm = min(PGROUP, mtiles - g * PGROUP);  // M-tiles in this group
  m0 = (g * PGROUP + w % gm) * TM;
  n0 = (w / gm) * WBN;
}
// tile t of the walk: its origin and width (256 or 128 columns)
__device__ __forceinline__ void p_tile(const TileWalk& tw, int t, int TM, int& m0, int& n0,
                                       int& wn) {
  if (t < tw.tmain) {
    wide_tile(t, tw.mtiles, tw.np2, TM, m0, n0);
    wn = WBN;
  } else if (t < tw.tmain + tw.nsplit) {
    const int s = t - tw.tmain;
    wide_tile(tw.tmain + s / 2, tw.mtiles, tw.np2, TM, m0, n0);
    n0 += (s & 1) * PBN;
    wn = PBN;
  } else {
    m0 = (t - tw.tmain - tw.nsplit) * TM;
    n0 = tw.np2 * WBN;
    wn = PBN;
  }
}

// LIN = 1: the linear module's epilogue (LinEpi) instead of storing C.
// PAIR: launched in clusters of two CTAs (see the head of the file).
template <int LIN, bool PAIR>
__global__ void __launch_bounds__(TC_THREADS, 1)
    k_gemm_tcp(const __grid_constant__ CUtensorMap ta_hi, const __grid_constant__ CUtensorMap ta_lo,
               const __grid_constant__ CUtensorMap tb_hi, const __grid_constant__ CUtensorMap tb_lo,
               float* __restrict__ C, int64_t ldc, int M, int N, int K, int a_k0, int b_k0,
               int n_off,
               const float* __restrict__ row_scale, float b_scale, int accumulate, int a_exact,
               const int* __restrict__ gate, const __grid_constant__ CUtensorMap tc_out,
               int use_reduce, int* status, const __grid_constant__ LinEpi le) {
  using Cfg = TcCfg<PAIR>;
  using Lay = TcLayout<PAIR>;
  constexpr int BK = Cfg::BK, NST = Cfg::STAGES, TM = Cfg::TM;
  constexpr int A_TILE = Lay::A_TILE, STAGE = Lay::STAGE;
  // (a gate read by both CTAs of a pair: they leave together, before any
  // cluster-wide step)
  if (gate != nullptr && *gate == 0) return;  // nothing to add
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stg_all = smem + NST * STAGE;
  uint64_t* full = (uint64_t*)(stg_all + 4 * P_STG_WARP);
  uint64_t* empty = full + NST;
  uint64_t* tm_full = empty + NST;
  uint64_t* tm_empty = tm_full + 2;
  uint32_t* tmem_slot = (uint32_t*)(tm_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // rank 0 of a pair issues the MMAs and owns the pair's full / TMEM-empty
  // barriers; both ranks own their empty and TMEM-full barriers
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int worker = PAIR ? (int)cluster_id_x() : (int)blockIdx.x;
  const int nworkers = PAIR ? (int)(gridDim.x / 2) : (int)gridDim.x;
  const TileWalk walk = tile_walk(M, N, nworkers, TM);
  const int tiles = walk.total;
  const int KT = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tm_full[b], 1);
      mbar_init(&tm_empty[b], PAIR ? 8 : 4);  // the epilogue warps (of both CTAs)
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(P_TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(P_TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // shared::cluster addresses of rank 0's barriers (the own ones on rank 0)
  const uint32_t full_r0 = PAIR ? map_to_rank(smem_u32(full), 0) : smem_u32(full);
  const uint32_t tm_empty_r0 = PAIR ? map_to_rank(smem_u32(tm_empty), 0) : smem_u32(tm_empty);

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer
    uint32_t it = 0;
    bool ok = true;
    for (int t = worker; t < tiles && ok; t += nworkers) {
      int m0, n0, wn;
      p_tile(walk, t, TM, m0, n0, wn);
      const int am0 = m0 + (int)rank * 128;              // this CTA's 128 rows of A
      const int brows = PAIR ? wn / 2 : wn;               // and its rows of B
      const int bn0 = n_off + n0 + (int)rank * brows;
      const int nbox = brows / Cfg::B_BOX;
      const uint32_t bytes = (uint32_t)((a_exact ? 1 : 2) * A_TILE + 2 * brows * BK * 2);
      for (int kt = 0; kt < KT; ++kt, ++it) {
        const int s = it % NST;
        if (it >= NST && !mbar_wait(&empty[s], (it / NST - 1) & 1)) {
          atomicOr(status, STATUS_TIMEOUT);
          ok = false;
          break;
        }
        uint8_t* base = smem + s * STAGE;
        const int kc_a = a_k0 + kt * BK, kc_b = b_k0 + kt * BK;
        if constexpr (PAIR) {
          // rank 0's full barrier counts both CTAs' bytes; rank 1's copies
          // complete on it from the peer
          const uint32_t fb = full_r0 + 8u * (uint32_t)s;
          if (rank == 0) mbar_expect_tx(&full[s], 2 * bytes);
          tma_load_2d_cg2(&ta_hi, fb, base, kc_a, am0);
          if (!a_exact) tma_load_2d_cg2(&ta_lo, fb, base + A_TILE, kc_a, am0);
          for (int b = 0; b < nbox; ++b) {
            uint8_t* bb = base + 2 * A_TILE + b * Cfg::B_BOX * BK * 2;
            tma_load_2d_cg2(&tb_hi, fb, bb, kc_b, bn0 + b * Cfg::B_BOX);
            tma_load_2d_cg2(&tb_lo, fb, bb + Cfg::B_HALF, kc_b, bn0 + b * Cfg::B_BOX);
          }
        } else {
          mbar_expect_tx(&full[s], bytes);
          tma_load_2d(&ta_hi, &full[s], base, kc_a, am0);
          if (!a_exact) tma_load_2d(&ta_lo, &full[s], base + A_TILE, kc_a, am0);
          for (int b = 0; b < nbox; ++b) {
            uint8_t* bb = base + 2 * A_TILE + b * Cfg::B_BOX * BK * 2;
            tma_load_2d(&tb_hi, &full[s], bb, kc_b, bn0 + b * Cfg::B_BOX);
            tma_load_2d(&tb_lo, &full[s], bb + Cfg::B_HALF, kc_b, bn0 + b * Cfg::B_BOX);
          }
        }
      }
    }
    // copies land before exit (rank 0's full barriers count both CTAs' copies;
    // rank 1 waits for rank 0 at the closing cluster barrier)
    if (rank == 0)
      for (uint32_t q = (it > (uint32_t)NST ? it - NST : 0); q < it; ++q)
        for (uint32_t i = 0; i < (1u << 25) && !mbar_try_wait(&full[q % NST], (q / NST) & 1); ++i)
          if (i > 256) __nanosleep(64);
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------------- MMA issuer
    uint32_t it = 0, tl = 0;
    bool ok = true;
    for (int t = worker; t < tiles && ok; t += nworkers, ++tl) {
      const int buf = tl & 1;
      int m0, n0, wn;
      p_tile(walk, t, TM, m0, n0, wn);
      const uint32_t idesc = wn == WBN ? Cfg::IDESC_W : Cfg::IDESC_N;
      if (tl >= 2 && !mbar_wait_cl(&tm_empty[buf], (tl / 2 - 1) & 1)) {
        atomicOr(status, STATUS_TIMEOUT);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)buf * WBN;
      for (int kt = 0; kt < KT; ++kt, ++it) {
        const int s = it % NST;
        if (!mbar_wait_cl(&full[s], (it / NST) & 1)) {
          atomicOr(status, STATUS_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_hi = smem_u32(smem + s * STAGE);
        const uint32_t a_lo = a_hi + A_TILE;
        const uint32_t b_hi = a_hi + 2 * A_TILE;  // this CTA's rows of B (the peer's at the same offset)
        const uint32_t b_lo = b_hi + Cfg::B_HALF;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint32_t off = kk * 32;  // 16 fp16 along a swizzled row
          const uint64_t dah = Cfg::desc(a_hi + off), dal = Cfg::desc(a_lo + off);
          const uint64_t dbh = Cfg::desc(b_hi + off), dbl = Cfg::desc(b_lo + off);
          const uint32_t acc0 = (kt | kk) != 0 ? 1u : 0u;
          if constexpr (PAIR) {
            umma_f16_cg2(d, dah, dbh, idesc, acc0);
            umma_f16_cg2(d, dah, dbl, idesc, 1u);
            if (!a_exact) umma_f16_cg2(d, dal, dbh, idesc, 1u);
          } else {
            umma_f16(d, dah, dbh, idesc, acc0);
            umma_f16(d, dah, dbl, idesc, 1u);
            if (!a_exact) umma_f16(d, dal, dbh, idesc, 1u);
          }
        }
        if constexpr (PAIR) {
          umma_commit_cg2(smem_u32(&empty[s]));                 // this CTA's stage
          umma_commit_cg2(map_to_rank(smem_u32(&empty[s]), 1));  // and the peer's
        } else {
          umma_commit(&empty[s]);
        }
      }
      if (ok) {
        if constexpr (PAIR) {
          umma_commit_cg2(smem_u32(&tm_full[buf]));
          umma_commit_cg2(map_to_rank(smem_u32(&tm_full[buf]), 1));
        } else {
          umma_commit(&tm_full[buf]);
        }
      }
    }
    for (uint32_t q = (tl > 2 ? tl - 2 : 0); q < tl; ++q)  // MMAs finish before TMEM is freed
      for (uint32_t i = 0; i < (1u << 25) && !mbar_try_wait(&tm_full[q & 1], (q / 2) & 1); ++i)
        if (i > 256) __nanosleep(64);
  } else if (warp >= 2) {
    // --------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may read
    uint8_t* stg0 = stg_all + (warp - 2) * P_STG_WARP;
    float* stage = reinterpret_cast<float*>(stg0);
    uint32_t tl = 0;
    int nb = 0;  // bulk reduce groups issued by this warp
    for (int t = worker; t < tiles; t += nworkers, ++tl) {
      const int buf = tl & 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait_cl(&tm_full[buf], (tl / 2) & 1));
      if (!ok) {
        if (lane == 0) atomicOr(status, STATUS_TIMEOUT);
        break;
      }
      tc_fence_after();
      int m0, n0, wn;
      p_tile(walk, t, TM, m0, n0, wn);
      m0 += (int)rank * 128;  // this CTA's rows of the tile
      const int row = m0 + q * 32 + lane;
      const float rs = (row < M) ? row_scale[row] * b_scale : 0.0f;
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)buf * WBN;
      // linear epilogue: this row's beta and gamma2, its M-step sums over the
      // tile's columns, and the operand scale b_scale 2^-e_bound (the row's
      // own 2^e_row cancels: p' = acc 2^e_row b_scale)
      float lb = 0.0f, lg2 = 0.0f, a2s = 0.0f, bsum = 0.0f;
      const float qk = LIN ? b_scale * ldexpf(1.0f, -le.e_bound) : 0.0f;
      if (LIN && row < M) {
        lb = (float)le.beta[row];
        lg2 = (float)le.gamma2[row];
      }
      for (int c0 = 0; c0 < wn; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tbase + (uint32_t)c0, v);
        if (c0 + 32 == wn) {  // the accumulator is read: hand it back to the MMAs
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (PAIR) mbar_arrive_cl(tm_empty_r0 + 8u * (uint32_t)buf);
            else mbar_arrive(&tm_empty[buf]);
          }
        }
        if (LIN && (c0 & (PBN - 1)) == 0) {  // a 128-column group starts: fresh sums
          a2s = 0.0f;
          bsum = 0.0f;
        }
        if (n0 + c0 >= N) {
          if (LIN && (c0 & (PBN - 1)) == PBN - 32 && row < M && n0 + c0 - (PBN - 32) < N)
            le.part[(int64_t)((n0 + c0) / PBN) * M + row] = make_float2(a2s, bsum);
          continue;
        }
        if constexpr (LIN) {
          // per element as the M-step states it, in fp32; columns past N are
          // written as zero (the operand's K padding)
          if (row < M) {
            uint32_t hv[16], lv[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              float qs[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int col = n0 + c0 + j + e;
                const float acc = __uint_as_float(v[j + e]);
                qs[e] = 0.0f;
                if (col < N) {
                  const float sl = __ldg(le.s32 + col);
                  const float pl = acc * rs;
                  const float u = sl * pl;
                  const float den = fmaf(lb * sl, sl, lg2);  // > 0
                  const float inv = __fdividef(1.0f, den);
                  const float f = lg2 * inv;
                  a2s += f;
                  bsum += fmaf(f * f * u, u, sl * sl * inv);
                  qs[e] = (le.full_rank ? -f : 1.0f - f) * acc * qk;
                  if (le.Uprime) le.Uprime[(int64_t)row * N + col] = (1.0f - f) * pl;
                }
              }
              const __half2 h = __floats2half2_rn(qs[0], qs[1]);
              const float2 hf = __half22float2(h);
              const __half2 l = __floats2half2_rn(qs[0] - hf.x, qs[1] - hf.y);
              hv[j / 2] = *reinterpret_cast<const uint32_t*>(&h);
              lv[j / 2] = *reinterpret_cast<const uint32_t*>(&l);
            }
            uint4* qh = reinterpret_cast<uint4*>(le.q_hi + (int64_t)row * le.ldq + n0 + c0);
            uint4* ql = reinterpret_cast<uint4*>(le.q_lo + (int64_t)row * le.ldq + n0 + c0);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              qh[k] = make_uint4(hv[4 * k], hv[4 * k + 1], hv[4 * k + 2], hv[4 * k + 3]);
              ql[k] = make_uint4(lv[4 * k], lv[4 * k + 1], lv[4 * k + 2], lv[4 * k + 3]);
            }
            if ((c0 & (PBN - 1)) == PBN - 32)  // the group's last chunk: its M-step sums
              le.part[(int64_t)((n0 + c0) / PBN) * M + row] = make_float2(a2s, bsum);
          }
          continue;
        }
        if (use_reduce) {
          // accumulate through the TMA unit: a 32 x 32 block in a
          // 128B-swizzled buffer (two per warp, alternating), tensor
          // reduce-add into C; L2 performs the read-modify-write
          uint8_t* sb = stg0 + (nb & 1) * 4096;
          if (lane == 0 && nb >= 2) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            float4 o = make_float4(__uint_as_float(v[4 * k]) * rs, __uint_as_float(v[4 * k + 1]) * rs,
                                   __uint_as_float(v[4 * k + 2]) * rs, __uint_as_float(v[4 * k + 3]) * rs);
            *reinterpret_cast<float4*>(sb + lane * 128 + ((k ^ (lane & 7)) * 16)) = o;
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) tma_reduce_add_2d(&tc_out, sb, n_off + n0 + c0, m0 + q * 32);
          ++nb;
        } else {
          // a 32 x 33 staging tile turns the lane-per-row TMEM layout into
          // row-contiguous, coalesced accesses
#pragma unroll
          for (int j = 0; j < 32; ++j) stage[lane * 33 + j] = __uint_as_float(v[j]) * rs;
          __syncwarp();
          const int col = n0 + c0 + lane;
          const int nrow = min(32, M - (m0 + q * 32));
          float* cbase = C + (int64_t)(m0 + q * 32) * ldc + n_off + col;
          if (col < N) {
            if (accumulate) {
              float prev[32];
#pragma unroll
              for (int rr = 0; rr < 32; ++rr)  // all loads in flight before any store
                prev[rr] = (rr < nrow) ? cbase[(int64_t)rr * ldc] : 0.0f;
#pragma unroll
              for (int rr = 0; rr < 32; ++rr)
                if (rr < nrow) cbase[(int64_t)rr * ldc] = prev[rr] + stage[rr * 33 + lane];
            } else {
#pragma unroll
              for (int rr = 0; rr < 32; ++rr)
                if (rr < nrow) cbase[(int64_t)rr * ldc] = stage[rr * 33 + lane];
            }
          }
          __syncwarp();
        }
      }
    }
    if (use_reduce && lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // no peer still reads this CTA's memory or barriers
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(P_TMEM_COLS));
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(P_TMEM_COLS));
  }
}

// --------------------------------------------------------------- splitting --
// Global-scale split of a fp32 matrix (plan-time operands V, V^T, H):
// dst = src * 2^-e as fp16 hi/lo, rows x ld (zero beyond K), e from max|src|.
__global__ void k_absmax(const float* __restrict__ x, int64_t count, unsigned* out) {
  float m = 0.0f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(x[i]));
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(out, __float_as_uint(m));  // m >= 0: order-preserving
}

__global__ void k_split_global(const float* __restrict__ src, int64_t rows, int64_t K,
                               int64_t ld, const unsigned* __restrict__ amax_bits,
                               __half* __restrict__ hi, __half* __restrict__ lo,
                               float* __restrict__ unscale) {
  const float amax = __uint_as_float(*amax_bits);
  int ex = 0;
  frexpf(amax, &ex);
  const int e = (amax > 0.0f) ? ex - 14 : 0;  // scaled |x| < 2^14
  const float down = ldexpf(1.0f, -e);
  if (blockIdx.x == 0 && threadIdx.x == 0) *unscale = ldexpf(1.0f, e);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows * ld;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / ld, c = i % ld;
    const float x = (c < K) ? src[r * K + c] * down : 0.0f;
    const __half h = __float2half_rn(x);
    hi[i] = h;
    lo[i] = __float2half_rn(x - __half2float(h));
  }
}

// ---------------------------------------------------- tensor-map encoding --
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_encode_mu;

mpq_status get_encoder() {
  std::lock_guard<std::mutex> lk(g_encode_mu);
  if (g_encode) return MPQ_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q{};
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
    return fail(MPQ_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return MPQ_OK;
}

bool g_smem_attr_set[64] = {};
int g_sms[64] = {};
int g_pairs[64] = {};

}  // namespace

namespace {
// K-major fp16 operand map: boxes of box_k x box_rows with the swizzle of the
// kernel that reads them (32 x rows with 64-byte, 64 x rows with 128-byte)
mpq_status encode_f16(CUtensorMap* tm, const void* base, int64_t inner, int64_t rows,
                      int64_t ld_elems, int box_k, int box_rows) {
  MPQ_TRY(get_encoder());
  if (((uintptr_t)base & 15) || (ld_elems * 2) % 16 || inner % 64 || rows < box_rows)
    return fail(MPQ_ERR_INVALID_ARG, "tensor map: misaligned operand");
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld_elems * 2)};
  cuuint32_t box[2] = {(cuuint32_t)box_k, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  const CUtensorMapSwizzle sw = box_k == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MPQ_ERR_CUDA, "cuTensorMapEncodeTiled failed with code " + std::to_string((int)r));
  return MPQ_OK;
}

// Maps of the pair kernel, encoded on first use over the operand's whole
// padded width (its zero K padding included) and kept: an encoding depends
// only on the key, so a key met again (memory reused with the same shape)
// maps the same bytes.
using PairKey = std::tuple<const void*, int64_t, int64_t, int>;
std::map<PairKey, CUtensorMap> g_pair_maps;
std::mutex g_pair_mu;

mpq_status pair_map(const void* base, int64_t rows_pad, int64_t ld, int box_rows,
                    CUtensorMap* out) {
  std::lock_guard<std::mutex> lk(g_pair_mu);
  const PairKey key{base, rows_pad, ld, box_rows};
  auto f = g_pair_maps.find(key);
  if (f != g_pair_maps.end()) {
    *out = f->second;
    return MPQ_OK;
  }
  if (g_pair_maps.size() > 4096) g_pair_maps.clear();
  MPQ_TRY(encode_f16(out, base, ld, rows_pad, ld, 64, box_rows));
  g_pair_maps.emplace(key, *out);
  return MPQ_OK;
}
}  // namespace

mpq_status make_tmap_f16(CUtensorMap* tm, const void* base, int64_t inner, int64_t rows,
                         int64_t ld_elems, int box_rows) {
  return encode_f16(tm, base, inner, rows, ld_elems, TcCfg<false>::BK, box_rows);
}

mpq_status make_tmap_f32_out(CUtensorMap* tm, const float* base, int64_t cols, int64_t rows,
                             int64_t ld_elems) {
  MPQ_TRY(get_encoder());
  if (((uintptr_t)base & 127) || (ld_elems * 4) % 16 || cols < 32 || rows < 32)
    return fail(MPQ_ERR_INVALID_ARG, "tensor map: misaligned output");
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld_elems * 4)};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MPQ_ERR_CUDA, "cuTensorMapEncodeTiled (fp32) failed with code " + std::to_string((int)r));
  return MPQ_OK;
}

mpq_status split_global(const float* src, int64_t rows, int64_t K, SplitOperand* dst,
                        cudaStream_t st) {
  unsigned* amax = nullptr;
  MPQ_CUDA(cudaMallocAsync(&amax, sizeof(unsigned), st));
  MPQ_CUDA(cudaMemsetAsync(amax, 0, sizeof(unsigned), st));
  {
    ProfScope ps_("k_absmax", st);
    k_absmax<<<(unsigned)std::min<int64_t>(cdiv(rows * K, 256), 148 * 8), 256, 0, st>>>(src, rows * K, amax);
  }
  {
    ProfScope ps_("k_split_global", st);
    k_split_global<<<(unsigned)std::min<int64_t>(cdiv(dst->rows_pad * dst->ld, 256), 148 * 16), 256, 0, st>>>(
        src, rows, K, dst->ld, amax, dst->hi, dst->lo, dst->unscale);
  }
  count_launch(2);
  MPQ_TRY(check_launch("split_global"));
  cudaFreeAsync(amax, st);
  return MPQ_OK;
}

mpq_status gemm_tc(const SplitOperand& A, const CUtensorMap& ta_hi, const CUtensorMap& ta_lo,
                   const SplitOperand& B, const CUtensorMap& tb_hi, const CUtensorMap& tb_lo,
                   float* C, int64_t ldc, int64_t M, int64_t N, int64_t K, float b_scale_host,
                   int* status, cudaStream_t st, const char* tag, const GemmOpts& o) {
  if (M <= 0 || N <= 0) return MPQ_OK;
  if (M > A.rows_pad || o.n0 < 0 || o.n0 + N > B.rows_pad || o.a_k0 < 0 || o.a_k0 + K > A.ld ||
      o.b_k0 < 0 || o.b_k0 + K > B.ld || o.a_k0 % 64 || o.b_k0 % 64)
    return fail(MPQ_ERR_INVALID_ARG, "gemm_tc: operand smaller than the problem");
  int dev = 0;
  MPQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(MPQ_ERR_CUDA, "gemm_tc: device index out of range");
  if (!g_smem_attr_set[dev]) {
    MPQ_CUDA(cudaFuncSetAttribute(k_gemm_tcp<0, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  TcLayout<false>::SMEM));
    MPQ_CUDA(cudaFuncSetAttribute(k_gemm_tcp<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  TcLayout<false>::SMEM));
    MPQ_CUDA(cudaFuncSetAttribute(k_gemm_tcp<0, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  TcLayout<true>::SMEM));
    MPQ_CUDA(cudaFuncSetAttribute(k_gemm_tcp<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  TcLayout<true>::SMEM));
    MPQ_CUDA(cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev));
    // CTA pairs that can be resident at once (0: no pair fits, single CTAs only)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (unsigned)g_sms[dev]);
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = TcLayout<true>::SMEM;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, k_gemm_tcp<0, true>, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      nc = 0;
    }
    g_pairs[dev] = nc;
    g_smem_attr_set[dev] = true;
  }
  if (o.c_reduce && !o.accumulate)
    return fail(MPQ_ERR_INVALID_ARG, "gemm_tc: reduce output needs accumulate");
  if (o.lin && (o.c_reduce || o.accumulate || o.n0 != 0 || o.lin->ldq < round_up(N, PBN) ||
                o.lin->ntiles != cdiv(N, PBN) || (o.lin->ldq % 8) != 0))
    return fail(MPQ_ERR_INVALID_ARG, "gemm_tc: linear epilogue needs a plain product over all N");
  const CUtensorMap& cmap = o.c_reduce ? *o.c_reduce : tb_hi;  // unused unless reducing
  const LinEpi le = o.lin ? *o.lin : LinEpi{};
  // CTA pairs for the long contractions; a short K (the CD updates, K = 128)
  // is better served by the single-CTA ring, whose four 48 KiB stages hold a
  // whole tile's K while the pair's three 64 KiB stages hold one and a half
  const bool pair = M > 128 && K >= 512 && g_pairs[dev] > 0;
  ProfScope ps_(tag, st);
  if (pair) {
    CUtensorMap pa_hi, pa_lo, pb_hi, pb_lo;
    MPQ_TRY(pair_map(A.hi, A.rows_pad, A.ld, 128, &pa_hi));
    MPQ_TRY(pair_map(A.lo, A.rows_pad, A.ld, 128, &pa_lo));
    MPQ_TRY(pair_map(B.hi, B.rows_pad, B.ld, TcCfg<true>::B_BOX, &pb_hi));
    MPQ_TRY(pair_map(B.lo, B.rows_pad, B.ld, TcCfg<true>::B_BOX, &pb_lo));
    const int64_t tiles = cdiv(M, 256) * cdiv(N, PBN);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (unsigned)std::min<int64_t>(tiles, g_pairs[dev]));
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = TcLayout<true>::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    MPQ_CUDA(cudaLaunchKernelEx(&cfg, o.lin ? k_gemm_tcp<1, true> : k_gemm_tcp<0, true>, pa_hi,
                                pa_lo, pb_hi, pb_lo, C, ldc, (int)M, (int)N, (int)K, (int)o.a_k0,
                                (int)o.b_k0, (int)o.n0, (const float*)A.row_unscale, b_scale_host,
                                o.accumulate ? 1 : 0, o.a_exact ? 1 : 0, o.gate, cmap,
                                o.c_reduce ? 1 : 0, status, le));
  } else {
    const int64_t tiles = cdiv(M, 128) * cdiv(N, PBN);
    const unsigned grid = (unsigned)std::min<int64_t>(tiles, g_sms[dev]);
    auto kern = o.lin ? k_gemm_tcp<1, false> : k_gemm_tcp<0, false>;
    kern<<<grid, TC_THREADS, TcLayout<false>::SMEM, st>>>(
        ta_hi, ta_lo, tb_hi, tb_lo, C, ldc, (int)M, (int)N, (int)K, (int)o.a_k0, (int)o.b_k0,
        (int)o.n0, A.row_unscale, b_scale_host, o.accumulate ? 1 : 0, o.a_exact ? 1 : 0, o.gate,
        cmap, o.c_reduce ? 1 : 0, status, le);
  }
  count_launch();
  return check_launch("k_gemm_tc");
}

}  // namespace mpq
