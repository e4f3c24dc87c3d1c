// Tensor-core GEMM for the fp32 contractions of the solve (sm_100a tcgen05).
//
//   C[M x N] = diag(row_scale) * (A_hi B_hi^T + A_hi B_lo^T + A_lo B_hi^T) * b_scale
//
// A and B are fp32 matrices stored as power-of-two-scaled fp16 pairs
// (x * 2^-e = hi + lo, hi = fp16(x * 2^-e), lo = fp16(x * 2^-e - hi)), so
// hi + lo carries ~22 significand bits and the three products recover an
// fp32-accurate contraction (the dropped lo*lo term is ~2^-22 relative).
// Both operands are K-major (K contiguous).  Persistent kernel, one CTA per
// SM walking 128 x 256 (or 128 x 128) tiles in K steps of 32: fp16 kind::f16
// MMAs with the fp32 accumulator in TMEM (two 256-column accumulators, so
// that the epilogue of one tile overlaps the MMAs of the next), operands
// staged by TMA (64-byte swizzle, no multicast) through a 4-stage mbarrier
// ring that runs across tiles.  Warp 0 issues TMA, warp 1 owns TMEM and issues the MMAs from one
// thread, warps 2-5 read the accumulators back (tcgen05.ld) and store C.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "mpq_internal.cuh"
#include "tc_ptx.cuh"

namespace mpq {
namespace {
using namespace tcx;

constexpr int BM = 128, BK = 32;
constexpr int A_TILE = BM * BK * 2;                 // 8 KiB
constexpr int TC_THREADS = 192;

// ------------------------------------------------------- persistent GEMM --
// One CTA per SM walks the output tiles: a 4-stage TMA ring of K = 32 slices
// (48 KiB per stage, so that three stages of loads are in flight while the
// MMAs read the fourth) runs across tiles, and two TMEM accumulators let the
// epilogue of one tile overlap the MMAs of the next.  Tiles are 128 x 256 (the three MMAs of a k-step then
// read 96 B of shared memory per cycle of tensor work, against 128 B, the
// whole shared-memory bandwidth, at 128 x 128) for as many full waves of
// the grid as the product holds; the 128 x 256 tiles left over for a last,
// partial wave run as two 128 x 128 tiles each, and an odd 128-column strip
// at the right edge as 128 x 128 tiles too.  Wide tiles go in groups of 8
// M-tiles (M fastest) so that the A and B panels in flight stay in L2.
constexpr int PBN = 128, WBN = 256, PSTAGES = 4, PGROUP = 8;
constexpr int P_B_TILE = PBN * BK * 2;                        // 8 KiB per 128 rows of B
constexpr int P_STAGE = 2 * A_TILE + 2 * 2 * P_B_TILE;        // 48 KiB
constexpr int P_STG_WARP = 8192;                              // epilogue staging per warp
constexpr int P_SMEM = PSTAGES * P_STAGE + 4 * P_STG_WARP + 1024 + 256;
constexpr uint32_t P_TMEM_COLS = 2 * WBN;
constexpr uint32_t P_IDESC_W = idesc_f16(BM, WBN), P_IDESC_N = idesc_f16(BM, PBN);

// The walk over tiles for a grid of G CTAs: T2 wide tiles in all, the first
// tmain (whole waves) as such, the rest split in halves, then the strip.
struct TileWalk {
  int mtiles, np2, tmain, nsplit, total;
};
__device__ __forceinline__ TileWalk tile_walk(int M, int N, int G) {
  TileWalk tw;
  tw.mtiles = (M + BM - 1) / BM;
  const int n128 = (N + PBN - 1) / PBN;
  tw.np2 = n128 / 2;
  const int t2 = tw.mtiles * tw.np2;
  tw.tmain = t2 / G * G;
  tw.nsplit = 2 * (t2 - tw.tmain);
  tw.total = tw.tmain + tw.nsplit + tw.mtiles * (n128 % 2);
  return tw;
}
__device__ __forceinline__ void wide_tile(int t, int mtiles, int np2, int& m0, int& n0) {
  const int per_group = PGROUP * np2;
  const int g = t / per_group, w = t % per_group;
  const int gm = min(PGROUP, mtiles - g * PGROUP);  // M-tiles in this group
  m0 = (g * PGROUP + w % gm) * BM;
  n0 = (w / gm) * WBN;
}
// tile t of the walk: its origin and width (256 or 128 columns)
__device__ __forceinline__ void p_tile(const TileWalk& tw, int t, int& m0, int& n0, int& wn) {
  if (t < tw.tmain) {
    wide_tile(t, tw.mtiles, tw.np2, m0, n0);
    wn = WBN;
  } else if (t < tw.tmain + tw.nsplit) {
    const int s = t - tw.tmain;
    wide_tile(tw.tmain + s / 2, tw.mtiles, tw.np2, m0, n0);
    n0 += (s & 1) * PBN;
    wn = PBN;
  } else {
    m0 = (t - tw.tmain - tw.nsplit) * BM;
    n0 = tw.np2 * WBN;
    wn = PBN;
  }
}

// LIN = 1: the linear module's epilogue (LinEpi) instead of storing C.
template <int LIN>
__global__ void __launch_bounds__(TC_THREADS, 1)
    k_gemm_tcp(const __grid_constant__ CUtensorMap ta_hi, const __grid_constant__ CUtensorMap ta_lo,
               const __grid_constant__ CUtensorMap tb_hi, const __grid_constant__ CUtensorMap tb_lo,
               float* __restrict__ C, int64_t ldc, int M, int N, int K, int a_k0, int b_k0,
               int n_off,
               const float* __restrict__ row_scale, float b_scale, int accumulate, int a_exact,
               const int* __restrict__ gate, const __grid_constant__ CUtensorMap tc_out,
               int use_reduce, int* status, const __grid_constant__ LinEpi le) {
  if (gate != nullptr && *gate == 0) return;  // nothing to add
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stg_all = smem + PSTAGES * P_STAGE;
  uint64_t* full = (uint64_t*)(stg_all + 4 * P_STG_WARP);
  uint64_t* empty = full + PSTAGES;
  uint64_t* tm_full = empty + PSTAGES;
  uint64_t* tm_empty = tm_full + 2;
  uint32_t* tmem_slot = (uint32_t*)(tm_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const TileWalk walk = tile_walk(M, N, gridDim.x);
  const int tiles = walk.total;
  const int KT = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tm_full[b], 1);
      mbar_init(&tm_empty[b], 4);  // the four epilogue warps
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(P_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer
    uint32_t it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      int m0, n0, wn;
      p_tile(walk, t, m0, n0, wn);
      const int nb = wn / PBN;  // 128-row boxes of B
      for (int kt = 0; kt < KT; ++kt, ++it) {
        const int s = it % PSTAGES;
        if (it >= PSTAGES && !mbar_wait(&empty[s], (it / PSTAGES - 1) & 1)) {
          atomicOr(status, STATUS_TIMEOUT);
          ok = false;
          break;
        }
        uint8_t* base = smem + s * P_STAGE;
        mbar_expect_tx(&full[s], (a_exact ? A_TILE : 2 * A_TILE) + 2 * nb * P_B_TILE);
        tma_load_2d(&ta_hi, &full[s], base, a_k0 + kt * BK, m0);
        if (!a_exact) tma_load_2d(&ta_lo, &full[s], base + A_TILE, a_k0 + kt * BK, m0);
        for (int b = 0; b < nb; ++b) {
          tma_load_2d(&tb_hi, &full[s], base + 2 * A_TILE + b * P_B_TILE, b_k0 + kt * BK,
                      n_off + n0 + b * PBN);
          tma_load_2d(&tb_lo, &full[s], base + 2 * A_TILE + (2 + b) * P_B_TILE, b_k0 + kt * BK,
                      n_off + n0 + b * PBN);
        }
      }
    }
    for (uint32_t q = (it > PSTAGES ? it - PSTAGES : 0); q < it; ++q)  // copies land before exit
      for (uint32_t i = 0; i < (1u << 25) && !mbar_try_wait(&full[q % PSTAGES], (q / PSTAGES) & 1); ++i)
        if (i > 256) __nanosleep(64);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------- MMA issuer
    uint32_t it = 0, tl = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tl) {
      const int buf = tl & 1;
      int m0, n0, wn;
      p_tile(walk, t, m0, n0, wn);
      const uint32_t idesc = wn == WBN ? P_IDESC_W : P_IDESC_N;
      if (tl >= 2 && !mbar_wait(&tm_empty[buf], (tl / 2 - 1) & 1)) {
        atomicOr(status, STATUS_TIMEOUT);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)buf * WBN;
      for (int kt = 0; kt < KT; ++kt, ++it) {
        const int s = it % PSTAGES;
        if (!mbar_wait(&full[s], (it / PSTAGES) & 1)) {
          atomicOr(status, STATUS_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_hi = smem_u32(smem + s * P_STAGE);
        const uint32_t a_lo = a_hi + A_TILE;
        const uint32_t b_hi = a_hi + 2 * A_TILE;     // wn rows: one or two 128-row boxes
        const uint32_t b_lo = b_hi + 2 * P_B_TILE;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint32_t off = kk * 32;
          const uint64_t dah = sw64_desc(a_hi + off), dal = sw64_desc(a_lo + off);
          const uint64_t dbh = sw64_desc(b_hi + off), dbl = sw64_desc(b_lo + off);
          umma_f16(d, dah, dbh, idesc, (kt | kk) != 0 ? 1u : 0u);
          umma_f16(d, dah, dbl, idesc, 1u);
          if (!a_exact) umma_f16(d, dal, dbh, idesc, 1u);
        }
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(&tm_full[buf]);
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
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tl) {
      const int buf = tl & 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tm_full[buf], (tl / 2) & 1));
      if (!ok) {
        if (lane == 0) atomicOr(status, STATUS_TIMEOUT);
        break;
      }
      tc_fence_after();
      int m0, n0, wn;
      p_tile(walk, t, m0, n0, wn);
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
          if (lane == 0) mbar_arrive(&tm_empty[buf]);
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
  if (warp == 1) {
    tc_fence_after();
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

}  // namespace

mpq_status make_tmap_f16(CUtensorMap* tm, const void* base, int64_t inner, int64_t rows,
                         int64_t ld_elems, int box_rows) {
  MPQ_TRY(get_encoder());
  if (((uintptr_t)base & 15) || (ld_elems * 2) % 16 || inner % 64 || rows < box_rows)
    return fail(MPQ_ERR_INVALID_ARG, "tensor map: misaligned operand");
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld_elems * 2)};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MPQ_ERR_CUDA, "cuTensorMapEncodeTiled failed with code " + std::to_string((int)r));
  return MPQ_OK;
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
  if (dev >= 0 && dev < 64 && !g_smem_attr_set[dev]) {
    MPQ_CUDA(cudaFuncSetAttribute(k_gemm_tcp<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM));
    MPQ_CUDA(cudaFuncSetAttribute(k_gemm_tcp<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM));
    MPQ_CUDA(cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev));
    g_smem_attr_set[dev] = true;
  }
  if (o.c_reduce && !o.accumulate)
    return fail(MPQ_ERR_INVALID_ARG, "gemm_tc: reduce output needs accumulate");
  if (o.lin && (o.c_reduce || o.accumulate || o.n0 != 0 || o.lin->ldq < round_up(N, PBN) ||
                o.lin->ntiles != cdiv(N, PBN) || (o.lin->ldq % 8) != 0))
    return fail(MPQ_ERR_INVALID_ARG, "gemm_tc: linear epilogue needs a plain product over all N");
  const int64_t tiles = cdiv(M, BM) * cdiv(N, PBN);
  const unsigned grid = (unsigned)std::min<int64_t>(tiles, dev < 64 ? g_sms[dev] : 148);
  const CUtensorMap& cmap = o.c_reduce ? *o.c_reduce : tb_hi;  // unused unless reducing
  {
    ProfScope ps_(tag, st);
    const LinEpi le = o.lin ? *o.lin : LinEpi{};
    auto kern = o.lin ? k_gemm_tcp<1> : k_gemm_tcp<0>;
    kern<<<grid, TC_THREADS, P_SMEM, st>>>(
        ta_hi, ta_lo, tb_hi, tb_lo, C, ldc, (int)M, (int)N, (int)K, (int)o.a_k0, (int)o.b_k0,
        (int)o.n0, A.row_unscale,
        b_scale_host, o.accumulate ? 1 : 0, o.a_exact ? 1 : 0, o.gate, cmap, o.c_reduce ? 1 : 0,
        status, le);
  }
  count_launch();
  return check_launch("k_gemm_tc");
}

}  // namespace mpq
