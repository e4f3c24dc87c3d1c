// Exact block coordinate descent in the metric H = T^T T.
//
// Source: "MPQ: A Message-Passing View of Post-Training Quantization"
// (papernotes.org note), Key design 3: for block b, minimising
// 1/2 |u - T_b (c - x_b)|^2 over c in C_b (equivalently the Mahalanobis
// nearest codeword to mu_b = x_b + G_b^-1 T_b^T u in G_b = T_b^T T_b);
// hyper-parameter section: at most S_CD sweeps, stop after a sweep in which
// no block changes.  With the gradient h = T^T u = H (w - x) the energy
// change of moving block b to c is  dE = -delta^T h_b + 1/2 delta^T G_b delta,
// delta = c - x_b, and accepting it updates h <- h - H[:, b] delta.
#include <math.h>

#include <type_traits>

#include "mpq_internal.cuh"

namespace mpq {
namespace {

// ------------------------------------------------------------------ d = 1 --
// A sweep visits the columns in tiles of CD_TILE.  For tile j the decide
// kernel runs one warp per row; lane l keeps, in registers, the state of the
// tile's columns l, l + 32, l + 64, l + 96 (gradient, level, and the two
// per-column constants of the energy change).  The warp takes the tile 32
// columns at a time: all live lanes evaluate their column, which is exact up
// to the first lane that accepts a change; the warp commits that change,
// updates the gradient of the later columns with the row of H, and resumes
// right after it -- identical to visiting the columns one by one.  The
// tile's changes leave as Delta/scale (small integers, exact in fp16) in the
// A operand of a tensor-core update  h += (-scale) Delta H[tile, :]  over all
// columns, which also reproduces the in-tile updates for the next tile and
// the next sweep.
//
// Tiles go in groups of CD1_GROUP.  The gradient in memory is brought up to
// date once per group (one GEMM with K = the group's width over the panel);
// within a group, tile k starts from that gradient and first applies the
// changes of the group's tiles before it to its own columns, in registers,
// from their Delta rows and the blocks H[earlier tile, this tile] staged in
// shared memory.
constexpr int CD1_WARPS = 32;  // at most; the launch takes as many as spread the rows evenly
constexpr int CD1_SLOTS = CD_TILE / 32;
constexpr int CD1_GROUP = 3;   // (1 + earlier tiles) H blocks of 64 KiB fit in shared memory
constexpr int CD1_BLOCK = CD_TILE * CD_TILE * 4;
constexpr int CD1_SMEM = CD1_BLOCK + CD_TILE * 4;
constexpr int CD1_SMEM_MAX = CD1_SMEM + (CD1_GROUP - 1) * CD1_BLOCK;

// 4- and 16-byte asynchronous copies global -> shared; bytes past src_bytes
// are filled with zeros
__device__ __forceinline__ void cp_async4(float* dst, const float* src, int src_bytes) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(d), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async16(float* dst, const float* src, int src_bytes) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(src_bytes)
               : "memory");
}

// H[r0 .. r0+rw, c0 .. c0+cw] into a zero-padded CD_TILE x CD_TILE shared
// block: 16-byte copies when the rows of H are 16-byte aligned (n % 4 == 0;
// r0 and c0 are multiples of 128), else 4-byte copies.  The copies are
// committed, not waited for.
__device__ __forceinline__ void load_h_block(float* sH, const float* H, int64_t n, int64_t r0,
                                             int rw, int64_t c0, int cw) {
  if ((n & 3) == 0) {
    constexpr int CH = CD_TILE / 4;  // 16-byte chunks per row
    for (int e = threadIdx.x; e < CD_TILE * CH; e += blockDim.x) {
      const int i = e / CH, j = 4 * (e % CH);
      const int bytes = i < rw ? 4 * max(0, min(4, cw - j)) : 0;
      cp_async16(sH + i * CD_TILE + j, bytes ? H + (r0 + i) * n + c0 + j : H, bytes);
    }
  } else {
    for (int e = threadIdx.x; e < CD_TILE * CD_TILE; e += blockDim.x) {
      const int i = e / CD_TILE, j = e % CD_TILE;
      const bool in = i < rw && j < cw;
      cp_async4(sH + e, in ? H + (r0 + i) * n + c0 + j : H, in ? 4 : 0);
    }
  }
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

// gk: this tile's place in its group (the gk tiles before it, full width,
// end at t0; their Delta rows end where this tile's begins)
__global__ void __launch_bounds__(CD1_WARPS * 32, 1)
    k_cd_tile_decide(int64_t m, int64_t n, int L, int64_t t0, int tw, int gk,
                     const float* __restrict__ scale, int ng, int gi,
                     const float* __restrict__ sref, const float* __restrict__ H,
                     uint16_t* __restrict__ idx, const float* __restrict__ h, int64_t ldh,
                     int sweeps, int sw,
                     int32_t* __restrict__ changes, __half* __restrict__ dhi,
                     __half* __restrict__ dlo, int64_t lda, float* __restrict__ d_unscale,
                     int* __restrict__ tile_flag, int* __restrict__ panel_flag,
                     const int32_t* __restrict__ skip) {
  extern __shared__ float cd_smem[];
  float* sH = cd_smem;                   // H[tile, tile], zero outside tw x tw
  float* s_rg = sH + CD_TILE * CD_TILE;  // 1 / H_jj (0 where H_jj <= 0)
  float* sHp = s_rg + CD_TILE;           // gk blocks H[earlier tile p, tile]
  load_h_block(sH, H, n, t0, tw, t0, tw);
  for (int p = 0; p < gk; ++p)
    load_h_block(sHp + p * CD_TILE * CD_TILE, H, n, t0 - (int64_t)(gk - p) * CD_TILE, CD_TILE, t0,
                 tw);
  // the row's gradient and levels in the tile travel while the H blocks do
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + wid;
  float h_in[CD1_SLOTS], k_in[CD1_SLOTS];
#pragma unroll
  for (int q = 0; q < CD1_SLOTS; ++q) {
    const int col = 32 * q + lane;
    const bool in = row < m && col < tw;
    h_in[q] = in ? h[row * ldh + t0 + col] : 0.0f;
    k_in[q] = in ? (float)idx[row * n + t0 + col] : 0.0f;
  }
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
  __syncthreads();
  bool pos = true;  // every diagonal entry of the tile positive
  for (int j = threadIdx.x; j < CD_TILE; j += blockDim.x) {
    const float gj = sH[j * CD_TILE + j];
    s_rg[j] = gj > 0.0f ? 1.0f / gj : 0.0f;
    if (j < tw && !(gj > 0.0f)) pos = false;
  }
  pos = __syncthreads_and(pos);
  if (row >= m) return;
  __half* drow_hi = dhi + row * lda;
  __half* drow_lo = dlo + row * lda;
  // the tile's grid: the row's, or its group's (a group holds whole tiles).
  // With group-wise grids the tiles of a panel have different scales, so
  // Delta leaves as (k_new - k_old) scale / sref, an fp16 pair, against the
  // row's reference scale sref; otherwise as the exact level difference.
  const float sc = scale[row * ng + gi];
  const float dsc = sref ? sc / sref[row] : 1.0f;
  if (lane == 0) d_unscale[row] = sref ? -sref[row] : -sc;
  uint16_t* ir = idx + row * n + t0;
  // a row stops after a sweep without change, and a skipped row never starts
  // (its Delta row stays zero)
  if ((sw > 0 && changes[row * sweeps + sw - 1] == 0) || (skip && skip[row])) {
    for (int i = lane; i < CD_TILE; i += 32) {
      drow_hi[i] = __float2half_rn(0.0f);
      drow_lo[i] = __float2half_rn(0.0f);
    }
    return;
  }
  // Energy change of level k in index units u = k - kc (dE = u (a u - hs),
  // hs = scale h, a = scale^2 H_jj / 2): a parabola in k with its vertex at
  // kcont = kc + hs rq, rq = 1 / (scale^2 H_jj).  The best level is the one
  // nearest kcont (the lower on an exact half: lowest index on ties), clamped
  // to the grid; a reciprocal instead of a division moves kcont by ulps,
  // which changes the choice only between levels whose energies tie to
  // rounding.  With H_jj <= 0 the candidates are the grid ends.
  const float s2 = sc * sc, is2 = 1.0f / s2, Lm1 = (float)(L - 1);
  float hs[CD1_SLOTS], kc[CD1_SLOTS], a[CD1_SLOTS], rq[CD1_SLOTS];
#pragma unroll
  for (int q = 0; q < CD1_SLOTS; ++q) {
    const int col = 32 * q + lane;
    hs[q] = sc * h_in[q];
    kc[q] = k_in[q];
    a[q] = 0.5f * s2 * sH[col * CD_TILE + col];
    rq[q] = is2 * s_rg[col];
  }
  // the changes of the group's earlier tiles: h += du sum_j Delta_j H[j, .]
  // (Delta_j = hi + lo as the update GEMM reads it, du = -scale, or -sref
  // with group-wise grids), scaled like hs
  if (gk > 0) {
    const float f0 = sc * (sref ? -sref[row] : -sc);
    for (int p = 0; p < gk; ++p) {
      const __half* ph = drow_hi - (int64_t)(gk - p) * CD_TILE;
      const __half* pl = drow_lo - (int64_t)(gk - p) * CD_TILE;
      const float* Hp = sHp + p * CD_TILE * CD_TILE + lane;
#pragma unroll
      for (int q = 0; q < CD1_SLOTS; ++q) {
        const float av = __half2float(ph[32 * q + lane]) + __half2float(pl[32 * q + lane]);
        unsigned mk = __ballot_sync(0xffffffffu, av != 0.0f);
        while (mk) {
          const int l = __ffs(mk) - 1;
          mk &= mk - 1u;
          const float f = f0 * __shfl_sync(0xffffffffu, av, l);
          const float* Hj = Hp + (32 * q + l) * CD_TILE;
#pragma unroll
          for (int qq = 0; qq < CD1_SLOTS; ++qq) hs[qq] = fmaf(Hj[32 * qq], f, hs[qq]);
        }
      }
    }
  }
  auto sweep_tile = [&](auto all_pos) -> int {
    constexpr bool POS = decltype(all_pos)::value;
    int nchg = 0;
#pragma unroll
    for (int q = 0; q < CD1_SLOTS; ++q) {
      if (32 * q >= tw) break;
      unsigned live = tw - 32 * q >= 32 ? 0xffffffffu : (1u << (tw - 32 * q)) - 1u;
      while (true) {
        float kn, e;
        {
          const float kcont = fmaf(hs[q], rq[q], kc[q]);
          kn = fminf(fmaxf(ceil_small(kcont - 0.5f), 0.0f), Lm1);
          const float u = kn - kc[q];
          e = u * fmaf(a[q], u, -hs[q]);
        }
        if (!POS && !(a[q] > 0.0f)) {
          const float u0 = -kc[q], u1 = Lm1 - kc[q];
          const float e0 = u0 * fmaf(a[q], u0, -hs[q]), e1 = u1 * fmaf(a[q], u1, -hs[q]);
          kn = kc[q];
          e = 0.0f;  // staying put
          if (e0 < e) {
            e = e0;
            kn = 0.0f;
          }
          if (e1 < e) {
            e = e1;
            kn = Lm1;
          }
        }
        const unsigned mask = __ballot_sync(0xffffffffu, e < 0.0f) & live;
        if (mask == 0u) break;
        const int first = __ffs(mask) - 1;
        const float u = __shfl_sync(0xffffffffu, kn - kc[q], first);
        if (lane == first) kc[q] = kn;
        live &= ~((2u << first) - 1u);  // this column and the ones before it are done
        ++nchg;
        // gradient of the later columns: hs <- hs - scale^2 H[jj, :] u
        const float* Hj = sH + (32 * q + first) * CD_TILE + lane;
        const float s2u = s2 * u;
#pragma unroll
        for (int qq = q; qq < CD1_SLOTS; ++qq) hs[qq] = fmaf(-Hj[32 * qq], s2u, hs[qq]);
      }
    }
    return nchg;
  };
  const int ntile = pos ? sweep_tile(std::true_type{}) : sweep_tile(std::false_type{});
  // levels and Delta/scale = k_new - k_old (zero outside the tile's columns)
#pragma unroll
  for (int q = 0; q < CD1_SLOTS; ++q) {
    const int col = 32 * q + lane;
    float dk = 0.0f;
    if (col < tw) {
      const int knew = (int)kc[q];
      dk = (float)(knew - (int)k_in[q]);
      ir[col] = (uint16_t)knew;
    }
    const float dv = dk * dsc;  // exact when dsc = 1
    const __half dh = __float2half_rn(dv);
    drow_hi[col] = dh;
    drow_lo[col] = __float2half_rn(dv - __half2float(dh));
  }
  if (lane == 0 && ntile > 0) {
    changes[row * sweeps + sw] += ntile;
    *tile_flag = 1;  // gates of the updates: some row changed
    *panel_flag = 1;
  }
}

// ------------------------------------------------------------------ d = 8 --
// Per block step b (all rows together): score(c) = qtab_b(c) - c . g',
// with qtab_b(c) = 1/2 c^T G_b c, g' = (h_b + G_b x_b)/scale; the energy
// change of codeword c is scale^2 (score(c) - score(c_cur)).
// A sweep visits the blocks in tiles of CD_TILE columns (16 blocks), like the
// scalar path: within a tile the gradient lives in a tile-local copy hl that
// the apply step updates with H[tile, block]; the tile's changes leave as
// Delta/scale = c_new - c_old in the A operand of the tensor-core update
// h += (-scale) Delta H[tile, :] over all columns, run once per tile.
// Kernel A: partial argmin over a chunk of codewords for a tile of rows.
// Kernel B: combine chunks, accept if strictly better, update idx, hl, Delta.
constexpr int CD8_ROWS = 256;   // rows per eval CTA (8 warps x 4 groups of 8 rows)
constexpr int CD8_CHUNK = 1024; // codewords per eval CTA
constexpr int CD8_APPLY_WARPS = 16;

__device__ __forceinline__ bool row_active(const int32_t* changes, const int32_t* skip,
                                           int64_t row, int sweeps, int sw) {
  return (sw == 0 || changes[row * sweeps + sw - 1] > 0) && !(skip && skip[row]);
}

// g' for one row at block b from the block's 8 gradient entries hb; G_b and
// x_b in weight units.
__device__ __forceinline__ void block_gradient(const float* __restrict__ H, int64_t n,
                                               const float* __restrict__ hb,
                                               const float* __restrict__ cb, int kcur,
                                               float sc, int64_t b, float* gout) {
  float x[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) x[j] = sc * cb[(int64_t)kcur * 8 + j];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float g = hb[i];
    const float* Hi = H + (8 * b + i) * n + 8 * b;
#pragma unroll
    for (int j = 0; j < 8; ++j) g = fmaf(Hi[j], x[j], g);
    gout[i] = g / sc;
  }
}

// the block's current gradient: h itself at the first block of a tile, else
// the tile-local copy (h at the tile start plus the tile's own updates)
__device__ __forceinline__ const float* block_h(const float* h, int64_t ldh, const float* hl,
                                                int64_t row, int64_t b, int64_t t0) {
  return (8 * b == t0) ? h + row * ldh + 8 * b : hl + row * CD_TILE + (8 * b - t0);
}

__global__ void __launch_bounds__(256)
    k_cd_vec_eval(int64_t m, int64_t n, int K, int64_t b, int64_t t0, const float* __restrict__ cb,
                  const float* __restrict__ qtab, const float* __restrict__ H,
                  const float* __restrict__ scale, const uint16_t* __restrict__ idx,
                  const float* __restrict__ h, int64_t ldh, const float* __restrict__ hl,
                  int sweeps, int sw, const int32_t* __restrict__ changes,
                  const int32_t* __restrict__ skip, float* __restrict__ part_val,
                  int* __restrict__ part_idx, int nchunks) {
  __shared__ float scb[8][CD8_CHUNK];  // transposed: lanes read consecutive codewords
  __shared__ float sq[CD8_CHUNK];
  __shared__ float sg[CD8_ROWS][8];
  __shared__ int sact[CD8_ROWS / 8];   // row groups with an active row
  const int64_t B = n / 8;
  const int chunk = blockIdx.x;
  const int64_t r0 = (int64_t)blockIdx.y * CD8_ROWS;
  const int c0 = chunk * CD8_CHUNK;
  const int cn = min(CD8_CHUNK, K - c0);
  for (int e = threadIdx.x; e < cn * 8; e += blockDim.x) scb[e % 8][e / 8] = cb[(int64_t)c0 * 8 + e];
  for (int e = threadIdx.x; e < cn; e += blockDim.x) sq[e] = qtab[b * K + c0 + e];
  if (threadIdx.x < CD8_ROWS / 8) sact[threadIdx.x] = 0;
  __syncthreads();
  for (int rl = threadIdx.x; rl < CD8_ROWS; rl += blockDim.x) {
    const int64_t row = r0 + rl;
    const bool act = row < m && row_active(changes, skip, row, sweeps, sw);
    if (act) {
      float g[8];
      block_gradient(H, n, block_h(h, ldh, hl, row, b, t0), cb, idx[row * B + b], scale[row], b, g);
#pragma unroll
      for (int i = 0; i < 8; ++i) sg[rl][i] = g[i];
      sact[rl / 8] = 1;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) sg[rl][i] = 0.0f;
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  // warp w takes row groups w, w + 8, ... of 8 rows; the lanes split the codewords
  for (int grp = w; grp < CD8_ROWS / 8; grp += 8) {
    if (!sact[grp]) continue;
    float g[8][8];
#pragma unroll
    for (int rr = 0; rr < 8; ++rr)
#pragma unroll
      for (int i = 0; i < 8; ++i) g[rr][i] = sg[8 * grp + rr][i];
    float best[8];
    int bidx[8];
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      best[rr] = INFINITY;
      bidx[rr] = 0x7fffffff;
    }
    for (int c = lane; c < cn; c += 32) {
      float cv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) cv[i] = scb[i][c];
      const float q = sq[c];
#pragma unroll
      for (int rr = 0; rr < 8; ++rr) {
        float s = q;
#pragma unroll
        for (int i = 0; i < 8; ++i) s = fmaf(-cv[i], g[rr][i], s);
        if (s < best[rr]) {
          best[rr] = s;
          bidx[rr] = c0 + c;
        }
      }
    }
    // warp argmin per row, lowest index on ties
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      float v = best[rr];
      int k = bidx[rr];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
        const int k2 = __shfl_xor_sync(0xffffffffu, k, o);
        if (v2 < v || (v2 == v && k2 < k)) {
          v = v2;
          k = k2;
        }
      }
      const int64_t row = r0 + 8 * grp + rr;
      if (lane == 0 && row < m) {
        part_val[row * nchunks + chunk] = v;
        part_idx[row * nchunks + chunk] = k;
      }
    }
  }
}

// One warp per row.  At the first block of a tile every row (active or not)
// clears its Delta row and copies h[tile] into hl.
__global__ void __launch_bounds__(CD8_APPLY_WARPS * 32)
    k_cd_vec_apply(int64_t m, int64_t n, int K, int64_t b, int64_t t0, int tw,
                   const float* __restrict__ cb, const float* __restrict__ qtab,
                   const float* __restrict__ H, const float* __restrict__ scale,
                   uint16_t* __restrict__ idx, const float* __restrict__ h, int64_t ldh,
                   float* __restrict__ hl, int sweeps, int sw, int32_t* __restrict__ changes,
                   const float* __restrict__ part_val, const int* __restrict__ part_idx,
                   int nchunks, __half* __restrict__ dhi, __half* __restrict__ dlo, int64_t lda,
                   float* __restrict__ d_unscale, int* __restrict__ tile_flag,
                   int* __restrict__ panel_flag, const int32_t* __restrict__ skip) {
  __shared__ float sHb[CD_TILE][8];  // H[tile, block b]
  const int64_t B = n / 8;
  const bool first = 8 * b == t0;
  for (int e = threadIdx.x; e < tw * 8; e += blockDim.x)
    sHb[e / 8][e % 8] = H[(t0 + e / 8) * n + 8 * b + e % 8];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * CD8_APPLY_WARPS + (threadIdx.x >> 5);
  if (row >= m) return;
  float* hlr = hl + row * CD_TILE;
  const float sc = scale[row];
  if (first) {
    for (int i = lane; i < CD_TILE; i += 32) {
      dhi[row * lda + i] = __float2half_rn(0.0f);
      dlo[row * lda + i] = __float2half_rn(0.0f);
      hlr[i] = i < tw ? h[row * ldh + t0 + i] : 0.0f;
    }
    if (lane == 0) d_unscale[row] = -sc;
  }
  if (!row_active(changes, skip, row, sweeps, sw)) return;
  // combine the chunk minima (lowest index on ties)
  float v = INFINITY;
  int k = 0x7fffffff;
  for (int c = lane; c < nchunks; c += 32) {
    const float v2 = part_val[row * nchunks + c];
    const int k2 = part_idx[row * nchunks + c];
    if (v2 < v || (v2 == v && k2 < k)) {
      v = v2;
      k = k2;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
    const int k2 = __shfl_xor_sync(0xffffffffu, k, o);
    if (v2 < v || (v2 == v && k2 < k)) {
      v = v2;
      k = k2;
    }
  }
  __syncwarp();  // hl of the first block is written before it is read
  const int kcur = idx[row * B + b];
  float g[8];
  block_gradient(H, n, hlr + (8 * b - t0), cb, kcur, sc, b, g);
  // the candidate's score is recomputed here in the same fp32 arithmetic as
  // the current codeword's, so that acceptance (strictly lower) does not
  // depend on how the scan evaluated it
  if (k < 0 || k >= K || k == kcur) return;
  float scur = qtab[b * K + kcur], snew = qtab[b * K + k];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    scur = fmaf(-cb[(int64_t)kcur * 8 + i], g[i], scur);
    snew = fmaf(-cb[(int64_t)k * 8 + i], g[i], snew);
  }
  if (!(snew < scur)) return;
  float dd[8], dl[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    dd[j] = cb[(int64_t)k * 8 + j] - cb[(int64_t)kcur * 8 + j];
    dl[j] = sc * dd[j];
  }
  if (lane == 0) {
    idx[row * B + b] = (uint16_t)k;
    changes[row * sweeps + sw] += 1;
    *tile_flag = 1;  // gates of the updates: some row changed
    *panel_flag = 1;
  }
  if (lane < 8) {  // Delta / scale as an fp16 pair (exact for lattice codebooks)
    const __half hi = __float2half_rn(dd[lane]);
    dhi[row * lda + 8 * b - t0 + lane] = hi;
    dlo[row * lda + 8 * b - t0 + lane] = __float2half_rn(dd[lane] - __half2float(hi));
  }
  for (int i = lane; i < tw; i += 32) {
    float acc = hlr[i];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc = fmaf(-sHb[i][j], dl[j], acc);
    hlr[i] = acc;
  }
}

// per-row maximum of the group scales (the reference scale of grouped Delta)
__global__ void k_row_max(const float* __restrict__ scale, int64_t m, int64_t ng,
                          float* __restrict__ out) {
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= m) return;
  float mx = scale[row * ng];
  for (int64_t g = 1; g < ng; ++g) mx = fmaxf(mx, scale[row * ng + g]);
  out[row] = mx;
}

// Adaptive CD: rows whose terminal precision gamma1 s^2 (s the row's scale,
// its largest group scale with group-wise grids) exceeds the threshold skip
// CD and keep the marginal MAP.
__global__ void k_cd_skip(const double* __restrict__ gamma1, const float* __restrict__ scale,
                          int64_t m, int64_t ng, double threshold, int32_t* __restrict__ skip) {
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= m) return;
  float s = scale[row * ng];
  for (int64_t g = 1; g < ng; ++g) s = fmaxf(s, scale[row * ng + g]);
  skip[row] = gamma1[row] * (double)s * (double)s > threshold ? 1 : 0;
}

}  // namespace

mpq_status launch_cd_skip(const double* gamma1, const float* scale, int64_t m, int64_t ng,
                          double threshold, int32_t* skip, cudaStream_t st) {
  if (m <= 0) return MPQ_OK;
  {
    ProfScope ps_("k_cd_skip", st);
    k_cd_skip<<<(unsigned)cdiv(m, 256), 256, 0, st>>>(gamma1, scale, m, ng, threshold, skip);
  }
  count_launch();
  return check_launch("k_cd_skip");
}

mpq_status launch_row_max(const float* scale, int64_t m, int64_t ng, float* out, cudaStream_t st) {
  if (m <= 0) return MPQ_OK;
  {
    ProfScope ps_("k_row_max", st);
    k_row_max<<<(unsigned)cdiv(m, 256), 256, 0, st>>>(scale, m, ng, out);
  }
  count_launch();
  return check_launch("k_row_max");
}

// Width of a CD panel: whole tiles, with the panel's slab of the gradient
// (m x P fp32) within CD_PANEL_BYTES so that it stays in L2 while the
// panel's tiles update it; never below CD_PANEL_MIN columns (the K of the
// GEMM that closes a panel) and never above the padded width.
int64_t cd_panel_cols(int64_t m, int64_t n) {
  const int64_t fit = CD_PANEL_BYTES / (4 * std::max<int64_t>(m, 1)) / CD_TILE * CD_TILE;
  return std::min(std::max<int64_t>(fit, CD_PANEL_MIN), round_up(n, CD_TILE));
}

mpq_status launch_cd(mpq_plan_s* p, const float* W, int64_t m, const float* scale,
                     const float* offset, uint16_t* idx, float* h, int64_t ldh, int32_t sweeps,
                     int32_t* changes, cudaStream_t st, const int32_t* skip) {
  (void)W;
  (void)offset;
  if (m <= 0 || sweeps <= 0) return MPQ_OK;
  if (changes == nullptr) return fail(MPQ_ERR_INVALID_ARG, "CD needs a changes buffer");
  MPQ_CUDA(cudaMemsetAsync(changes, 0, sizeof(int32_t) * m * sweeps, st));
  Workspace& w = p->ws;
  const int64_t n = p->n;
  const int nt = (int)cdiv(n, CD_TILE);
  // Columns are visited in panels of whole tiles whose slab of h (m x P
  // fp32) stays in L2.  Each tile's changes update the gradient of its own
  // panel only (all of the panel's columns, so the panel stays exact for the
  // next sweep too); at the end of a panel one GEMM with K = P brings every
  // column outside it up to date.  With one panel this is the plain
  // per-tile update of all columns.
  const int64_t P = p->params.cd_panel > 0 ? std::min<int64_t>(p->params.cd_panel, round_up(n, CD_TILE))
                                           : cd_panel_cols(m, n);
  const int np = (int)cdiv(n, P);
  int* tile_flags = w.tile_count;                       // sweeps x nt
  int* panel_flags = w.tile_count + (int64_t)sweeps * nt;  // sweeps x np
  MPQ_CUDA(cudaMemsetAsync(w.tile_count, 0, sizeof(int) * sweeps * (nt + np), st));
  const CUtensorMap* c_reduce = (h == w.Hg) ? &w.tm_hg : nullptr;
  // c_new - c_old is exact in fp16 (level differences, lattice coordinates);
  // with group-wise grids Delta carries the group's scale ratio (an fp16 pair)
  const bool a_exact = (p->d == 1 && !p->G) || p->vec_tc;
  if (p->d == 1 && p->G) MPQ_TRY(launch_row_max(scale, m, p->ng, w.sref, st));
  auto update = [&](int64_t a_k0, int64_t b_k0, int64_t K, int64_t c0, int64_t c1,
                    const int* gate, const char* tag) -> mpq_status {
    if (c1 <= c0) return MPQ_OK;
    GemmOpts o;
    o.a_k0 = a_k0;
    o.b_k0 = b_k0;
    o.n0 = c0;
    o.accumulate = true;
    o.a_exact = a_exact;
    o.gate = gate;
    o.c_reduce = c_reduce;
    return gemm_tc(w.As, w.tm_an_hi, w.tm_an_lo, p->H_s, p->tm_h_hi, p->tm_h_lo, h, ldh, m,
                   c1 - c0, K, p->H_s.unscale_host, p->status, st, tag, o);
  };
  // candidate scan of the vector path: tensor cores for lattice codebooks
  // (one partial minimum per codebook slice), else the SIMT kernel (one per
  // chunk of CD8_CHUNK codewords)
  const bool tc = p->d == 8 && p->vec_tc;
  const int nchunks = p->d == 1 ? 0 : tc ? cd_scan_slices(m, p->K) : (int)cdiv(p->K, CD8_CHUNK);
  float* part_val = nullptr;
  int* part_idx = nullptr;
  int dev = 0, sms = 148;
  if (p->d == 1) {
    MPQ_CUDA(cudaFuncSetAttribute(k_cd_tile_decide, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  CD1_SMEM_MAX));
    MPQ_CUDA(cudaGetDevice(&dev));
    MPQ_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  } else {
    MPQ_CUDA(cudaMallocAsync(&part_val, sizeof(float) * m * nchunks, st));
    MPQ_CUDA(cudaMallocAsync(&part_idx, sizeof(int) * m * nchunks, st));
  }
  float* hl = w.Hl;  // d = 8: m x CD_TILE tile-local gradient
  mpq_status rc = MPQ_OK;
  // Within a panel the tiles go in groups.  d = 1 (CD1_GROUP tiles): each
  // tile applies the group's earlier changes to its own columns itself, and
  // one GEMM with K = the group's width brings the panel's gradient up to
  // date after the group.  d = 8 (CD_GROUP tiles): a tile's changes update
  // the gradient of its own group's columns at once (the next tile reads
  // them), and one GEMM after the group brings the rest of the panel up to
  // date.  Either way a per-tile update moves at most m x (group width) of
  // the gradient through L2 instead of the panel's slab.
  const int64_t GW = (int64_t)(p->d == 1 ? CD1_GROUP : CD_GROUP) * CD_TILE;
  for (int sw = 0; sw < sweeps && rc == MPQ_OK; ++sw) {
    const bool last = sw == sweeps - 1;
    for (int pi = 0; pi < np && rc == MPQ_OK; ++pi) {
      const int64_t ps = (int64_t)pi * P, pe = std::min<int64_t>(n, ps + P);
      int* pflag = panel_flags + (int64_t)sw * np + pi;
      for (int64_t g0 = ps; g0 < pe && rc == MPQ_OK; g0 += GW) {
      const int64_t g1 = std::min<int64_t>(pe, g0 + GW);
      for (int64_t t0 = g0; t0 < g1 && rc == MPQ_OK; t0 += CD_TILE) {
        const int j = (int)(t0 / CD_TILE);
        const int tw = (int)std::min<int64_t>(CD_TILE, n - t0);
        int* tflag = tile_flags + (int64_t)sw * nt + j;
        // the tile's Delta/scale lands at its place in the panel's A operand
        __half* dhi = w.As.hi + (t0 - ps);
        __half* dlo = w.As.lo + (t0 - ps);
        if (p->d == 1) {
          // one CTA per SM, with rows per CTA such that one wave holds all
          // rows with the fewest on the busiest SM (every CTA stages the same
          // H blocks from L2, so fewer CTAs move fewer bytes)
          const int gk = (int)((t0 - g0) / CD_TILE);
          const int warps = (int)std::min<int64_t>(CD1_WARPS, std::max<int64_t>(4, cdiv(m, sms)));
          ProfScope ps_("k_cd_tile_decide", st);
          k_cd_tile_decide<<<(unsigned)cdiv(m, warps), warps * 32, CD1_SMEM + gk * CD1_BLOCK, st>>>(
              m, n, p->K, t0, tw, gk, scale, (int)p->ng, p->G ? (int)(t0 / p->G) : 0,
              p->G ? w.sref : nullptr, p->H32, idx, h, ldh, sweeps, sw, changes, dhi, dlo,
              w.As.ld, w.As.row_unscale, tflag, pflag, skip);
          count_launch();
          rc = check_launch("k_cd_tile_decide");
        } else {
          for (int64_t b = t0 / 8; b < (t0 + tw) / 8; ++b) {
            if (tc) {
              rc = launch_cd_vec_scan(p, m, b, t0, scale, idx, h, ldh, hl, part_val, part_idx,
                                      nchunks, st);
              if (rc != MPQ_OK) break;
            } else {
              dim3 ga((unsigned)nchunks, (unsigned)cdiv(m, CD8_ROWS));
              ProfScope ps_("k_cd_vec_eval", st);
              k_cd_vec_eval<<<ga, 256, 0, st>>>(m, n, p->K, b, t0, p->cb, p->qtab, p->H32, scale,
                                                idx, h, ldh, hl, sweeps, sw, changes, skip,
                                                part_val, part_idx, nchunks);
            }
            {
              ProfScope ps_("k_cd_vec_apply", st);
              k_cd_vec_apply<<<(unsigned)cdiv(m, CD8_APPLY_WARPS), CD8_APPLY_WARPS * 32, 0, st>>>(
                  m, n, p->K, b, t0, tw, p->cb, p->qtab, p->H32, scale, idx, h, ldh, hl, sweeps,
                  sw, changes, part_val, part_idx, nchunks, dhi, dlo, w.As.ld, w.As.row_unscale,
                  tflag, pflag, skip);
            }
            count_launch(tc ? 1 : 2);
            rc = check_launch("k_cd_vec");
            if (rc != MPQ_OK) break;
          }
        }
        if (rc != MPQ_OK) break;
        // d = 8: the group's columns; in the last sweep only the ones still
        // to be visited (the gradient is not read after it)
        if (p->d != 1) rc = update(t0 - ps, t0, tw, last ? t0 + tw : g0, g1, tflag, "gemm_cd_update");
      }
      // the group's changes reach the rest of the panel (d = 1: the whole
      // panel, the group's own columns too), gated on any change in the panel
      // so far, which covers this group's; in the last sweep only the columns
      // after the group
      if (rc == MPQ_OK && p->d == 1 && !last) {
        rc = update(g0 - ps, g0, g1 - g0, ps, pe, pflag, "gemm_cd_group");
      } else {
        if (rc == MPQ_OK && !last && g0 > ps)
          rc = update(g0 - ps, g0, g1 - g0, ps, g0, pflag, "gemm_cd_group");
        if (rc == MPQ_OK && g1 < pe)
          rc = update(g0 - ps, g0, g1 - g0, g1, pe, pflag, "gemm_cd_group");
      }
      }
      if (rc != MPQ_OK || np == 1) continue;
      if (!last) rc = update(0, ps, pe - ps, 0, ps, pflag, "gemm_cd_panel");  // columns before
      if (rc == MPQ_OK) rc = update(0, ps, pe - ps, pe, n, pflag, "gemm_cd_panel");  // and after
    }
  }
  if (part_val) cudaFreeAsync(part_val, st);
  if (part_idx) cudaFreeAsync(part_idx, st);
  return rc;
}

}  // namespace mpq
