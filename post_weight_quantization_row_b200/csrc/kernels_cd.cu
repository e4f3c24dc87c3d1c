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

#include "mpq_internal.cuh"

namespace mpq {
namespace {

// ------------------------------------------------------------------ d = 1 --
// One warp per row, all sweeps in one launch.  Columns are visited in tiles
// of CD1_TILE.  Inside a tile the gradient of the tile's own columns lives in
// shared memory: the 32 lanes evaluate 32 consecutive columns against it;
// the decisions are exact up to the first lane that accepts a change, so the
// warp commits that change, updates the tile-local gradient with the row of
// H and resumes right after it (identical to visiting columns one by one).
// When the tile is done its changes are applied to the rest of h in one pass
// (h_i -= sum_changes H[c, i] delta_c), so h is read and written once per
// tile instead of once per change.
constexpr int CD1_WARPS = 8;
constexpr int CD1_TILE = 128;

__global__ void __launch_bounds__(CD1_WARPS * 32)
    k_cd_scalar(int64_t m, int64_t n, int L, const float* __restrict__ scale,
                const float* __restrict__ H, const float* __restrict__ Hdiag,
                uint16_t* __restrict__ idx, float* __restrict__ h, int sweeps,
                int32_t* __restrict__ changes) {
  __shared__ float s_h[CD1_WARPS][CD1_TILE];
  __shared__ int s_col[CD1_WARPS][CD1_TILE];
  __shared__ float s_dl[CD1_WARPS][CD1_TILE];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * CD1_WARPS + wid;
  if (row >= m) return;
  const float sc = scale[row];
  float* hr = h + row * n;
  uint16_t* ir = idx + row * n;
  float* sh = s_h[wid];
  int* scol = s_col[wid];
  float* sdl = s_dl[wid];
  for (int sw = 0; sw < sweeps; ++sw) {
    int nchg = 0;
    for (int64_t t0 = 0; t0 < n; t0 += CD1_TILE) {
      const int tw = (int)((n - t0) < CD1_TILE ? (n - t0) : CD1_TILE);
      for (int i = lane; i < tw; i += 32) sh[i] = hr[t0 + i];
      __syncwarp();
      int ntile = 0;  // changes in this tile
      int c = 0;
      while (c < tw) {
        const int j = c + lane;
        bool acc = false;
        int kb = 0, kc = 0;
        if (j < tw) {
          const float hj = sh[j], g = Hdiag[t0 + j];
          kc = ir[t0 + j];
          float best = 0.0f;  // staying put
          for (int k = 0; k < L; ++k) {
            const float dl = sc * (float)(k - kc);
            const float dE = dl * fmaf(0.5f * dl, g, -hj);
            if (dE < best) {
              best = dE;
              kb = k;
            }
          }
          acc = best < 0.0f;
        }
        const unsigned mask = __ballot_sync(0xffffffffu, acc);
        if (mask == 0u) {
          c += 32;
          continue;
        }
        const int first = __ffs(mask) - 1;
        const int jj = c + first;
        const int knew = __shfl_sync(0xffffffffu, kb, first);
        const int kold = __shfl_sync(0xffffffffu, kc, first);
        const float dl = sc * (float)(knew - kold);
        if (lane == first) {
          ir[t0 + jj] = (uint16_t)knew;
          scol[ntile] = (int)(t0 + jj);
          sdl[ntile] = dl;
        }
        ++ntile;
        const float* Hj = H + (t0 + jj) * n + t0;
        for (int i = lane; i < tw; i += 32) sh[i] = fmaf(-Hj[i], dl, sh[i]);
        __syncwarp();
        c = jj + 1;
      }
      __syncwarp();
      nchg += ntile;
      // write the tile back and apply its changes to every other column
      for (int i = lane; i < tw; i += 32) hr[t0 + i] = sh[i];
      if (ntile > 0) {
        for (int64_t i = lane; i < n; i += 32) {
          if (i >= t0 && i < t0 + tw) continue;
          float a = hr[i];
          for (int q = 0; q < ntile; ++q) a = fmaf(-H[(int64_t)scol[q] * n + i], sdl[q], a);
          hr[i] = a;
        }
      }
      __syncwarp();
    }
    if (lane == 0 && changes) changes[row * sweeps + sw] = nchg;
    if (nchg == 0) {
      if (lane == 0 && changes)
        for (int s2 = sw + 1; s2 < sweeps; ++s2) changes[row * sweeps + s2] = 0;
      break;
    }
  }
}

// ------------------------------------------------------------------ d = 8 --
// Per block step b (all rows together): score(c) = qtab_b(c) - c . g'/1,
// with qtab_b(c) = 1/2 c^T G_b c, g' = (h_b + G_b x_b)/scale; the energy
// change of codeword c is scale^2 (score(c) - score(c_cur)).
// Kernel A: partial argmin over a chunk of codewords for a tile of rows.
// Kernel B: combine chunks, accept if strictly better, update idx and h.
constexpr int CD8_ROWS = 64;    // rows per CTA (8 warps x 8 rows)
constexpr int CD8_CHUNK = 1024; // codewords per CTA

__device__ __forceinline__ bool row_active(const int32_t* changes, int64_t row, int sweeps,
                                           int sw) {
  return sw == 0 || changes[row * sweeps + sw - 1] > 0;
}

// g' for one row at block b; G_b and x_b in weight units.
__device__ __forceinline__ void block_gradient(const float* __restrict__ H, int64_t n,
                                               const float* __restrict__ hrow,
                                               const float* __restrict__ cb, int kcur,
                                               float sc, int64_t b, float* gout) {
  float x[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) x[j] = sc * cb[(int64_t)kcur * 8 + j];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float g = hrow[8 * b + i];
    const float* Hi = H + (8 * b + i) * n + 8 * b;
#pragma unroll
    for (int j = 0; j < 8; ++j) g = fmaf(Hi[j], x[j], g);
    gout[i] = g / sc;
  }
}

__global__ void __launch_bounds__(256)
    k_cd_vec_eval(int64_t m, int64_t n, int K, int64_t b, const float* __restrict__ cb,
                  const float* __restrict__ qtab, const float* __restrict__ H,
                  const float* __restrict__ scale, const uint16_t* __restrict__ idx,
                  const float* __restrict__ h, int sweeps, int sw,
                  const int32_t* __restrict__ changes, float* __restrict__ part_val,
                  int* __restrict__ part_idx, int nchunks) {
  __shared__ float scb[CD8_CHUNK][8];
  __shared__ float sq[CD8_CHUNK];
  __shared__ float sg[CD8_ROWS][8];
  const int64_t B = n / 8;
  const int chunk = blockIdx.x;
  const int64_t r0 = (int64_t)blockIdx.y * CD8_ROWS;
  const int c0 = chunk * CD8_CHUNK;
  const int cn = min(CD8_CHUNK, K - c0);
  for (int e = threadIdx.x; e < cn * 8; e += blockDim.x) scb[e / 8][e % 8] = cb[(int64_t)c0 * 8 + e];
  for (int e = threadIdx.x; e < cn; e += blockDim.x) sq[e] = qtab[b * K + c0 + e];
  if (threadIdx.x < CD8_ROWS) {
    const int64_t row = r0 + threadIdx.x;
    const bool act = row < m && row_active(changes, row, sweeps, sw);
    if (act) {
      float g[8];
      block_gradient(H, n, h + row * n, cb, idx[row * B + b], scale[row], b, g);
#pragma unroll
      for (int i = 0; i < 8; ++i) sg[threadIdx.x][i] = g[i];
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) sg[threadIdx.x][i] = 0.0f;
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;  // warp w: rows 8w..8w+7
  float g[8][8];
#pragma unroll
  for (int rr = 0; rr < 8; ++rr)
#pragma unroll
    for (int i = 0; i < 8; ++i) g[rr][i] = sg[8 * w + rr][i];
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
    for (int i = 0; i < 8; ++i) cv[i] = scb[c][i];
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
    const int64_t row = r0 + 8 * w + rr;
    if (lane == 0 && row < m) {
      part_val[row * nchunks + chunk] = v;
      part_idx[row * nchunks + chunk] = k;
    }
  }
}

__global__ void __launch_bounds__(256)
    k_cd_vec_apply(int64_t m, int64_t n, int K, int64_t b, const float* __restrict__ cb,
                   const float* __restrict__ qtab, const float* __restrict__ H,
                   const float* __restrict__ scale, uint16_t* __restrict__ idx,
                   float* __restrict__ h, int sweeps, int sw, int32_t* __restrict__ changes,
                   const float* __restrict__ part_val, const int* __restrict__ part_idx,
                   int nchunks) {
  __shared__ float sdelta[8];
  __shared__ int sdo;
  const int64_t row = blockIdx.x;
  const int64_t B = n / 8;
  if (!row_active(changes, row, sweeps, sw)) {
    if (threadIdx.x == 0 && b == 0) changes[row * sweeps + sw] = 0;
    return;
  }
  if (threadIdx.x == 0) {
    if (b == 0) changes[row * sweeps + sw] = 0;
    float v = INFINITY;
    int k = 0x7fffffff;
    for (int c = 0; c < nchunks; ++c) {
      const float v2 = part_val[row * nchunks + c];
      const int k2 = part_idx[row * nchunks + c];
      if (v2 < v || (v2 == v && k2 < k)) {
        v = v2;
        k = k2;
      }
    }
    const int kcur = idx[row * B + b];
    const float sc = scale[row];
    float g[8];
    block_gradient(H, n, h + row * n, cb, kcur, sc, b, g);
    float scur = qtab[b * K + kcur];
#pragma unroll
    for (int i = 0; i < 8; ++i) scur = fmaf(-cb[(int64_t)kcur * 8 + i], g[i], scur);
    const bool accept = (v < scur) && k >= 0 && k < K;
    sdo = accept;
    if (accept) {
      idx[row * B + b] = (uint16_t)k;
      changes[row * sweeps + sw] += 1;
#pragma unroll
      for (int i = 0; i < 8; ++i) sdelta[i] = sc * (cb[(int64_t)k * 8 + i] - cb[(int64_t)kcur * 8 + i]);
    }
  }
  __syncthreads();
  if (!sdo) return;
  float dl[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) dl[j] = sdelta[j];
  float* hr = h + row * n;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
    const float* Hi = H + i * n + 8 * b;
    float acc = hr[i];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc = fmaf(-Hi[j], dl[j], acc);
    hr[i] = acc;
  }
}

}  // namespace

mpq_status launch_cd(const mpq_plan_s* p, const float* W, int64_t m, const float* scale,
                     const float* offset, uint16_t* idx, float* h, int32_t sweeps,
                     int32_t* changes, cudaStream_t st) {
  (void)W;
  (void)offset;
  if (m <= 0 || sweeps <= 0) return MPQ_OK;
  if (p->d == 1) {
    {
      ProfScope ps_("k_cd_scalar", st);
      k_cd_scalar<<<(unsigned)cdiv(m, CD1_WARPS), CD1_WARPS * 32, 0, st>>>(
          m, p->n, p->K, scale, p->H32, p->Hdiag, idx, h, sweeps, changes);
    }
    count_launch();
    return check_launch("k_cd_scalar");
  }
  // d = 8 needs the change counters for its early stop
  if (changes == nullptr) return fail(MPQ_ERR_INVALID_ARG, "vector CD needs a changes buffer");
  const int nchunks = (int)cdiv(p->K, CD8_CHUNK);
  float* part_val = nullptr;
  int* part_idx = nullptr;
  MPQ_CUDA(cudaMallocAsync(&part_val, sizeof(float) * m * nchunks, st));
  MPQ_CUDA(cudaMallocAsync(&part_idx, sizeof(int) * m * nchunks, st));
  const int64_t B = p->n / 8;
  mpq_status rc = MPQ_OK;
  for (int sw = 0; sw < sweeps && rc == MPQ_OK; ++sw) {
    for (int64_t b = 0; b < B; ++b) {
      dim3 ga((unsigned)nchunks, (unsigned)cdiv(m, CD8_ROWS));
      {
        ProfScope ps_("k_cd_vec_eval", st);
        k_cd_vec_eval<<<ga, 256, 0, st>>>(m, p->n, p->K, b, p->cb, p->qtab, p->H32, scale, idx, h,
                                          sweeps, sw, changes, part_val, part_idx, nchunks);
      }
      {
        ProfScope ps_("k_cd_vec_apply", st);
        k_cd_vec_apply<<<(unsigned)m, 256, 0, st>>>(m, p->n, p->K, b, p->cb, p->qtab, p->H32,
                                                    scale, idx, h, sweeps, sw, changes, part_val,
                                                    part_idx, nchunks);
      }
      count_launch(2);
      rc = check_launch("k_cd_vec");
      if (rc != MPQ_OK) break;
    }
  }
  cudaFreeAsync(part_val, st);
  cudaFreeAsync(part_idx, st);
  return rc;
}

}  // namespace mpq
