// Row kernels of the MPQ solve: init, blockwise denoisers, extrinsic
// updates, the per-row epilogue of the rank-space linear module with the
// beta M-step, residuals and energies.
//
// Source: "MPQ: A Message-Passing View of Post-Training Quantization"
// (papernotes.org note), Key design 1 (denoiser, extrinsic updates, linear
// module in rank space), Key design 2 (beta M-step), hyper-parameter
// section (gamma1_0 = 1/MSE(w, w_rtn), rho_damp); the min-max grid follows
// the NeUQI note, existing pain points section.
#include <math.h>

#include <type_traits>

#include "f32x2.cuh"
#include "mpq_internal.cuh"

namespace mpq {
namespace {

constexpr int ROW_THREADS = 256;
constexpr int ROW_UNROLL = 4;  // elements per thread whose loads are in flight together

// ------------------------------------------------------------ reductions ---
template <typename T, typename Op>
__device__ __forceinline__ T warp_reduce(T v, Op op) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Deterministic block reduction (fixed tree), result broadcast to all threads.
template <typename T, typename Op>
__device__ T block_reduce(T v, Op op, T* smem /* >= 32 */) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  v = warp_reduce(v, op);
  __syncthreads();
  if (lane == 0) smem[wid] = v;
  __syncthreads();
  if (wid == 0) {
    T x = lane < nw ? smem[lane] : smem[0];
    if (lane >= nw) x = smem[0];
    // lanes >= nw duplicate element 0; op must be idempotent for those
    // (min/max) or we mask them explicitly for sums below
    x = warp_reduce(x, op);
    if (lane == 0) smem[32] = x;
  }
  __syncthreads();
  return smem[32];
}

struct SumD {
  __device__ double operator()(double a, double b) const { return a + b; }
};
struct MinF {
  __device__ float operator()(float a, float b) const { return fminf(a, b); }
};
struct MaxF {
  __device__ float operator()(float a, float b) const { return fmaxf(a, b); }
};

__device__ double block_sum(double v, double* smem) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  v = warp_reduce(v, SumD());
  __syncthreads();
  if (lane == 0) smem[wid] = v;
  __syncthreads();
  if (wid == 0) {
    double x = lane < nw ? smem[lane] : 0.0;
    x = warp_reduce(x, SumD());
    if (lane == 0) smem[32] = x;
  }
  __syncthreads();
  return smem[32];
}

__device__ __forceinline__ double clip_count(double v, double lo, double hi, int* cnt) {
  double c = isnan(v) ? lo : fmin(fmax(v, lo), hi);
  if (c != v) ++*cnt;
  return c;
}

// 2^x by the hardware approximation (MUFU ex2, relative error ~2^-22;
// flushes subnormal results to zero, which is harmless for posterior weights)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Split of a row for the tensor-core GEMM: a per-row power of two e with
// max|x| * 2^-e < 2^14, then hi = fp16(x 2^-e), lo = fp16(x 2^-e - hi).
__device__ __forceinline__ int split_exponent(float amax) {
  int ex = 0;
  frexpf(amax, &ex);
  return (amax > 0.0f) ? ex - 14 : 0;
}

// the same split for four adjacent elements (o a multiple of 4), two packed
// conversions and one 8-byte store per half
__device__ __forceinline__ void split_store4(const float (&x)[4], __half* __restrict__ hi,
                                             __half* __restrict__ lo, int64_t o) {
  const __half2 h0 = __floats2half2_rn(x[0], x[1]), h1 = __floats2half2_rn(x[2], x[3]);
  const float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
  const __half2 l0 = __floats2half2_rn(x[0] - f0.x, x[1] - f0.y);
  const __half2 l1 = __floats2half2_rn(x[2] - f1.x, x[3] - f1.y);
  uint2 hv, lv;
  hv.x = *reinterpret_cast<const uint32_t*>(&h0);
  hv.y = *reinterpret_cast<const uint32_t*>(&h1);
  lv.x = *reinterpret_cast<const uint32_t*>(&l0);
  lv.y = *reinterpret_cast<const uint32_t*>(&l1);
  *reinterpret_cast<uint2*>(hi + o) = hv;
  *reinterpret_cast<uint2*>(lo + o) = lv;
}

__device__ __forceinline__ void split_store(float xs, __half* __restrict__ hi,
                                            __half* __restrict__ lo, int64_t o) {
  const __half h = __float2half_rn(xs);
  hi[o] = h;
  lo[o] = __float2half_rn(xs - __half2float(h));
}

// ------------------------------------------------------------------ init ---
// d = 1: per-row min-max grid (unless given), nearest level, gamma1_0.
__global__ void __launch_bounds__(ROW_THREADS)
    k_init_scalar(const float* __restrict__ W, int64_t n, int L, int given,
                  float* __restrict__ scale, float* __restrict__ offset,
                  uint16_t* __restrict__ idx, double* __restrict__ gamma1_0, int* status) {
  __shared__ float fs[33];
  __shared__ double ds[33];
  const int64_t row = blockIdx.x;
  const float* w = W + row * n;
  if (!given) {
    float lo = INFINITY, hi = -INFINITY;
    bool bad = false;
    for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
      const float x = w[j];
      bad |= !isfinite(x);
      lo = fminf(lo, x);
      hi = fmaxf(hi, x);
    }
    if (bad) atomicOr(status, STATUS_NONFINITE);
    lo = block_reduce(lo, MinF(), fs);
    hi = block_reduce(hi, MaxF(), fs);
    if (threadIdx.x == 0) {
      double s = ((double)hi - (double)lo) / (double)(L - 1);
      if (!(hi > lo)) s = (hi != 0.0f) ? fabs((double)hi) : 1.0;
      double z = rint(-(double)lo / s);
      z = fmin(fmax(z, 0.0), (double)(L - 1));
      scale[row] = (float)s;
      offset[row] = (float)(-s * z);
    }
    __syncthreads();
  }
  const double sc = scale[row], off = offset[row];
  double se = 0.0;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    const double x = w[j];
    double t = (x - off) / sc;
    double k0 = fmin(fmax(floor(t), 0.0), (double)(L - 1));
    double k1 = fmin(k0 + 1.0, (double)(L - 1));
    const double d0 = fabs(sc * k0 + off - x), d1 = fabs(sc * k1 + off - x);
    const double k = (d1 < d0) ? k1 : k0;
    idx[row * n + j] = (uint16_t)k;
    const double e = x - (sc * k + off);
    se += e * e;
  }
  se = block_sum(se, ds);
  if (threadIdx.x == 0) gamma1_0[row] = 1.0 / fmax(se / (double)n, 1e-30);
}

// d = 1 with group-wise grids: one min-max grid per group of G consecutive
// columns (unless given; scale/offset are m x n/G), nearest level, and
// gamma1_0 from the whole row.  One warp per group.
__global__ void __launch_bounds__(ROW_THREADS)
    k_init_scalar_groups(const float* __restrict__ W, int64_t n, int L, int G, int given,
                         float* __restrict__ scale, float* __restrict__ offset,
                         uint16_t* __restrict__ idx, double* __restrict__ gamma1_0, int* status) {
  __shared__ double ds[33];
  const int64_t row = blockIdx.x;
  const int ng = (int)(n / G);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const float* w = W + row * n;
  double se = 0.0;
  bool bad = false;
  for (int g = wid; g < ng; g += nw) {
    const float* wg = w + (int64_t)g * G;
    float s32, o32;
    if (!given) {
      float lo = INFINITY, hi = -INFINITY;
      for (int j = lane; j < G; j += 32) {
        const float x = wg[j];
        bad |= !isfinite(x);
        lo = fminf(lo, x);
        hi = fmaxf(hi, x);
      }
      lo = warp_reduce(lo, MinF());
      hi = warp_reduce(hi, MaxF());
      double s = ((double)hi - (double)lo) / (double)(L - 1);
      if (!(hi > lo)) s = (hi != 0.0f) ? fabs((double)hi) : 1.0;
      double z = rint(-(double)lo / s);
      z = fmin(fmax(z, 0.0), (double)(L - 1));
      s32 = (float)s;
      o32 = (float)(-s * z);
      if (lane == 0) {
        scale[row * ng + g] = s32;
        offset[row * ng + g] = o32;
      }
    } else {
      s32 = scale[row * ng + g];
      o32 = offset[row * ng + g];
    }
    const double sc = s32, off = o32;
    for (int j = lane; j < G; j += 32) {
      const double x = wg[j];
      const double t = (x - off) / sc;
      const double k0 = fmin(fmax(floor(t), 0.0), (double)(L - 1));
      const double k1 = fmin(k0 + 1.0, (double)(L - 1));
      const double d0 = fabs(sc * k0 + off - x), d1 = fabs(sc * k1 + off - x);
      const double k = (d1 < d0) ? k1 : k0;
      idx[row * n + (int64_t)g * G + j] = (uint16_t)k;
      const double e = x - (sc * k + off);
      se += e * e;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, STATUS_NONFINITE);
  se = block_sum(se, ds);
  if (threadIdx.x == 0) gamma1_0[row] = 1.0 / fmax(se / (double)n, 1e-30);
}

// d = 8: per-row RMS scale (unless given), offset 0.
__global__ void __launch_bounds__(ROW_THREADS)
    k_init_rms(const float* __restrict__ W, int64_t n, int given, float* __restrict__ scale,
               float* __restrict__ offset, int* status) {
  __shared__ double ds[33];
  const int64_t row = blockIdx.x;
  const float* w = W + row * n;
  double ss = 0.0;
  bool bad = false;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    const double x = w[j];
    bad |= !isfinite(w[j]);
    ss += x * x;
  }
  if (bad) atomicOr(status, STATUS_NONFINITE);
  ss = block_sum(ss, ds);
  if (!given && threadIdx.x == 0) {
    double rho = sqrt(ss / (double)n);
    if (!(rho > 0.0)) rho = 1.0;
    scale[row] = (float)rho;
    offset[row] = 0.0f;
  }
}

// d = 8: gamma1_0 from the nearest codewords already in idx.
__global__ void __launch_bounds__(ROW_THREADS)
    k_gamma0_vec(const float* __restrict__ W, int64_t n, const float* __restrict__ cb,
                 const float* __restrict__ scale, const float* __restrict__ offset,
                 const uint16_t* __restrict__ idx, double* __restrict__ gamma1_0) {
  __shared__ double ds[33];
  const int64_t row = blockIdx.x;
  const double sc = scale[row], off = offset[row];
  double se = 0.0;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    const int k = idx[row * (n / 8) + j / 8];
    const double e = (double)W[row * n + j] - (sc * cb[k * 8 + (j & 7)] + off);
    se += e * e;
  }
  se = block_sum(se, ds);
  if (threadIdx.x == 0) gamma1_0[row] = 1.0 / fmax(se / (double)n, 1e-30);
}

// ------------------------------------------------------- scalar denoiser ---
// Posterior over levels k = 0..L-1 (weights scale*k + offset) of
// q(k) ~ exp(-gamma1/2 (scale k + offset - r)^2) [* anchor]; in level units
// t = (r - offset)/scale, g = gamma1 scale^2, logit_k = -g/2 (k - t)^2.

// per-row constants (the stage kernel and the fused VAMP row kernel share them)
struct ScalarDen {
  float sc, off, inv_sc, Lm1, sc2f, A2;
  float hwf, kmax0;  // window half-width and last window start, as floats
  double doff, inv_dsc, g, ga, geff;
  double cr, cw, coff;  // anchored centre in level units: cr r + cw w - coff
  float crh, crl, cwh, cwl, cofh, cofl;  // the same as fp32 pairs (hi + lo)
  int L, hw, nlev;
  bool anchored, precise;
};

// The prior anchor (reading of the pages' "anchor scale" tau) has a width of
// tau grid steps: its precision in level units is 1/tau^2 for every row.
__device__ __forceinline__ ScalarDen scalar_den_row(float sc, float off, double gamma1, int L,
                                                    bool anchored, double inv_tau2) {
  ScalarDen c;
  c.sc = sc;
  c.off = off;
  const double dsc = sc;
  c.doff = off;
  c.inv_dsc = 1.0 / dsc;
  const double sc2 = dsc * dsc;
  c.g = fmin(gamma1 * sc2, 1e30);
  c.anchored = anchored;
  c.ga = anchored ? fmin(inv_tau2, 1e30) : 0.0;
  c.geff = c.g + c.ga;
  // (g (r - off) + ga (w - off)) / (scale geff), with the division and the
  // offset folded into row constants ((g + ga) / geff = 1)
  c.cr = c.g * c.inv_dsc / c.geff;
  c.cw = c.ga * c.inv_dsc / c.geff;
  c.coff = c.doff * c.inv_dsc;
  c.crh = (float)c.cr;
  c.crl = (float)(c.cr - (double)c.crh);
  c.cwh = (float)c.cw;
  c.cwl = (float)(c.cw - (double)c.cwh);
  c.cofh = (float)c.coff;
  c.cofl = (float)(c.coff - (double)c.cofh);
  c.A2 = (float)(-0.5 * c.geff * 1.4426950408889634);  // -geff/2 log2(e)
  c.L = L;
  // Levels far from the nearest one carry no weight: with |dt| <= 1/2 (or dt
  // pointing away from the grid at its ends) the log2-weight of level k* + dk
  // relative to k* is at most A2 (dk^2 - |dk|), so a window of 2hw+1 levels
  // with |A2| hw (hw+1) >= 64 drops only weights below 2^-64 of the largest
  // (at most 2^-55 relative in the moments).  hw is uniform over the row.
  c.hw = L;  // half-width of the window
  if (-c.A2 > 0.0f) {
    const double w = ceil(0.5 * (-1.0 + sqrt(1.0 + 256.0 / (double)(-c.A2))));
    c.hw = (int)fmin(w, (double)L);
  }
  // high precision (|A| > 5): the exact exponent form below
  c.precise = -c.A2 > 5.0f;
  c.nlev = min(2 * c.hw + 1, L);
  c.hwf = (float)c.hw;
  c.kmax0 = (float)(L - c.nlev);
  c.inv_sc = (float)c.inv_dsc;
  c.Lm1 = (float)(L - 1);
  c.sc2f = (float)sc2;
  return c;
}

// One weight: cavity r (and w for the anchored prior) -> posterior mean xh,
// variance (returned) and the most likely level ks (an integer as a float).
// Instantiated per precision regime and prior, both uniform over a row.
// PAIR_CENTRE (anchored rows): form the centre as an fp32 pair instead of in
// fp64; the nearest level ks is then decided from the pair's rounded sum, so
// it may differ from the exact rounding by one level at an exact half, which
// only moves the window's centre (use it where ks is not an output).
template <bool PRECISE, bool ANCH, bool PAIR_CENTRE = false>
__device__ __forceinline__ float scalar_den_elem(const ScalarDen& c, const float r, const float wr,
                                                 float& xh, float& ks) {
  const float sc = c.sc, off = c.off, inv_sc = c.inv_sc, A2 = c.A2;
  // nearest level and the offset from it in level units, dt ~ dh + dl
  // (the pair matters only in the high-precision rows)
  float dh, dl;
  if constexpr (!ANCH) {
    ks = fminf(fmaxf(ceil_small((r - off) * inv_sc - 0.5f), 0.0f), c.Lm1);
    // r - (scale ks + offset) without rounding the level value: error-free
    // products and sums (Dekker / Knuth) give it as d0 + lo.  The explicitly
    // rounded intrinsics keep the compiler from contracting or
    // reassociating these steps.
    const float pr = __fmul_rn(sc, ks);
    const float pe = fmaf(sc, ks, -pr);
    const float s = __fadd_rn(pr, off);
    const float bb = __fsub_rn(s, pr);
    const float se = __fadd_rn(__fsub_rn(pr, __fsub_rn(s, bb)), __fsub_rn(off, bb));
    const float d0 = __fsub_rn(r, s);
    if constexpr (PRECISE) {
      const float b2 = __fsub_rn(d0, r);
      const float de = __fadd_rn(__fsub_rn(r, __fsub_rn(d0, b2)), __fsub_rn(-s, b2));  // r - s = d0 + de
      const float lo = __fsub_rn(de, __fadd_rn(pe, se));
      dh = __fmul_rn(__fadd_rn(d0, lo), inv_sc);
      dl = __fmul_rn(__fadd_rn(fmaf(-dh, sc, d0), lo), inv_sc);
    } else {
      dh = __fmul_rn(__fsub_rn(d0, __fadd_rn(pe, se)), inv_sc);
      dl = 0.0f;
    }
  } else if constexpr (PAIR_CENTRE) {
    // anchored prior, centre cr r + cw w - coff as an fp32 pair: error-free
    // products (TwoProduct by fma) and sums (TwoSum), the small terms of the
    // constants' low halves added in plain fp32; the explicitly rounded
    // intrinsics keep the compiler from contracting or reassociating
    const float ph = __fmul_rn(c.crh, r), pe = fmaf(c.crh, r, -ph);
    const float qh = __fmul_rn(c.cwh, wr), qe = fmaf(c.cwh, wr, -qh);
    const float s1 = __fadd_rn(ph, qh), b1 = __fsub_rn(s1, ph);
    const float e1 = __fadd_rn(__fsub_rn(ph, __fsub_rn(s1, b1)), __fsub_rn(qh, b1));
    const float s2 = __fsub_rn(s1, c.cofh), b2 = __fsub_rn(s2, s1);
    const float e2 = __fadd_rn(__fsub_rn(s1, __fsub_rn(s2, b2)), __fsub_rn(-c.cofh, b2));
    const float lo = __fadd_rn(__fadd_rn(__fadd_rn(pe, qe), __fadd_rn(e1, e2)),
                               __fsub_rn(fmaf(c.crl, r, __fmul_rn(c.cwl, wr)), c.cofl));
    ks = fminf(fmaxf(ceil_small(__fadd_rn(s2, lo) - 0.5f), 0.0f), c.Lm1);
    const float d0 = __fsub_rn(s2, ks);  // exact: s2 lies within a level or so of ks
    dh = __fadd_rn(d0, lo);
    const float bd = __fsub_rn(dh, d0);
    dl = __fadd_rn(__fsub_rn(d0, __fsub_rn(dh, bd)), __fsub_rn(lo, bd));
  } else {
    // anchored prior: the effective centre mixes r and w (fp64)
    const double tt = fma(c.cr, (double)r, fma(c.cw, (double)wr, -c.coff));
    const double kd = fmin(fmax(ceil(tt - 0.5), 0.0), (double)(c.L - 1));
    ks = (float)kd;
    const double dtd = tt - kd;
    dh = (float)dtd;
    dl = (float)(dtd - (double)dh);
  }
  // min(2hw+1, L) consecutive levels around k*, shifted to stay on the grid;
  // dk = k - k* counts up from the window start as an exact float
  float dk = fminf(fmaxf(ks - c.hwf, 0.0f), c.kmax0) - ks;
  // Two levels per packed f32x2 instruction (dk, dk + 1); each level's
  // arithmetic is the scalar form's, the sums run over even and odd levels
  // separately.  An odd window ends with one scalar level.
  uint64_t dkp = f2_pack(dk, dk + 1.0f);
  uint64_t S0p = 0, S1p = 0, S2p = 0;  // (+0, +0)
  const uint64_t two = f2_pack(2.0f, 2.0f);
  const int npair = c.nlev >> 1;
  float e_t = 0.0f, dk_t = dk + (float)(2 * npair);  // the odd level, if any
  if constexpr (PRECISE) {
    // q_k / q_k* = 2^(A dk (dk - 2 dt)) with dk an exact integer and A =
    // -geff/2 log2(e).  Here geff is large: dk - 2 dt is formed from the
    // pair (dh, dl) before scaling by A, so the exponent keeps fp32 accuracy
    // relative to itself (A dk^2 - 2 A dk dt would cancel, and a plain fp32
    // dt would cost more than 1e-4 of a weight).
    const float m2dh = -2.0f * dh, m2dl = -2.0f * dl;  // exact
    const uint64_t mh = f2_pack(m2dh, m2dh), ml = f2_pack(m2dl, m2dl), a2 = f2_pack(A2, A2);
#pragma unroll 2
    for (int i = 0; i < npair; ++i, dkp = f2_add(dkp, two)) {
      const uint64_t z = f2_mul(f2_mul(a2, dkp), f2_add(f2_add(dkp, mh), ml));
      float z0, z1;
      f2_unpack(z, z0, z1);
      const uint64_t e = f2_pack(fast_exp2(z0), fast_exp2(z1));
      S0p = f2_add(S0p, e);
      const uint64_t ed = f2_mul(e, dkp);
      S1p = f2_add(S1p, ed);
      S2p = f2_fma(ed, dkp, S2p);
    }
    if (c.nlev & 1) e_t = fast_exp2((A2 * dk_t) * ((dk_t + m2dh) + m2dl));
  } else {
    // q_k / q_k* = 2^(dk (A dk + B)), B = -2 A dt: with |A| <= 5 the
    // rounding of B costs under 1e-5 of a weight
    const float B2 = -2.0f * A2 * dh;
    const uint64_t a2 = f2_pack(A2, A2), b2 = f2_pack(B2, B2);
#pragma unroll 2
    for (int i = 0; i < npair; ++i, dkp = f2_add(dkp, two)) {
      const uint64_t z = f2_mul(f2_fma(a2, dkp, b2), dkp);
      float z0, z1;
      f2_unpack(z, z0, z1);
      const uint64_t e = f2_pack(fast_exp2(z0), fast_exp2(z1));
      S0p = f2_add(S0p, e);
      const uint64_t ed = f2_mul(e, dkp);
      S1p = f2_add(S1p, ed);
      S2p = f2_fma(ed, dkp, S2p);
    }
    if (c.nlev & 1) e_t = fast_exp2(fmaf(A2, dk_t, B2) * dk_t);
  }
  float s0a, s0b, s1a, s1b, s2a, s2b;
  f2_unpack(S0p, s0a, s0b);
  f2_unpack(S1p, s1a, s1b);
  f2_unpack(S2p, s2a, s2b);
  const float ed_t = e_t * dk_t;
  const float S0 = (s0a + s0b) + e_t;
  const float S1 = (s1a + s1b) + ed_t;
  const float S2 = fmaf(ed_t, dk_t, s2a + s2b);
  // S0 >= 1 (k* itself has weight 1): the hardware reciprocal (~1 ulp) is
  // far inside the stage tolerance
  float inv;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv) : "f"(S0));
  const float m1 = S1 * inv;
  const float var = fmaxf(fmaf(S2, inv, -m1 * m1), 0.0f);
  xh = fmaf(sc, ks + m1, off);
  return c.sc2f * var;
}

// With GROUPED, scale/offset hold one grid per group of G columns and the
// per-group constants (precision regime included) live in shared memory.
template <bool GROUPED>
__global__ void __launch_bounds__(ROW_THREADS)
    k_denoise_scalar(const float* __restrict__ R1, const double* __restrict__ gamma1,
                     const float* __restrict__ scale, const float* __restrict__ offset,
                     int64_t n, int L, int G, const float* __restrict__ W,
                     const double* __restrict__ gamma1_0, double inv_tau2,
                     float* __restrict__ xhat, float* __restrict__ vblock,
                     double* __restrict__ vsum, uint16_t* __restrict__ idx) {
  __shared__ double ds[33];
  extern __shared__ __align__(16) uint8_t den_smem[];
  ScalarDen* s_den = reinterpret_cast<ScalarDen*>(den_smem);  // GROUPED: one per group
  const int64_t row = blockIdx.x;
  const bool anchored = (W != nullptr);
  const int ng = GROUPED ? (int)(n / G) : 1;
  const ScalarDen c = scalar_den_row(scale[row * ng], offset[row * ng], gamma1[row], L, anchored,
                                     inv_tau2);
  if (GROUPED) {
    for (int g = threadIdx.x; g < ng; g += blockDim.x)
      s_den[g] = scalar_den_row(scale[row * ng + g], offset[row * ng + g], gamma1[row], L,
                                anchored, inv_tau2);
    __syncthreads();
  }
  // the per-weight loop, instantiated once per precision regime and prior so
  // that the row-uniform choices cost no branch per weight
  auto weights = [&](auto prec, auto anch) -> float {
    constexpr bool PRECISE = decltype(prec)::value;
    constexpr bool ANCH = decltype(anch)::value;
    float acc = 0.0f;
    // ROW_UNROLL weights per thread and pass, all loads issued before the
    // first is used
    for (int64_t j0 = threadIdx.x; j0 < n; j0 += ROW_UNROLL * blockDim.x) {
      float rv[ROW_UNROLL], wv[ROW_UNROLL];
#pragma unroll
      for (int u = 0; u < ROW_UNROLL; ++u) {
        const int64_t j = j0 + (int64_t)u * blockDim.x;
        rv[u] = j < n ? R1[row * n + j] : 0.0f;
        wv[u] = (ANCH && j < n) ? W[row * n + j] : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < ROW_UNROLL; ++u) {
        const int64_t j = j0 + (int64_t)u * blockDim.x;
        if (j < n) {
          const int64_t o = row * n + j;
          float xh, ks, v;
          if constexpr (GROUPED) {
            const ScalarDen& cg = s_den[j / G];  // uniform over a warp (G % 32 == 0)
            v = cg.precise ? scalar_den_elem<true, ANCH>(cg, rv[u], wv[u], xh, ks)
                           : scalar_den_elem<false, ANCH>(cg, rv[u], wv[u], xh, ks);
          } else {
            v = scalar_den_elem<PRECISE, ANCH>(c, rv[u], wv[u], xh, ks);
          }
          xhat[o] = xh;
          if (vblock) vblock[o] = v;
          if (idx) idx[o] = (uint16_t)(int)ks;
          acc += v;
        }
      }
    }
    return acc;
  };
  using T_ = std::true_type;
  using F_ = std::false_type;
  const bool pr = !GROUPED && c.precise;  // grouped rows choose the regime per group
  const float acc = anchored ? (pr ? weights(T_{}, T_{}) : weights(F_{}, T_{}))
                             : (pr ? weights(T_{}, F_{}) : weights(F_{}, F_{}));
  const double tot = block_sum((double)acc, ds);
  if (threadIdx.x == 0) vsum[row] = tot;
}

// ------------------------------------------------------- vector denoiser ---
// One thread per block of 8 weights; the codebook streams through shared
// memory in chunks that every thread of the CTA reads in lock step.
constexpr int VEC_THREADS = 128;
constexpr int VEC_CHUNK = 512;

struct VecDenoiseArgs {
  const float* R1;
  const double* gamma1;
  const float* scale;
  const float* offset;
  int64_t m, n;
  int K;
  const float* cb;       // K x 8
  const float* cb_norm;  // K
  const float* W;        // anchor (nullable)
  const double* gamma1_0;
  double inv_tau2;
  float* xhat;
  float* vblock;
  uint16_t* idx;
  int nearest_only;      // 1: only the argmax (nearest codeword) into idx
};

__global__ void __launch_bounds__(VEC_THREADS) k_denoise_vec(VecDenoiseArgs a) {
  __shared__ float scb[VEC_CHUNK][9];
  const int64_t B = a.n / 8;
  const int64_t blk = (int64_t)blockIdx.x * VEC_THREADS + threadIdx.x;
  const bool active = blk < a.m * B;
  const int64_t row = active ? blk / B : 0;
  float t[8];
  double t64[8];
  float g = 0.0f;
  if (active) {
    const double sc = a.scale[row];
    const double sc2 = sc * sc;
    const float* r = a.R1 + blk * 8;
    double gg = 1.0, ga = 0.0;
    if (!a.nearest_only) {
      gg = a.gamma1[row] * sc2;
      ga = a.W ? a.inv_tau2 : 0.0;  // anchor: tau codebook units wide
    }
    g = (float)fmin(gg + ga, 1e30);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      double ti = (double)r[i] / sc;
      if (a.W && !a.nearest_only) ti = (gg * ti + ga * ((double)a.W[blk * 8 + i] / sc)) / (gg + ga);
      t64[i] = ti;
      t[i] = (float)ti;
    }
  }
  // pass 1: best score  s(c) = c.t - |c|^2/2  (logit = g s + const)
  float best = -INFINITY;
  int bidx = 0;
  for (int c0 = 0; c0 < a.K; c0 += VEC_CHUNK) {
    const int cn = min(VEC_CHUNK, a.K - c0);
    __syncthreads();
    for (int e = threadIdx.x; e < cn * 9; e += VEC_THREADS) {
      const int c = e / 9, i = e % 9;
      scb[c][i] = (i < 8) ? a.cb[(int64_t)(c0 + c) * 8 + i] : a.cb_norm[c0 + c];
    }
    __syncthreads();
    if (active) {
      for (int c = 0; c < cn; ++c) {
        float s = -0.5f * scb[c][8];
#pragma unroll
        for (int i = 0; i < 8; ++i) s = fmaf(scb[c][i], t[i], s);
        if (s > best) {
          best = s;
          bidx = c0 + c;
        }
      }
    }
  }
  if (a.nearest_only) {
    if (active) a.idx[blk] = (uint16_t)bidx;
    return;
  }
  // pass 2: moments centred on the argmax codeword c*.  With dc = c - c*
  // and tp = t - c*, the logit relative to the best is g (dc.tp - |dc|^2/2);
  // its two terms cancel (both O(1) for the codewords that matter), so it is
  // formed in fp64 before the fp32 exponential.
  float cs[8];
  double tp[8];
  const double gd = (double)g;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    cs[i] = active ? a.cb[(int64_t)bidx * 8 + i] : 0.0f;
    tp[i] = t64[i] - (double)cs[i];
  }
  float S0 = 0.0f, m2 = 0.0f, m1[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m1[i] = 0.0f;
  for (int c0 = 0; c0 < a.K; c0 += VEC_CHUNK) {
    const int cn = min(VEC_CHUNK, a.K - c0);
    __syncthreads();
    for (int e = threadIdx.x; e < cn * 9; e += VEC_THREADS) {
      const int c = e / 9, i = e % 9;
      scb[c][i] = (i < 8) ? a.cb[(int64_t)(c0 + c) * 8 + i] : a.cb_norm[c0 + c];
    }
    __syncthreads();
    if (active) {
      for (int c = 0; c < cn; ++c) {
        float dc[8];
        double dot = 0.0, nn = 0.0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const double d = (double)scb[c][i] - (double)cs[i];  // exact
          dc[i] = (float)d;
          dot = fma(d, tp[i], dot);
          nn = fma(d, d, nn);
        }
        const float q = __expf((float)(gd * (dot - 0.5 * nn)));
        S0 += q;
        m2 = fmaf(q, (float)nn, m2);
#pragma unroll
        for (int i = 0; i < 8; ++i) m1[i] = fmaf(q, dc[i], m1[i]);
      }
    }
  }
  if (!active) return;
  const float sc = a.scale[row], off = a.offset[row];
  const float inv = 1.0f / S0;
  float mm = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float mi = m1[i] * inv;
    mm = fmaf(mi, mi, mm);
    a.xhat[blk * 8 + i] = fmaf(sc, cs[i] + mi, off);
  }
  const float var = fmaxf(m2 * inv - mm, 0.0f);
  a.vblock[blk] = (float)((double)sc * sc * var);
  if (a.idx) a.idx[blk] = (uint16_t)bidx;
}

// per-row sum of the block variances (deterministic)
__global__ void __launch_bounds__(ROW_THREADS)
    k_row_sum(const float* __restrict__ v, int64_t B, double* __restrict__ out) {
  __shared__ double ds[33];
  const int64_t row = blockIdx.x;
  double acc = 0.0;
  for (int64_t j = threadIdx.x; j < B; j += blockDim.x) acc += (double)v[row * B + j];
  acc = block_sum(acc, ds);
  if (threadIdx.x == 0) out[row] = acc;
}

// ------------------------------------------------- extrinsic d -> linear ---
// Row scalars: alpha1 = gamma1 vsum / n and gamma2 = gamma1 (1 - alpha1) /
// alpha1, both clipped (clips counted); returns 1 / (1 - alpha1).
__device__ __forceinline__ float d2l_row(double g1, double vsum, int64_t n, double g0, double glo,
                                         double ghi, double amin, double amax, double* gamma2,
                                         int32_t* clamps) {
  int cnt = 0;
  const double a1 = clip_count(g1 * vsum / (double)n, amin, amax, &cnt);
  *gamma2 = clip_count(g1 * (1.0 - a1) / a1, glo * g0, ghi * g0, &cnt);
  if (clamps) *clamps += cnt;
  return (float)(1.0 / (1.0 - a1));
}

// alpha1 = gamma1 vsum / n (clipped), gamma2 = gamma1 (1 - alpha1)/alpha1
// (clipped), r2 = r1 + (xhat1 - r1)/(1 - alpha1)  [= (xhat1 - alpha1 r1)/
// (1 - alpha1) = (eta1 xhat1 - gamma1 r1)/gamma2].  Also writes the GEMM1
// operand w - r2 split for the tensor cores (K = n view, zero up to ldn).
__global__ void __launch_bounds__(ROW_THREADS)
    k_extrinsic_d2l(const float* __restrict__ W, int64_t n, const float* __restrict__ R1,
                    const double* __restrict__ gamma1, const float* __restrict__ X1,
                    const double* __restrict__ vsum, const double* __restrict__ gamma1_0,
                    double glo, double ghi, double amin, double amax, float* __restrict__ R2,
                    __half* __restrict__ ahi, __half* __restrict__ alo, int64_t lda, int64_t ldn,
                    float* __restrict__ a_unscale, double* __restrict__ gamma2,
                    int32_t* __restrict__ clamps) {
  __shared__ float cf;
  __shared__ float fs[33];
  const int64_t row = blockIdx.x;
  if (threadIdx.x == 0)
    cf = d2l_row(gamma1[row], vsum[row], n, gamma1_0[row], glo, ghi, amin, amax, gamma2 + row,
                 clamps ? clamps + row : nullptr);
  __syncthreads();
  const float c = cf;
  float mx = 0.0f;
  for (int64_t j0 = threadIdx.x; j0 < n; j0 += ROW_UNROLL * blockDim.x) {
    float r1v[ROW_UNROLL], xv[ROW_UNROLL], wv[ROW_UNROLL];
#pragma unroll
    for (int u = 0; u < ROW_UNROLL; ++u) {
      const int64_t j = j0 + (int64_t)u * blockDim.x;
      const bool in = j < n;
      r1v[u] = in ? R1[row * n + j] : 0.0f;
      xv[u] = in ? X1[row * n + j] : 0.0f;
      wv[u] = in ? W[row * n + j] : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < ROW_UNROLL; ++u) {
      const int64_t j = j0 + (int64_t)u * blockDim.x;
      if (j < n) {
        const float r2 = fmaf(c, xv[u] - r1v[u], r1v[u]);
        R2[row * n + j] = r2;
        mx = fmaxf(mx, fabsf(wv[u] - r2));
      }
    }
  }
  mx = block_reduce(mx, MaxF(), fs);
  const int ex = split_exponent(mx);
  const float down = ldexpf(1.0f, -ex);
  for (int64_t j0 = threadIdx.x; j0 < ldn; j0 += ROW_UNROLL * blockDim.x) {
    float xv[ROW_UNROLL];
#pragma unroll
    for (int u = 0; u < ROW_UNROLL; ++u) {
      const int64_t j = j0 + (int64_t)u * blockDim.x;
      xv[u] = (j < n) ? (W[row * n + j] - R2[row * n + j]) * down : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < ROW_UNROLL; ++u) {
      const int64_t j = j0 + (int64_t)u * blockDim.x;
      if (j < ldn) split_store(xv[u], ahi, alo, row * lda + j);
    }
  }
  if (threadIdx.x == 0) a_unscale[row] = ldexpf(1.0f, ex);
}

// ------------------------------------------------------ M-step finisher ---
// The projection GEMM's linear epilogue left, per row and column tile of
// 128 rank components, sum F and sum F^2 u^2 + s^2/(beta s^2 + gamma2) with
// u = s p', F = gamma2/(beta s^2 + gamma2) (the MPQ note's key design 2:
// 1/beta_hat = (1/r) sum_l [(gamma2/(beta s_l^2 + gamma2))^2 u_l^2 +
// s_l^2/(beta s_l^2 + gamma2)]).  One warp per row adds the tiles in fp64 in
// a fixed order, then: alpha2 = [sum F + n - r]/n (reading R6), beta_hat, beta <-
// (1 - rho) beta + rho beta_hat (R7), gamma1' = gamma2 (1 - alpha2)/alpha2
// and the l2d coefficients 1/(1 - alpha2), alpha2/(1 - alpha2), each clipped
// (R5), and the second GEMM's row scale 2^(e_row + e_bound).
// The M-step's per-row finish (one warp per row): lane l adds the column
// groups l, l + 32, ... in fp64, then a butterfly over the lanes (a fixed
// order: the sums are deterministic); lane 0 forms alpha2, beta_hat, the
// damped beta, gamma1' and the l2d coefficients.  Shared by the finisher
// kernel and the fused row kernel that runs it in its prologue.

__device__ __forceinline__ void linear_finish_row(const LinFinish& f, int64_t row, int lane) {
  double a2tot = 0.0, bstot = 0.0;
  for (int t = lane; t < f.ntiles; t += 32) {
    const float2 v = f.part[(int64_t)t * f.m + row];
    a2tot += (double)v.x;
    bstot += (double)v.y;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a2tot += __shfl_xor_sync(0xffffffffu, a2tot, o);
    bstot += __shfl_xor_sync(0xffffffffu, bstot, o);
  }
  if (lane != 0) return;
  if (f.q_unscale) f.q_unscale[row] = ldexpf(f.a_unscale[row], f.e_bound);
  int cnt = 0;
  const double b = f.beta[row], g2 = f.gamma2[row];
  const double alpha2 = (a2tot + (double)(f.n - f.r)) / (double)f.n;
  const double bhat = (double)f.r / bstot;
  f.beta[row] = (1.0 - f.damping) * b + f.damping * bhat;
  const double a2 = clip_count(alpha2, f.amin, f.amax, &cnt);
  const double g0 = f.gamma1_0[row];
  f.gamma1_out[row] = clip_count(g2 * (1.0 - a2) / a2, f.glo * g0, f.ghi * g0, &cnt);
  f.coef[row] = 1.0 / (1.0 - a2);
  f.kappa[row] = a2 / (1.0 - a2);
  if (f.alpha2_out) f.alpha2_out[row] = alpha2;
  if (f.beta_hat_out) f.beta_hat_out[row] = bhat;
  if (f.clamps) f.clamps[row] += cnt;
}

__global__ void __launch_bounds__(256) k_linear_finish(const __grid_constant__ LinFinish f) {
  const int lane = threadIdx.x & 31;
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (row >= f.m) return;
  linear_finish_row(f, row, lane);
}

// ------------------------------------------------- extrinsic linear -> d ---
// r1' = (xhat2 - alpha2 r2)/(1 - alpha2) = (eta2 xhat2 - gamma2 r2)/gamma1'.
//   r < n: G = xhat2 - r2:  r1' = r2 + coef G,              xhat2 = r2 + G
//   r = n: G = xhat2 - w:   r1' = w + kappa (w - r2) + coef G,  xhat2 = w + G
__global__ void __launch_bounds__(ROW_THREADS)
    k_extrinsic_l2d(const float* __restrict__ W, const float* __restrict__ R2,
                    const float* __restrict__ G, int64_t n, const double* __restrict__ coef,
                    const double* __restrict__ kappa, int full_rank, float* __restrict__ R1,
                    float* __restrict__ xhat2) {
  const int64_t row = blockIdx.x;
  const float c = (float)coef[row];
  const float k = (float)kappa[row];
  for (int64_t j0 = threadIdx.x; j0 < n; j0 += ROW_UNROLL * blockDim.x) {
    float gv[ROW_UNROLL], r2v[ROW_UNROLL], wv[ROW_UNROLL];
#pragma unroll
    for (int u = 0; u < ROW_UNROLL; ++u) {
      const int64_t j = j0 + (int64_t)u * blockDim.x;
      const bool in = j < n;
      gv[u] = in ? G[row * n + j] : 0.0f;
      r2v[u] = in ? R2[row * n + j] : 0.0f;
      wv[u] = (in && full_rank) ? W[row * n + j] : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < ROW_UNROLL; ++u) {
      const int64_t j = j0 + (int64_t)u * blockDim.x;
      if (j >= n) continue;
      const int64_t o = row * n + j;
      const float g = gv[u], r2 = r2v[u];
      if (full_rank) {
        const float w = wv[u];
        R1[o] = fmaf(c, g, fmaf(k, w - r2, w));
        if (xhat2) xhat2[o] = w + g;
      } else {
        R1[o] = fmaf(c, g, r2);
        if (xhat2) xhat2[o] = r2 + g;
      }
    }
  }
}

// ------------------------------------------------ fused scalar VAMP row ---
// One row of a scalar (d = 1) VAMP iteration in one pass over HBM: the
// extrinsic linear -> denoiser step (r1 from the GEMM output G, r2 and w, as
// in k_extrinsic_l2d; r1 = w in the first iteration), the denoiser
// (scalar_den_elem), and the extrinsic denoiser -> linear step with the split
// GEMM operand w - r2 (as in k_extrinsic_d2l).  r1 and x_hat1 of the row stay
// in shared memory between the two halves; each arithmetic step is the one
// of the separate kernels, in the same order.  MAP = 1: the marginal MAP
// after the last iteration (l2d and the denoiser's argmax only).
// first: 0 = r1 from the l2d step; 1 = r1 = w (the solve's first iteration);
// 2 = r1 read from G (an injected cavity, for the per-stage hook).  R1o, if
// not NULL, receives the r1 the kernel forms.
constexpr int FUSED_MAX_THREADS = 1024;

template <int MAP, bool GROUPED>
__global__ void __launch_bounds__(FUSED_MAX_THREADS)
    k_vamp_row_scalar(const float* __restrict__ W, const float* __restrict__ G,
                      float* __restrict__ R2, int64_t n, int gsize, int first, int full_rank,
                      const double* coef, const double* kappa,
                      const double* gamma1, const float* __restrict__ scale,
                      const float* __restrict__ offset, int L, int anchored,
                      const double* __restrict__ gamma1_0, double inv_tau2, double glo,
                      double ghi, double amin, double amax, __half* __restrict__ ahi,
                      __half* __restrict__ alo, int64_t lda, int64_t ldn,
                      float* __restrict__ a_unscale, double* gamma2,
                      int32_t* clamps, uint16_t* __restrict__ idx,
                      float* __restrict__ R1o, const __grid_constant__ LinFinish fin, int has_fin) {
  extern __shared__ __align__(16) float vrow[];  // the row: r1 (then r2), x_hat1 (then w - r2), w
  __shared__ double ds[33];
  __shared__ float fs[33];
  __shared__ float cf_s;
  const int nn = (int)n;  // a row fits in shared memory: 32-bit in-row indices
  const int np4 = (nn + 3) & ~3;
  float* s_r = vrow;
  float* s_x = vrow + np4;
  float* s_w = vrow + 2 * np4;
  ScalarDen* s_den = reinterpret_cast<ScalarDen*>(vrow + 3 * np4);  // GROUPED: one per group
  const int64_t row = blockIdx.x;
  const float* Wr = W + row * n;
  const float* Gr = G + row * n;
  float* R2r = R2 + row * n;
  // gamma1, coef and kappa may be written by this kernel's own prologue (the
  // previous linear step's M-step finish for this row): no __restrict__ on
  // them, and the reads go through L2 (ld.global.cg) after the barrier
  if (has_fin) {
    if (threadIdx.x < 32) linear_finish_row(fin, row, threadIdx.x);
    __syncthreads();
  }
  const double g1row = __ldcg(gamma1 + row);
  const int ng = GROUPED ? nn / gsize : 1;
  const ScalarDen c = scalar_den_row(scale[row * ng], offset[row * ng], g1row, L,
                                     anchored != 0, inv_tau2);
  if (GROUPED) {
    for (int g = threadIdx.x; g < ng; g += blockDim.x)
      s_den[g] = scalar_den_row(scale[row * ng + g], offset[row * ng + g], g1row, L,
                                anchored != 0, inv_tau2);
    __syncthreads();
  }
  const float lc = first ? 0.0f : (float)__ldcg(coef + row);
  const float lk = first ? 0.0f : (float)__ldcg(kappa + row);
  const bool injected = first == 2;
  float* R1or = R1o ? R1o + row * n : nullptr;
  const int bs = blockDim.x;
  // Rows of a multiple of 4 weights move as float4 (rows start 16-byte
  // aligned then): each thread takes VQ groups of 4 consecutive weights, their
  // loads in flight together.  Other rows go one weight at a time.
  constexpr int VQ = 1;  // more spills registers at the 64 a 1024-thread launch allows
  const bool vec = (nn & 3) == 0;
  const int nq = nn >> 2;
  auto pass1 = [&](auto prec, auto anch) -> float {
    constexpr bool PRECISE = decltype(prec)::value;
    constexpr bool ANCH = decltype(anch)::value;
    float acc = 0.0f;
    // weight j: r1 from the l2d step, then the denoiser; x_hat1 returned
    auto one = [&](const int j, const float g, const float r2, const float w, float& r1) -> float {
      r1 = injected ? g
           : first  ? w
           : full_rank ? fmaf(lc, g, fmaf(lk, w - r2, w))
                       : fmaf(lc, g, r2);
      if (R1or) R1or[j] = r1;
      float xh, ks, v;
      if constexpr (GROUPED) {
        const ScalarDen& cg = s_den[j / gsize];  // uniform over a warp (gsize % 32 == 0)
        v = cg.precise ? scalar_den_elem<true, ANCH, !MAP>(cg, r1, w, xh, ks)
                       : scalar_den_elem<false, ANCH, !MAP>(cg, r1, w, xh, ks);
      } else {
        v = scalar_den_elem<PRECISE, ANCH, !MAP>(c, r1, w, xh, ks);
      }
      if (MAP) idx[row * n + j] = (uint16_t)(int)ks;
      acc += v;
      return xh;
    };
    if (vec) {
      const float4* G4 = reinterpret_cast<const float4*>(Gr);
      const float4* R4 = reinterpret_cast<const float4*>(R2r);
      const float4* W4 = reinterpret_cast<const float4*>(Wr);
      for (int q0 = threadIdx.x; q0 < nq; q0 += VQ * bs) {
        float4 gv[VQ], rv[VQ], wv[VQ];
#pragma unroll
        for (int u = 0; u < VQ; ++u) {
          const int q = q0 + u * bs;
          const bool in = q < nq;
          const float4 z = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          gv[u] = (in && first != 1) ? G4[q] : z;
          rv[u] = (in && !first) ? R4[q] : z;
          wv[u] = in ? W4[q] : z;
        }
#pragma unroll
        for (int u = 0; u < VQ; ++u) {
          const int q = q0 + u * bs;
          if (q >= nq) continue;
          float4 r1, xh;
          xh.x = one(4 * q, gv[u].x, rv[u].x, wv[u].x, r1.x);
          xh.y = one(4 * q + 1, gv[u].y, rv[u].y, wv[u].y, r1.y);
          xh.z = one(4 * q + 2, gv[u].z, rv[u].z, wv[u].z, r1.z);
          xh.w = one(4 * q + 3, gv[u].w, rv[u].w, wv[u].w, r1.w);
          if (!MAP) {
            reinterpret_cast<float4*>(s_r)[q] = r1;
            reinterpret_cast<float4*>(s_x)[q] = xh;
            reinterpret_cast<float4*>(s_w)[q] = wv[u];
          }
        }
      }
    } else {
      for (int j = threadIdx.x; j < nn; j += bs) {
        const float w = Wr[j];
        float r1;
        const float xh = one(j, (first == 1) ? 0.0f : Gr[j], first ? 0.0f : R2r[j], w, r1);
        if (!MAP) {
          s_r[j] = r1;
          s_x[j] = xh;
          s_w[j] = w;
        }
      }
    }
    return acc;
  };
  using T_ = std::true_type;
  using F_ = std::false_type;
  const bool pr = !GROUPED && c.precise;  // grouped rows choose the regime per group
  const float acc = anchored ? (pr ? pass1(T_{}, T_{}) : pass1(F_{}, T_{}))
                             : (pr ? pass1(T_{}, F_{}) : pass1(F_{}, F_{}));
  if (MAP) return;
  const double vsum = block_sum((double)acc, ds);  // its barriers also publish the row
  if (threadIdx.x == 0)
    cf_s = d2l_row(g1row, vsum, n, gamma1_0[row], glo, ghi, amin, amax, gamma2 + row,
                   clamps ? clamps + row : nullptr);
  __syncthreads();
  const float cf = cf_s;
  // r2 = r1 + cf (x_hat1 - r1) out, and w - r2 kept (in s_x) for the split
  float mx = 0.0f;
  if (vec) {
    for (int q = threadIdx.x; q < nq; q += bs) {
      const float4 r1 = reinterpret_cast<const float4*>(s_r)[q];
      const float4 xh = reinterpret_cast<const float4*>(s_x)[q];
      const float4 w = reinterpret_cast<const float4*>(s_w)[q];
      float4 r2, d;
      r2.x = fmaf(cf, xh.x - r1.x, r1.x);
      r2.y = fmaf(cf, xh.y - r1.y, r1.y);
      r2.z = fmaf(cf, xh.z - r1.z, r1.z);
      r2.w = fmaf(cf, xh.w - r1.w, r1.w);
      reinterpret_cast<float4*>(R2r)[q] = r2;
      d.x = w.x - r2.x;
      d.y = w.y - r2.y;
      d.z = w.z - r2.z;
      d.w = w.w - r2.w;
      reinterpret_cast<float4*>(s_x)[q] = d;
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(d.x), fabsf(d.y)), fmaxf(fabsf(d.z), fabsf(d.w))));
    }
  } else {
    for (int j = threadIdx.x; j < nn; j += bs) {
      const float r1 = s_r[j];
      const float r2 = fmaf(cf, s_x[j] - r1, r1);
      R2r[j] = r2;
      const float d = s_w[j] - r2;
      s_x[j] = d;
      mx = fmaxf(mx, fabsf(d));
    }
  }
  mx = block_reduce(mx, MaxF(), fs);  // its barriers also publish w - r2
  const int ex = split_exponent(mx);
  const float down = ldexpf(1.0f, -ex);
  __half* ahr = ahi + row * lda;
  __half* alr = alo + row * lda;
  const int ldnn = (int)ldn;  // a multiple of 64 (and lda even): whole quads, 8-byte aligned
  for (int q = threadIdx.x; q < ldnn / 4; q += bs) {
    const int j = 4 * q;
    float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (vec && j < nn) {
      const float4 d = reinterpret_cast<const float4*>(s_x)[q];
      x[0] = d.x * down;
      x[1] = d.y * down;
      x[2] = d.z * down;
      x[3] = d.w * down;
    } else if (!vec) {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (j + e < nn) x[e] = s_x[j + e] * down;
    }
    split_store4(x, ahr, alr, j);
  }
  if (threadIdx.x == 0) a_unscale[row] = ldexpf(1.0f, ex);
}

// --------------------------------------------------- residual / energies ---
__global__ void __launch_bounds__(ROW_THREADS)
    k_residual(const float* __restrict__ W, int64_t n, int d, int G, const float* __restrict__ cb,
               const float* __restrict__ scale, const float* __restrict__ offset,
               const uint16_t* __restrict__ idx, float* __restrict__ E,
               float* __restrict__ w_hat) {
  const int64_t row = blockIdx.x;
  const int64_t ng = G ? n / G : 1;  // grids per row (G = 0: one)
  const int64_t B = n / d;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    const int64_t gi = row * ng + (G ? j / G : 0);
    const float sc = scale[gi], off = offset[gi];
    const int k = idx[row * B + j / d];  // in range: sanitised on entry
    const float c = (d == 1) ? (float)k : cb[(int64_t)k * d + (j % d)];
    const float wh = fmaf(sc, c, off);
    E[row * n + j] = W[row * n + j] - wh;
    if (w_hat) w_hat[row * n + j] = wh;
  }
}

// residual w - w_hat split for the tensor cores (K = n view), w_hat optional
__global__ void __launch_bounds__(ROW_THREADS)
    k_residual_split(const float* __restrict__ W, int64_t n, int d, int G,
                     const float* __restrict__ cb, const float* __restrict__ scale,
                     const float* __restrict__ offset, const uint16_t* __restrict__ idx,
                     float* __restrict__ w_hat, __half* __restrict__ ahi,
                     __half* __restrict__ alo, int64_t lda, int64_t ldn,
                     float* __restrict__ a_unscale) {
  __shared__ float fs[33];
  const int64_t row = blockIdx.x;
  const int64_t ng = G ? n / G : 1;  // grids per row (G = 0: one)
  const int64_t B = n / d;
  float mx = 0.0f;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    const int64_t gi = row * ng + (G ? j / G : 0);
    const float sc = scale[gi], off = offset[gi];
    const int k = idx[row * B + j / d];
    const float c = (d == 1) ? (float)k : cb[(int64_t)k * d + (j % d)];
    const float wh = fmaf(sc, c, off);
    if (w_hat) w_hat[row * n + j] = wh;
    mx = fmaxf(mx, fabsf(W[row * n + j] - wh));
  }
  mx = block_reduce(mx, MaxF(), fs);
  const int ex = split_exponent(mx);
  const float down = ldexpf(1.0f, -ex);
  for (int64_t j = threadIdx.x; j < ldn; j += blockDim.x) {
    float x = 0.0f;
    if (j < n) {
      const int64_t gi = row * ng + (G ? j / G : 0);
      const int k = idx[row * B + j / d];
      const float c = (d == 1) ? (float)k : cb[(int64_t)k * d + (j % d)];
      x = (W[row * n + j] - fmaf(scale[gi], c, offset[gi])) * down;
    }
    split_store(x, ahi, alo, row * lda + j);
  }
  if (threadIdx.x == 0) a_unscale[row] = ldexpf(1.0f, ex);
}

__global__ void __launch_bounds__(ROW_THREADS)
    k_energy_rows(const float* __restrict__ P, int64_t r, const double* __restrict__ s,
                  float* __restrict__ energy) {
  __shared__ double ds[33];
  const int64_t row = blockIdx.x;
  double acc = 0.0;
  for (int64_t l = threadIdx.x; l < r; l += blockDim.x) {
    const double u = s[l] * (double)P[row * r + l];
    acc += u * u;
  }
  acc = block_sum(acc, ds);
  if (threadIdx.x == 0) energy[row] = (float)(0.5 * acc);
}

__global__ void k_sanitize_idx(uint16_t* __restrict__ idx, int64_t count, int K, int* status) {
  bool bad = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x) {
    if (idx[i] >= K) {
      idx[i] = (uint16_t)(K - 1);
      bad = true;
    }
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, STATUS_BADINDEX);
}

__global__ void k_check_finite(const float* __restrict__ x, int64_t count, int* status) {
  bool bad = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x)
    bad |= !isfinite(x[i]);
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, STATUS_NONFINITE);
}

inline unsigned rows_grid(int64_t m) { return (unsigned)m; }

}  // namespace

// =============================================================== launchers ==

mpq_status launch_init(const mpq_plan_s* p, const float* W, int64_t m, int given, float* scale,
                       float* offset, uint16_t* idx, double* gamma1_0, cudaStream_t st,
                       bool rtn) {
  if (m <= 0) return MPQ_OK;
  if (p->d == 1) {
    {
      ProfScope ps_("k_init_scalar", st);
      if (p->G)
        k_init_scalar_groups<<<rows_grid(m), ROW_THREADS, 0, st>>>(W, p->n, p->K, p->G, given,
                                                                   scale, offset, idx, gamma1_0,
                                                                   p->status);
      else
        k_init_scalar<<<rows_grid(m), ROW_THREADS, 0, st>>>(W, p->n, p->K, given, scale, offset,
                                                            idx, gamma1_0, p->status);
    }
    count_launch();
    return check_launch("k_init_scalar");
  }
  {
    ProfScope ps_("k_init_rms", st);
    k_init_rms<<<rows_grid(m), ROW_THREADS, 0, st>>>(W, p->n, given, scale, offset, p->status);
  }
  count_launch();
  MPQ_TRY(check_launch("k_init_rms"));
  if (!rtn) return MPQ_OK;  // the scale alone (idx and gamma1_0 are not needed)
  const int64_t nb = m * (p->n / 8);
  if (p->vec_tc) {
    MPQ_TRY(launch_denoise_vec_tc(p, W, nullptr, scale, offset, m, nullptr, nullptr, 0.0, nullptr,
                                  nullptr, idx, 1, st));
  } else {
  VecDenoiseArgs a{};
  a.R1 = W;
  a.scale = scale;
  a.offset = offset;
  a.m = m;
  a.n = p->n;
  a.K = p->K;
  a.cb = p->cb;
  a.cb_norm = p->cb_norm;
  a.idx = idx;
  a.nearest_only = 1;
  {
    ProfScope ps_("k_denoise_vec", st);
    k_denoise_vec<<<(unsigned)cdiv(nb, VEC_THREADS), VEC_THREADS, 0, st>>>(a);
  }
  count_launch();
  MPQ_TRY(check_launch("k_denoise_vec(nearest)"));
  }
  {
    ProfScope ps_("k_gamma0_vec", st);
    k_gamma0_vec<<<rows_grid(m), ROW_THREADS, 0, st>>>(W, p->n, p->cb, scale, offset, idx, gamma1_0);
  }
  count_launch();
  return check_launch("k_gamma0_vec");
}

mpq_status launch_denoise(const mpq_plan_s* p, const float* R1, const double* gamma1,
                          const float* scale, const float* offset, int64_t m, const float* W,
                          const double* gamma1_0, float* xhat1, float* vblock, double* vsum,
                          uint16_t* idx, cudaStream_t st, bool map_only) {
  if (m <= 0) return MPQ_OK;
  const bool anchored = std::isfinite(p->params.tau);
  const double inv_tau2 = anchored ? 1.0 / (p->params.tau * p->params.tau) : 0.0;
  if (p->d == 1) {
    {
      ProfScope ps_("k_denoise_scalar", st);
      if (p->G) {
        const size_t smem = sizeof(ScalarDen) * (size_t)(p->n / p->G);
        MPQ_CUDA(cudaFuncSetAttribute(k_denoise_scalar<true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        k_denoise_scalar<true><<<rows_grid(m), ROW_THREADS, smem, st>>>(
            R1, gamma1, scale, offset, p->n, p->K, p->G, anchored ? W : nullptr, gamma1_0,
            inv_tau2, xhat1, vblock, vsum, idx);
      } else {
        k_denoise_scalar<false><<<rows_grid(m), ROW_THREADS, 0, st>>>(
            R1, gamma1, scale, offset, p->n, p->K, 0, anchored ? W : nullptr, gamma1_0, inv_tau2,
            xhat1, vblock, vsum, idx);
      }
    }
    count_launch();
    return check_launch("k_denoise_scalar");
  }
  if (vblock == nullptr) return fail(MPQ_ERR_INVALID_ARG, "vector denoiser needs vblock");
  if (p->vec_tc) {
    MPQ_TRY(launch_denoise_vec_tc(p, R1, gamma1, scale, offset, m, anchored ? W : nullptr,
                                  gamma1_0, inv_tau2, xhat1, vblock, idx,
                                  map_only && idx ? 2 : 0, st));
    if (map_only && idx) return MPQ_OK;  // no x_hat, no variance sums
  } else {
  VecDenoiseArgs a{};
  a.R1 = R1;
  a.gamma1 = gamma1;
  a.scale = scale;
  a.offset = offset;
  a.m = m;
  a.n = p->n;
  a.K = p->K;
  a.cb = p->cb;
  a.cb_norm = p->cb_norm;
  a.W = anchored ? W : nullptr;
  a.gamma1_0 = gamma1_0;
  a.inv_tau2 = inv_tau2;
  a.xhat = xhat1;
  a.vblock = vblock;
  a.idx = idx;
  a.nearest_only = 0;
  const int64_t nb = m * (p->n / 8);
  {
    ProfScope ps_("k_denoise_vec", st);
    k_denoise_vec<<<(unsigned)cdiv(nb, VEC_THREADS), VEC_THREADS, 0, st>>>(a);
  }
  count_launch();
  MPQ_TRY(check_launch("k_denoise_vec"));
  }
  {
    ProfScope ps_("k_row_sum", st);
    k_row_sum<<<rows_grid(m), ROW_THREADS, 0, st>>>(vblock, p->n / 8, vsum);
  }
  count_launch();
  return check_launch("k_row_sum");
}

mpq_status launch_extrinsic_d2l(const mpq_plan_s* p, const float* W, int64_t m, const float* R1,
                                const double* gamma1, const float* xhat1, const double* vsum,
                                const double* gamma1_0, float* R2, SplitOperand* As,
                                double* gamma2, int32_t* clamps, cudaStream_t st) {
  if (m <= 0) return MPQ_OK;
  const mpq_params& q = p->params;
  {
    ProfScope ps_("k_extrinsic_d2l", st);
    k_extrinsic_d2l<<<rows_grid(m), ROW_THREADS, 0, st>>>(
        W, p->n, R1, gamma1, xhat1, vsum, gamma1_0, q.gamma_lo_rel, q.gamma_hi_rel, q.alpha_min,
        q.alpha_max, R2, As->hi, As->lo, As->ld, round_up(p->n, 64), As->row_unscale, gamma2,
        clamps);
  }
  count_launch();
  return check_launch("k_extrinsic_d2l");
}

LinFinish make_lin_finish(const mpq_plan_s* p, int64_t m, const float2* part, int ntiles,
                          int e_bound, const float* a_unscale, float* q_unscale,
                          const double* gamma2, const double* gamma1_0, double* beta,
                          double* gamma1_out, double* coef, double* kappa, double* alpha2,
                          double* beta_hat, int32_t* clamps) {
  const mpq_params& q = p->params;
  LinFinish f;
  f.part = part;
  f.ntiles = ntiles;
  f.e_bound = e_bound;
  f.m = m;
  f.n = p->n;
  f.r = p->r;
  f.a_unscale = a_unscale;
  f.q_unscale = q_unscale;
  f.gamma2 = gamma2;
  f.gamma1_0 = gamma1_0;
  f.beta = beta;
  f.damping = q.damping;
  f.glo = q.gamma_lo_rel;
  f.ghi = q.gamma_hi_rel;
  f.amin = q.alpha_min;
  f.amax = q.alpha_max;
  f.gamma1_out = gamma1_out;
  f.coef = coef;
  f.kappa = kappa;
  f.alpha2_out = alpha2;
  f.beta_hat_out = beta_hat;
  f.clamps = clamps;
  return f;
}

mpq_status launch_linear_finish(const mpq_plan_s* p, int64_t m, const float2* part, int ntiles,
                                int e_bound, const float* a_unscale, float* q_unscale,
                                const double* gamma2, const double* gamma1_0, double* beta,
                                double* gamma1_out, double* coef, double* kappa, double* alpha2,
                                double* beta_hat, int32_t* clamps, cudaStream_t st) {
  if (m <= 0) return MPQ_OK;
  const LinFinish f = make_lin_finish(p, m, part, ntiles, e_bound, a_unscale, q_unscale, gamma2,
                                      gamma1_0, beta, gamma1_out, coef, kappa, alpha2, beta_hat,
                                      clamps);
  {
    ProfScope ps_("k_linear_finish", st);
    k_linear_finish<<<(unsigned)cdiv(m * 32, 256), 256, 0, st>>>(f);
  }
  count_launch();
  return check_launch("k_linear_finish");
}

mpq_status launch_extrinsic_l2d(const mpq_plan_s* p, const float* W, int64_t m, const float* R2,
                                const float* G, const double* coef, const double* kappa,
                                float* R1_out, float* xhat2, cudaStream_t st) {
  if (m <= 0) return MPQ_OK;
  {
    ProfScope ps_("k_extrinsic_l2d", st);
    k_extrinsic_l2d<<<rows_grid(m), ROW_THREADS, 0, st>>>(W, R2, G, p->n, coef, kappa,
                                                          p->r == p->n ? 1 : 0, R1_out, xhat2);
  }
  count_launch();
  return check_launch("k_extrinsic_l2d");
}

// Threads per row of the fused scalar kernel: its shared memory holds two
// floats per weight; 0 when the row does not fit (the separate kernels run).
// (plus the per-group denoiser constants with group-wise grids)
int64_t vamp_row_smem(int64_t n, int G) {
  return 12 * ((n + 3) / 4 * 4) + (G ? (n / G) * (int64_t)sizeof(ScalarDen) : 0);
}

int vamp_row_threads(int64_t n, int G) {
  const int64_t bytes = vamp_row_smem(n, G);
  if (bytes <= 56 * 1024) return 256;    // 4 CTAs per SM
  if (bytes <= 112 * 1024) return 512;   // 2 CTAs per SM
  if (bytes <= 220 * 1024) return 1024;  // 1 CTA per SM
  return 0;
}

mpq_status launch_vamp_row_scalar(const mpq_plan_s* p, const float* W, int64_t m, int first,
                                  int map, const float* G, float* R2, const double* coef,
                                  const double* kappa, const double* gamma1, const float* scale,
                                  const float* offset, const double* gamma1_0, SplitOperand* As,
                                  double* gamma2, int32_t* clamps, uint16_t* idx, cudaStream_t st,
                                  float* R1o, const LinFinish* fin) {
  if (m <= 0) return MPQ_OK;
  const int threads = vamp_row_threads(p->n, p->G);
  if (p->d != 1 || threads == 0) return fail(MPQ_ERR_INVALID_ARG, "fused row kernel: d = 1 rows that fit");
  const mpq_params& q = p->params;
  const bool anchored = std::isfinite(q.tau);
  const double inv_tau2 = anchored ? 1.0 / (q.tau * q.tau) : 0.0;
  const size_t smem = (size_t)vamp_row_smem(p->n, p->G);
  using Kern = void (*)(const float*, const float*, float*, int64_t, int, int, int, const double*,
                        const double*, const double*, const float*, const float*, int, int,
                        const double*, double, double, double, double, double, __half*, __half*,
                        int64_t, int64_t, float*, double*, int32_t*, uint16_t*, float*,
                        const LinFinish, int);
  const Kern kern = p->G ? (map ? k_vamp_row_scalar<1, true> : k_vamp_row_scalar<0, true>)
                         : (map ? k_vamp_row_scalar<1, false> : k_vamp_row_scalar<0, false>);
  MPQ_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  {
    ProfScope ps_(map ? "k_vamp_row_scalar(map)" : "k_vamp_row_scalar", st);
    kern<<<rows_grid(m), threads, smem, st>>>(
        W, G, R2, p->n, p->G, first, p->r == p->n ? 1 : 0, coef, kappa, gamma1, scale, offset, p->K,
        anchored ? 1 : 0, gamma1_0, inv_tau2, q.gamma_lo_rel, q.gamma_hi_rel, q.alpha_min,
        q.alpha_max, As ? As->hi : nullptr, As ? As->lo : nullptr, As ? As->ld : 0,
        round_up(p->n, 64), As ? As->row_unscale : nullptr, gamma2, clamps, idx, R1o, fin ? *fin : LinFinish{}, fin ? 1 : 0);
  }
  count_launch();
  return check_launch("k_vamp_row_scalar");
}

mpq_status launch_residual_split(const mpq_plan_s* p, const float* W, int64_t m,
                                 const float* scale, const float* offset, const uint16_t* idx,
                                 SplitOperand* As, float* w_hat, cudaStream_t st) {
  if (m <= 0) return MPQ_OK;
  {
    ProfScope ps_("k_residual_split", st);
    k_residual_split<<<rows_grid(m), ROW_THREADS, 0, st>>>(W, p->n, p->d, p->G, p->cb, scale, offset,
                                                           idx, w_hat, As->hi, As->lo, As->ld,
                                                           round_up(p->n, 64), As->row_unscale);
  }
  count_launch();
  return check_launch("k_residual_split");
}

mpq_status launch_residual(const mpq_plan_s* p, const float* W, int64_t m, const float* scale,
                           const float* offset, const uint16_t* idx, float* E, float* w_hat,
                           cudaStream_t st) {
  if (m <= 0) return MPQ_OK;
  {
    ProfScope ps_("k_residual", st);
    k_residual<<<rows_grid(m), ROW_THREADS, 0, st>>>(W, p->n, p->d, p->G, p->cb, scale, offset, idx, E,
                                                     w_hat);
  }
  count_launch();
  return check_launch("k_residual");
}

mpq_status launch_energy_rows(const mpq_plan_s* p, int64_t m, const float* P, float* energy,
                              cudaStream_t st) {
  if (m <= 0) return MPQ_OK;
  {
    ProfScope ps_("k_energy_rows", st);
    k_energy_rows<<<rows_grid(m), ROW_THREADS, 0, st>>>(P, p->r, p->s64, energy);
  }
  count_launch();
  return check_launch("k_energy_rows");
}

mpq_status launch_sanitize_idx(const mpq_plan_s* p, uint16_t* idx, int64_t count, cudaStream_t st) {
  if (count <= 0) return MPQ_OK;
  const unsigned blocks = (unsigned)std::min<int64_t>(cdiv(count, 256), 148 * 8);
  {
    ProfScope ps_("k_sanitize_idx", st);
    k_sanitize_idx<<<blocks, 256, 0, st>>>(idx, count, p->K, p->status);
  }
  count_launch();
  return check_launch("k_sanitize_idx");
}

mpq_status launch_check_finite(const float* x, int64_t count, int* status, cudaStream_t st) {
  if (count <= 0) return MPQ_OK;
  const unsigned blocks = (unsigned)std::min<int64_t>(cdiv(count, 256), 148 * 8);
  {
    ProfScope ps_("k_check_finite", st);
    k_check_finite<<<blocks, 256, 0, st>>>(x, count, status);
  }
  count_launch();
  return check_launch("k_check_finite");
}

}  // namespace mpq
