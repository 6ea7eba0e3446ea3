// 4-bit activation quantizer of BitNet a4.8 (arXiv 2411.04965, §3.4):
//   quant_a4_kernel -- INT4 absmean (Eq. 6-7) or FP4 E2M1 MinMax (Eq. 8-9), and
//                      the ablation variants INT4 absmax, INT4 absmean with
//                      beta = 2 mean|x|, FP4 E1M2 (Fig. 5 and 6)
// An HBM-bound row kernel: one pass over coalesced 16-byte loads, the row held
// in registers, reductions by warp shuffles and a few shared words.  (Top-K +
// INT8 rows are in topk.cuh.)
#pragma once

#include "common.cuh"

namespace bl {

// fp32 nearest to sqrt(7) (0x402953FD).
__device__ __forceinline__ float sqrt7_f32() { return __uint_as_float(0x402953FDu); }

// 2^n as an fp32 (n >= -149), built from its bit pattern.
__device__ __forceinline__ float exact_pow2(int n) {
  return n >= -126 ? __uint_as_float(static_cast<uint32_t>(n + 127) << 23)
                   : __uint_as_float(1u << (n + 149));
}

// x * 2^n, exact for the ranges used here (x bf16-valued, result magnitude <= 6).
__device__ __forceinline__ float mul_pow2(float x, int n) {
  if (n <= 127) return __fmul_rn(x, exact_pow2(n));
  return __fmul_rn(__fmul_rn(x, exact_pow2(64)), exact_pow2(n - 64));
}

// Smallest p with g <= 6 * 2^p for g = the fp32 with bits `gbits` (sign clear);
// p = 0 for g = 0.  6 * 2^p = 1.5 * 2^(p+2), so with g = m * 2^e, m in [1, 2):
// p = e - 2 when m <= 1.5, else e - 1.
__device__ __forceinline__ int fp4_scale_exponent(uint32_t gbits) {
  if (gbits == 0) return 0;
  const uint32_t E = gbits >> 23;
  const uint32_t mant = gbits & 0x7FFFFFu;
  int e;
  uint32_t m24;
  if (E != 0) {
    e = static_cast<int>(E) - 127;
    m24 = mant | 0x800000u;
  } else {  // subnormal: normalise the leading one to bit 23
    const int lead = 31 - __clz(mant);
    const int sh = 23 - lead;
    m24 = mant << sh;
    e = -126 - sh;
  }
  return (m24 <= 0xC00000u) ? e - 2 : e - 1;
}

// Smallest p with g <= 1.75 * 2^p (FP4 E1M2's largest magnitude is 1.75):
// with g = m * 2^e, m in [1, 2), p = e when m <= 1.75, else e + 1.
__device__ __forceinline__ int e1m2_scale_exponent(uint32_t gbits) {
  if (gbits == 0) return 0;
  const uint32_t E = gbits >> 23;
  const uint32_t mant = gbits & 0x7FFFFFu;
  int e;
  uint32_t m24;
  if (E != 0) {
    e = static_cast<int>(E) - 127;
    m24 = mant | 0x800000u;
  } else {
    const int lead = 31 - __clz(mant);
    const int sh = 23 - lead;
    m24 = mant << sh;
    e = -126 - sh;
  }
  return (m24 <= 0xE00000u) ? e : e + 1;
}

// Eight fp32 -> eight E2M1 codes (element e in bits 4e..4e+3) by the hardware
// conversion: round to nearest, ties to the even encoding, saturating at 6.  A
// magnitude that rounds to zero is re-encoded as +0 (sign bit cleared).
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
  uint32_t w;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(w)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  const uint32_t nz = (w | (w >> 1) | (w >> 2)) & 0x11111111u;   // per nibble: magnitude bits nonzero
  return w & (0x77777777u | (nz << 3));
}

// Index of the nearest E2M1 magnitude {0,.5,1,1.5,2,3,4,6} to a (a >= 0),
// ties to the even index (the encoding with mantissa bit 0).  Each midpoint
// between an even and an odd index uses '>' (the tie stays on the even side
// below), each midpoint between an odd and an even index uses '>='.
__device__ __forceinline__ int e2m1_index(float a) {
  return (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
}

// ---------------------------------------------------------------------------
// quant_a4: 128 threads per row, two row slots per 256-thread CTA, persistent
// over rows.  Thread t of a row holds chunks c*128 + t (8 bf16 each) for
// c < CHUNKS; the next row's chunks are loaded before the current row is
// reduced and written, so every thread keeps a row's loads in flight.
// ---------------------------------------------------------------------------
constexpr int kQ4ThreadsPerRow = 128;

// Low bits of RN(RN(p) + 1.5*2^23) hold rint_even(p) for |p| < 2^22 (the sum's
// ulp is 1); p is clamped to the code range first.
__device__ __forceinline__ uint32_t q4_code_bits(float x, float mult) {
  const float p = fminf(fmaxf(__fmul_rn(x, mult), -8.f), 7.f);
  return __float_as_uint(__fadd_rn(p, 12582912.0f));
}

// Barrier of one row slot (128 threads); literal ids keep the CTA at two barriers.
__device__ __forceinline__ void q4_row_sync(int sub) {
  if (sub == 0) {
    asm volatile("bar.sync 1, 128;" ::: "memory");
  } else {
    asm volatile("bar.sync 2, 128;" ::: "memory");
  }
}

template <int CHUNKS>
__device__ __forceinline__ void q4_load(const uint16_t* x, int64_t row, int64_t M, int64_t ldx, int nchunk, int t,
                                        uint4 (&v)[CHUNKS]) {
  const bool ok = row < M;
  const uint16_t* xr = x + (ok ? row : 0) * ldx;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int idx = c * kQ4ThreadsPerRow + t;
    v[c] = (ok && idx < nchunk) ? ld_global_nc_v4(xr + static_cast<int64_t>(idx) * 8) : make_uint4(0, 0, 0, 0);
  }
}

// Quantizer variants (the values of bl_quant): absmean INT4 (Eq. 6-7), MinMax
// FP4 E2M1 (Eq. 8-9), and the ablation variants INT4 absmax, INT4 absmean with
// beta = 2 mean|x|, FP4 E1M2; kQInt4Tensor is absmean INT4 with a beta given in
// device memory (one for the whole tensor).
enum : int { kQInt4 = 0, kQFp4 = 1, kQInt4Absmax = 2, kQInt4Absmean2 = 3, kQFp4E1M2 = 4, kQInt4Tensor = 5 };

// ---------------------------------------------------------------------------
// RMSNorm prologue: ms = the exact mean of x^2 over the row, rounded once to
// fp32.  Each thread accumulates its squares (exact in fp64) as a double-double
// hi + lo with TwoSum; the partial pairs are combined the same way.  For rows
// whose squares, as multiples of the smallest one's last bit, sum below 2^90,
// every one of these additions is exact, so the pair holds the exact sum
// whatever the order (the error of a TwoSum is exact; lo stays below n * 2^-53
// of the sum, n <= 16384, so its additions fit 53 bits).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void two_sum_f64(double a, double b, double& s, double& e) {
  s = __dadd_rn(a, b);
  const double bp = __dsub_rn(s, a);
  e = __dadd_rn(__dsub_rn(a, __dsub_rn(s, bp)), __dsub_rn(b, bp));
}
__device__ __forceinline__ void dd_add(double& hi, double& lo, double a) {
  double s, e;
  two_sum_f64(hi, a, s, e);
  hi = s;
  lo = __dadd_rn(lo, e);
}
__device__ __forceinline__ void dd_add_dd(double& hi, double& lo, double h2, double l2) {
  double s, e;
  two_sum_f64(hi, h2, s, e);
  hi = s;
  lo = __dadd_rn(__dadd_rn(lo, l2), e);
}

// fp64 value of a bf16 magnitude key k (15 bits: exponent << 7 | mantissa),
// built from its bits with one multiply-add (no conversion unit): exact for a
// normal value (k >= 0x80); for a zero or subnormal key the result and the true
// value are both below 2^-126, an absolute error the certificates below count.
__device__ __forceinline__ double key_to_f64(uint32_t k) {
  return __hiloint2double(static_cast<int>(k * 8192u + 0x38000000u), 0);
}

// Certified rounding: c = RN_fp32(q), and true when every value within err of
// q rounds to the same fp32 (so c is the rounding of any quotient known to lie
// within err of q; the quotients here are non-negative).
__device__ __forceinline__ bool certify_f32(double q, double err, float& c) {
  c = __double2float_rn(q);
  const double up = 0.5 * (static_cast<double>(c) + static_cast<double>(nextafterf(c, __int_as_float(0x7F800000))));
  if (!(__dadd_rn(q, err) < up)) return false;
  if (c > 0.f) {
    const double dn = 0.5 * (static_cast<double>(c) + static_cast<double>(nextafterf(c, 0.f)));
    if (!(__dsub_rn(q, err) > dn)) return false;
  }
  return true;
}

// Relative error bound of an fp64 sum of n positive terms (at most n + 10
// roundings along any path of the partial-sums-then-warp-then-CTA reduction),
// with a factor of two to spare: 2 (n + 32) 2^-53.
__device__ __forceinline__ double sum_rel_bound(int n) { return static_cast<double>(2 * n + 64) * 0x1p-53; }

// RN_fp32((hi + lo) / K) for an exact sum hi + lo >= 0: the fp32 nearest to
// hi / K, then moved while the exact quotient lies beyond a midpoint to a
// neighbour (at a midpoint: the even one).  A midpoint m has at most 25
// significant bits and K at most 15, so K * m is exact in fp64, and the sign of
// (hi - K m) + lo is the sign of the exact S - K m (exact subtraction when hi
// and K m are within a factor of two, a difference much larger than lo
// otherwise).
__device__ __forceinline__ float dd_mean_f32(double hi, double lo, int K) {
  if (hi == 0.0 && lo == 0.0) return 0.f;
  const double dk = static_cast<double>(K);
  float c = __double2float_rn(__ddiv_rn(hi, dk));
  auto side = [&](float nb) -> int {   // sign of S/K - (c + nb)/2
    const double mid = 0.5 * (static_cast<double>(c) + static_cast<double>(nb));
    const double d = __dadd_rn(__dsub_rn(hi, __dmul_rn(mid, dk)), lo);
    return d > 0.0 ? 1 : (d < 0.0 ? -1 : 0);
  };
#pragma unroll 1
  for (int it = 0; it < 4; ++it) {
    const bool odd = (__float_as_uint(c) & 1u) != 0u;
    const float up = nextafterf(c, __int_as_float(0x7F800000));
    const int su = side(up);
    if (su > 0 || (su == 0 && odd)) {
      c = up;
      continue;
    }
    if (c > 0.f) {
      const float dn = nextafterf(c, 0.f);
      const int sd = side(dn);
      if (sd < 0 || (sd == 0 && odd)) {
        c = dn;
        continue;
      }
    }
    break;
  }
  return c;
}

// NORM: the row is first replaced by its RMSNorm, y = bf16((x * r) * g),
// r = 1 / sqrt(ms + eps_n) (fp32 IEEE operations; g = gnorm, or 1 when NULL),
// and the quantizer runs on y.  VAR == kQInt4Tensor reads beta from *beta_dev.
template <int CHUNKS, int VAR, bool PACKED, bool NORM>
__global__ void __launch_bounds__(256) quant_a4_kernel(const uint16_t* __restrict__ x, int64_t M, int K,
                                                       int64_t ldx, float eps, uint8_t* __restrict__ codes,
                                                       float* __restrict__ scale, const float* __restrict__ gnorm,
                                                       float eps_n, const float* __restrict__ beta_dev) {
  __shared__ double s_sum[2][2][4];
  __shared__ uint32_t s_max[2][2][4];
  __shared__ double s_dd[NORM ? 2 : 1][2][4][2];
  const int sub = threadIdx.x >> 7;
  const int t = threadIdx.x & 127;
  const int warp = t >> 5;
  const int lane = threadIdx.x & 31;
  const int nchunk = K >> 3;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * 2;
  int64_t row = static_cast<int64_t>(blockIdx.x) * 2 + sub;
  pdl_wait();
  pdl_trigger();

  // rows of up to 4096 values prefetch the next row; longer rows would need too
  // many registers for two rows, so they load at the top of each iteration
  constexpr bool kPrefetch = CHUNKS <= 4;
  uint4 v[CHUNKS];
  if (kPrefetch) q4_load<CHUNKS>(x, row, M, ldx, nchunk, t, v);
  for (int it = 0; row < M; row += stride, ++it) {
    uint4 nx[kPrefetch ? CHUNKS : 1];
    if constexpr (kPrefetch) {
      q4_load<CHUNKS>(x, row + stride, M, ldx, nchunk, t, nx);
    } else {
      q4_load<CHUNKS>(x, row, M, ldx, nchunk, t, v);
    }
    const int par = it & 1;
    constexpr bool kSum = VAR == kQInt4 || VAR == kQInt4Absmean2;   // mean|x| statistic, else max|x|
    constexpr bool kInt = VAR == kQInt4 || VAR == kQInt4Absmean2 || VAR == kQInt4Absmax || VAR == kQInt4Tensor;

    if constexpr (NORM) {
      // ---- RMSNorm: ms = RN_fp32(exact mean of x^2), r, and y in place of x ----
      // Fast path: a plain fp64 sum of the squares (each exact; one rounding per
      // addition, at most K + 8 of them in any order), so the sum is within
      // (K + 8) * 2^-53 of the exact one, relatively.  If every quotient in that
      // interval (and the division's own rounding) rounds to the same fp32, that
      // fp32 is ms; otherwise -- a quotient within about K * 2^-53 of an fp32
      // midpoint, one row in ~2^15 -- the row's sum is recomputed exactly as a
      // double-double.  The decision is the same for every thread of the row.
      double sp[4] = {0.0, 0.0, 0.0, 0.0};   // independent partial sums: short dependency chains
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) {
        uint32_t k[8];
        bf16x8_mag_keys(v[c], k);   // chunks past K hold zeros
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const double d = key_to_f64(k[e]);
          sp[e & 3] = __fma_rn(d, d, sp[e & 3]);
        }
      }
      double sa = warp_sum_f64((sp[0] + sp[1]) + (sp[2] + sp[3]));
      if (lane == 0) s_dd[par][sub][warp][0] = sa;
      q4_row_sync(sub);
      sa = (s_dd[par][sub][0][0] + s_dd[par][sub][1][0]) + (s_dd[par][sub][2][0] + s_dd[par][sub][3][0]);
      const double q = __ddiv_rn(sa, static_cast<double>(K));
      // zero and subnormal keys: each square off by less than 2^-252
      float ms;
      const bool certain = certify_f32(q, __dadd_rn(__dmul_rn(q, sum_rel_bound(K)), 0x1p-252), ms);
      if (!certain) {
        double hi = 0.0, lo = 0.0;
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
          float f[8];
          unpack_bf16x8(v[c], f);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const double d = static_cast<double>(f[e]);
            dd_add(hi, lo, __dmul_rn(d, d));
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
          dd_add_dd(hi, lo, __shfl_xor_sync(0xFFFFFFFFu, hi, o), __shfl_xor_sync(0xFFFFFFFFu, lo, o));
        // the fast-path words of this row slot were read by every thread before the barrier below
        q4_row_sync(sub);
        if (lane == 0) {
          s_dd[par][sub][warp][0] = hi;
          s_dd[par][sub][warp][1] = lo;
        }
        q4_row_sync(sub);
        hi = s_dd[par][sub][0][0];
        lo = s_dd[par][sub][0][1];
#pragma unroll
        for (int w = 1; w < 4; ++w) dd_add_dd(hi, lo, s_dd[par][sub][w][0], s_dd[par][sub][w][1]);
        ms = dd_mean_f32(hi, lo, K);
      }
      const float r = __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(ms, eps_n)));
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) {
        const int idx = c * kQ4ThreadsPerRow + t;
        if (idx >= nchunk) continue;
        float f[8];
        unpack_bf16x8(v[c], f);
        float g[8];
        if (gnorm != nullptr) {
          const uint4 g0 = ld_global_nc_v4(gnorm + 8 * static_cast<int64_t>(idx));
          const uint4 g1 = ld_global_nc_v4(gnorm + 8 * static_cast<int64_t>(idx) + 4);
          g[0] = __uint_as_float(g0.x); g[1] = __uint_as_float(g0.y); g[2] = __uint_as_float(g0.z);
          g[3] = __uint_as_float(g0.w); g[4] = __uint_as_float(g1.x); g[5] = __uint_as_float(g1.y);
          g[6] = __uint_as_float(g1.z); g[7] = __uint_as_float(g1.w);
        }
        float tv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          tv[e] = __fmul_rn(f[e], r);
          if (gnorm != nullptr) tv[e] = __fmul_rn(tv[e], g[e]);
        }
        // paired conversions (round to nearest even; no conversion-unit instruction)
        uint32_t hb[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 b = __floats2bfloat162_rn(tv[2 * e], tv[2 * e + 1]);
          hb[e] = *reinterpret_cast<const uint32_t*>(&b);
        }
        v[c] = make_uint4(hb[0], hb[1], hb[2], hb[3]);
      }
    }

    // ---- the row statistic ----
    double S = 0.0;       // sum |x| (exact in fp64 for in-contract rows: order-free)
    uint32_t mk = 0;      // max |x| as the largest 15-bit bf16 magnitude
    float beta_c = 0.f;   // beta, when the certified fast path settles it (RMSNorm rows)
    bool beta_ok = false;
    if constexpr (kSum && NORM) {
      // beta = RN_fp32(RN_fp64(S / K)) with S the exact sum of |y| (exact in fp64
      // for in-contract rows).  Fast path: doubles built from the bits, four
      // partial sums, and a certificate; the exact sum only for rows the
      // certificate cannot settle.  (Measured: faster here, where the norm
      // already keeps the conversion unit busy; slower than the exact sum alone
      // in the plain quantizer, which keeps that.)
      double ap[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) {
        uint32_t k[8];
        bf16x8_mag_keys(v[c], k);
#pragma unroll
        for (int e = 0; e < 8; ++e) ap[e & 3] = __dadd_rn(ap[e & 3], key_to_f64(k[e]));
      }
      double acc = warp_sum_f64((ap[0] + ap[1]) + (ap[2] + ap[3]));
      if (lane == 0) s_sum[par][sub][warp] = acc;
      q4_row_sync(sub);
      const double sa = (s_sum[par][sub][0] + s_sum[par][sub][1]) + (s_sum[par][sub][2] + s_sum[par][sub][3]);
      const double two = VAR == kQInt4Absmean2 ? 2.0 : 1.0;   // exact doubling
      const double q = __ddiv_rn(two * sa, static_cast<double>(K));
      // + the fp64 division's own rounding (2^-53 relative, inside the bound) and
      // zero / subnormal keys (each off by less than 2^-126)
      beta_ok = certify_f32(q, __dadd_rn(__dmul_rn(q, sum_rel_bound(K)), two * 0x1p-126), beta_c);
      if (!beta_ok) {
        double ex = 0.0;
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
          float f[8];
          unpack_bf16x8(v[c], f);
#pragma unroll
          for (int e = 0; e < 8; ++e) ex += static_cast<double>(fabsf(f[e]));
        }
        ex = warp_sum_f64(ex);
        q4_row_sync(sub);   // every thread has read the fast-path words
        if (lane == 0) s_sum[par][sub][warp] = ex;
        q4_row_sync(sub);
        S = (s_sum[par][sub][0] + s_sum[par][sub][1]) + (s_sum[par][sub][2] + s_sum[par][sub][3]);
      }
    } else if constexpr (kSum) {
      double acc = 0.0;
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) {
        float f[8];
        unpack_bf16x8(v[c], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc += static_cast<double>(fabsf(f[e]));
      }
      acc = warp_sum_f64(acc);
      if (lane == 0) s_sum[par][sub][warp] = acc;
      q4_row_sync(sub);
      S = (s_sum[par][sub][0] + s_sum[par][sub][1]) + (s_sum[par][sub][2] + s_sum[par][sub][3]);
    } else if constexpr (VAR != kQInt4Tensor) {
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) {
        uint32_t k[8];
        bf16x8_mag_keys(v[c], k);
#pragma unroll
        for (int e = 0; e < 8; ++e) mk = max(mk, k[e]);
      }
      mk = __reduce_max_sync(0xFFFFFFFFu, mk);
      if (lane == 0) s_max[par][sub][warp] = mk;
      q4_row_sync(sub);
      mk = max(max(s_max[par][sub][0], s_max[par][sub][1]), max(s_max[par][sub][2], s_max[par][sub][3]));
    }

    if constexpr (kInt) {
      // ---- INT4 codes RoundClip(x * mult, -8, 7) ----
      float mult;
      if constexpr (VAR == kQInt4Tensor) {
        const float beta = ld_dep_f32(beta_dev);   // the tensor's exact mean |x|
        mult = __fdiv_rn(sqrt7_f32(), __fadd_rn(beta, eps));
        if (t == 0) scale[row] = __fdiv_rn(beta, sqrt7_f32());
      } else if constexpr (VAR == kQInt4Absmax) {
        const float gamma = __uint_as_float(mk << 16);   // max |x| (a bf16 value)
        mult = __fdiv_rn(7.f, __fadd_rn(gamma, eps));
        if (t == 0) scale[row] = __fdiv_rn(gamma, 7.f);
      } else {
        // beta = mean|x| (INT4) or 2 mean|x| (the doubling is exact)
        const float beta =
            beta_ok ? beta_c : __double2float_rn((VAR == kQInt4Absmean2 ? 2.0 * S : S) / static_cast<double>(K));
        mult = __fdiv_rn(sqrt7_f32(), __fadd_rn(beta, eps));
        if (t == 0) scale[row] = __fdiv_rn(beta, sqrt7_f32());
      }
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) {
        const int idx = c * kQ4ThreadsPerRow + t;
        if (idx >= nchunk) continue;
        float f[8];
        unpack_bf16x8(v[c], f);
        uint32_t q[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) q[e] = q4_code_bits(f[e], mult);
        if constexpr (PACKED) {
          uint32_t word = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) word |= (q[e] & 0xFu) << (4 * e);
          reinterpret_cast<uint32_t*>(codes + row * (K >> 1))[idx] = word;
        } else {
          uint2 w2;
          // the low byte of each sum's bits is the code as a two's-complement int8
          w2.x = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
          w2.y = __byte_perm(__byte_perm(q[4], q[5], 0x0040), __byte_perm(q[6], q[7], 0x0040), 0x5410);
          reinterpret_cast<uint2*>(codes + row * static_cast<int64_t>(K))[idx] = w2;
        }
      }
    } else {
      // ---- MinMax FP4: a power-of-two scale 2^p, the nearest grid magnitude ----
      constexpr bool kE1M2 = VAR == kQFp4E1M2;
      const int p = kE1M2 ? e1m2_scale_exponent(mk << 16) : fp4_scale_exponent(mk << 16);
      // bytes hold 2 x the E2M1 value or 4 x the E1M2 value
      if (t == 0) scale[row] = exact_pow2(PACKED ? p : (kE1M2 ? p - 2 : p - 1));
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) {
        const int idx = c * kQ4ThreadsPerRow + t;
        if (idx >= nchunk) continue;
        float f[8];
        unpack_bf16x8(v[c], f);
        float sv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) sv[e] = mul_pow2(f[e], -p);   // exact
        uint32_t word = 0;
        uint2 w2 = make_uint2(0, 0);
        if constexpr (!kE1M2) {
          word = cvt_e2m1x8(sv);
          if constexpr (!PACKED) {
            // bytes: twice the E2M1 value {0,1,2,3,4,6,8,12} with its sign
            uint32_t b0, b1;
            split_nibbles(word, b0, b1);
            w2 = make_uint2(e2m1_bytes_to_twice(b0), e2m1_bytes_to_twice(b1));
          }
        } else {
          // the E1M2 magnitudes are the quarters 0..7/4: index = rint(4 |v|)
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int i = min(__float2int_rn(__fmul_rn(fabsf(sv[e]), 4.f)), 7);
            const bool neg = (sv[e] < 0.f) && (i != 0);
            if constexpr (PACKED) {
              word |= (static_cast<uint32_t>(i) | (neg ? 8u : 0u)) << (4 * e);
            } else {
              const uint32_t b = static_cast<uint32_t>(neg ? -i : i) & 0xFFu;
              if (e < 4) w2.x |= b << (8 * e); else w2.y |= b << (8 * (e - 4));
            }
          }
        }
        if constexpr (PACKED) {
          reinterpret_cast<uint32_t*>(codes + row * (K >> 1))[idx] = word;
        } else {
          reinterpret_cast<uint2*>(codes + row * static_cast<int64_t>(K))[idx] = w2;
        }
      }
    }
    if constexpr (kPrefetch) {
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) v[c] = nx[c];
    }
  }
}

}  // namespace bl
