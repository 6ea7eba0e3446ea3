// Absmean ternary weight quantizer and packer (BitNet a4.8, §3.4 "Ternary
// Weight Quantization (BitLinear)", Eq. 2):
//   alpha = mean|W| (per tensor),  t = RoundClip(W / (alpha + eps), -1, 1).
//
// alpha is the exact mean rounded once to fp32.  |w| = m * 2^(max(E,1) - 150)
// with m the 24-bit significand and E the biased exponent, so the exact sum is
// held as unsigned 64-bit integer coefficients of powers of two (bins); integer
// adds are exact and order-free.  Twelve threads then form the 32-bit limbs of
//   Z = sum_e bins[e] << (e - 1)                 (the sum in units of 2^-149)
// and one thread divides it by N*K and rounds to nearest-even fp32.
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kBinThreads = 256;
// bins[e] is the integer coefficient of 2^(e - 150), e >= 1 (fp32 subnormals use
// e = 1, the same scale).  A window base is clamped to at most 223, so the high
// half of a flushed window sum (index base + 32) stays below 256.
constexpr int kBins = 256;
// Each bin receives at most one 32-bit half per flushed window (>= 1 weight)
// or one 24-bit significand per weight, so N*K < 2^31 keeps every 64-bit bin
// below overflow (2^31 * 2^32).
constexpr int64_t kMaxPackElems = int64_t(1) << 31;

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Exact sum of |w| into exponent bins.  Each lane keeps an fp64 accumulator
// holding an integer multiple of 2^(ub-150) below 2^(ub-150+53): weights with
// biased exponent E in the window [ub, ub + kWin - 1] are multiples of that unit
// and below 2^(ub-150+45), so up to 256 of them add exactly (every partial sum
// is representable).  The window is anchored 12 exponents below the largest
// weight of the lane's first nonzero load batch (ub clamped to [1, 223]);
// weights outside it, and fp32 subnormals, add their integer significand to
// their own bin.  Every 16 load batches (256 weights per lane) and at the end,
// the accumulator is flushed as an integer n < 2^53 into bins[ub] (low 32 bits)
// and bins[ub + 32] (high bits).
constexpr uint32_t kWin = 22;

__device__ __forceinline__ void bins_flush(unsigned long long* sb, uint32_t ub, double& acc) {
  if (acc != 0.0) {
    // n = acc * 2^(150 - ub), exact: 150 - ub is in [-73, 149]
    const double unit_inv = __hiloint2double(static_cast<int>((1023 + 150 - ub) << 20), 0);
    const unsigned long long n = __double2ull_rn(acc * unit_inv);
    atomicAdd(&sb[ub], n & 0xFFFFFFFFull);
    atomicAdd(&sb[ub + 32], n >> 32);
    acc = 0.0;
  }
}

__device__ void alpha_from_bins(const unsigned long long* gbins, unsigned long long D, float* alpha,
                                unsigned long long* sb);

// gbins (zeroed by the caller): bins 1..255 and, in bin 0, a count of finished
// CTAs; the last CTA to finish computes alpha.  BF16: w holds bf16 values (row
// stride ldw in bf16 elements), each exact as an fp32 -- the same exact mean
// of |x| for an activation tensor (the per-tensor INT4 scale).
template <bool BF16>
__global__ void __launch_bounds__(kBinThreads, 6) ternary_bins_kernel(const void* __restrict__ wv, int64_t N, int K,
                                                                   int64_t ldw,
                                                                   unsigned long long* __restrict__ gbins,
                                                                   float* __restrict__ alpha) {
  __shared__ unsigned long long sb[kBins];
  const int lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kBins; i += kBinThreads) sb[i] = 0ull;
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  constexpr int kPer = BF16 ? 8 : 4;   // values per 16-byte load
  const int per_row = K / kPer;        // 16-byte loads per row
  const int64_t gwarp = (static_cast<int64_t>(blockIdx.x) * kBinThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kBinThreads) >> 5;
  constexpr int kLoads = 4;   // float4 loads per lane issued together (16 weights)
  uint32_t ub = 0;            // 0: not anchored yet
  uint32_t lo_bits = 0x7F800000u;   // ub << 23 once anchored; before that no finite value is in the window
  double acc = 0.0;
  int batches = 0;
  for (int64_t n = gwarp; n < N; n += nwarps) {
    const uint8_t* wrow = static_cast<const uint8_t*>(wv) + n * ldw * (BF16 ? 2 : 4);
    for (int q0 = 0; q0 < per_row; q0 += 32 * kLoads) {
      // lane 0 asks L2 for the row's batch two ahead (and, at the row's start,
      // the next one too), so each warp keeps three batches in flight
      if (lane == 0) {
        for (int qa = q0 == 0 ? 32 * kLoads : 64 * kLoads; qa <= 64 * kLoads; qa += 32 * kLoads)
          if (q0 + qa < per_row)
            bulk_prefetch_l2(wrow + static_cast<int64_t>(q0 + qa) * 16,
                             static_cast<uint32_t>(min(32 * kLoads, per_row - q0 - qa)) * 16u);
      }
      uint32_t u[kPer * kLoads];   // |w| as fp32 bit patterns
#pragma unroll
      for (int j = 0; j < kLoads; ++j) {
        const int q = q0 + j * 32 + lane;
        const uint4 v = q < per_row ? ld_global_nc_v4(wrow + static_cast<int64_t>(q) * 16) : make_uint4(0, 0, 0, 0);
        if constexpr (BF16) {
          const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            u[8 * j + 2 * h] = (hw[h] << 16) & 0x7FFFFFFFu;
            u[8 * j + 2 * h + 1] = hw[h] & 0x7FFF0000u;
          }
        } else {
          u[4 * j] = v.x & 0x7FFFFFFFu;
          u[4 * j + 1] = v.y & 0x7FFFFFFFu;
          u[4 * j + 2] = v.z & 0x7FFFFFFFu;
          u[4 * j + 3] = v.w & 0x7FFFFFFFu;
        }
      }
      if (ub == 0) {
        uint32_t amax = 0;
#pragma unroll
        for (int i = 0; i < kPer * kLoads; ++i) amax = max(amax, u[i]);
        if (amax != 0) {
          const int E = static_cast<int>(amax >> 23);
          ub = static_cast<uint32_t>(min(max(E - 12, 1), 223));
          lo_bits = ub << 23;
        }
      }
#pragma unroll
      for (int i = 0; i < kPer * kLoads; ++i) {
        const uint32_t a = u[i];
        if (a - lo_bits < (kWin << 23)) {
          // exact: inside the window a is a normal fp32 (biased exponent >= ub >= 1),
          // so its fp64 is built from the bits -- exponent rebiased by 1023 - 127,
          // significand shifted up by 29 -- with integer operations instead of
          // the conversion unit
          acc += __hiloint2double(static_cast<int>((a >> 3) + ((1023u - 127u) << 20)), static_cast<int>(a << 29));
        } else if (a != 0) {
          const uint32_t E = a >> 23;
          const uint32_t m = (a & 0x7FFFFFu) | (E ? 0x800000u : 0u);
          atomicAdd(&sb[E ? E : 1u], static_cast<unsigned long long>(m));
        }
      }
      if (++batches == 128 / kPer) {   // every 256 values per lane (the exact-sum bound above)
        bins_flush(sb, ub, acc);
        batches = 0;
      }
    }
  }
  bins_flush(sb, ub, acc);
  __syncthreads();
  for (int b = threadIdx.x; b < kBins; b += kBinThreads)
    if (sb[b]) atomicAdd(&gbins[b], sb[b]);
  // the last CTA to finish sees every CTA's bins and forms alpha
  __threadfence();
  __syncthreads();
  __shared__ bool last;
  if (threadIdx.x == 0) last = atomicAdd(&gbins[0], 1ull) == gridDim.x - 1u;
  __syncthreads();
  if (!last) return;
  __threadfence();
  alpha_from_bins(gbins, static_cast<unsigned long long>(N) * static_cast<unsigned long long>(K), alpha, sb);
}

// Multi-word unsigned integer, little-endian 32-bit limbs.
constexpr int kLimbs = 12;  // 384 bits: bins < 2^64 shifted by <= 262 bits

__device__ __forceinline__ int big_bitlen(const uint32_t (&z)[kLimbs]) {
  for (int i = kLimbs - 1; i >= 0; --i)
    if (z[i]) return 32 * i + (32 - __clz(z[i]));
  return 0;
}

__device__ __forceinline__ uint32_t big_limb(const uint32_t (&z)[kLimbs], int i) {
  return (i >= 0 && i < kLimbs) ? z[i] : 0u;
}

__device__ __forceinline__ uint32_t big_bit(const uint32_t (&z)[kLimbs], int b) {
  return (b < 0) ? 0u : (big_limb(z, b >> 5) >> (b & 31)) & 1u;
}

// Any bit set strictly below position b?
__device__ __forceinline__ bool big_any_below(const uint32_t (&z)[kLimbs], int b) {
  if (b <= 0) return false;
  const int full = b >> 5;
  for (int i = 0; i < full && i < kLimbs; ++i)
    if (z[i]) return true;
  const int rem = b & 31;
  return rem && (big_limb(z, full) & ((1u << rem) - 1u));
}

// 64-bit window of z starting at bit sh >= 0.
__device__ __forceinline__ unsigned long long big_window64(const uint32_t (&z)[kLimbs], int sh) {
  const int li = sh >> 5, bo = sh & 31;
  const unsigned long long lo =
      static_cast<unsigned long long>(big_limb(z, li)) | (static_cast<unsigned long long>(big_limb(z, li + 1)) << 32);
  const unsigned long long hi = big_limb(z, li + 2);
  return bo ? ((lo >> bo) | (hi << (64 - bo))) : lo;
}

// alpha = RN_fp32( (Z * 2^-149) / D ),  Z = sum_e bins[e] << (e - 1), by the last
// CTA of the binning kernel (bin 0 holds the CTA counter and is not a bin):
// twelve threads form the limbs, thread 0 divides.
__device__ void alpha_from_bins(const unsigned long long* gbins, unsigned long long D, float* alpha,
                                unsigned long long* sb) {
  __shared__ unsigned long long limb_sum[kLimbs];
  for (int e = threadIdx.x; e < kBins; e += blockDim.x) sb[e] = e == 0 ? 0ull : __ldcg(gbins + e);
  __syncthreads();
  // thread l < kLimbs sums the 32-bit pieces of every shifted bin that fall in
  // limb l (at most 256 pieces < 2^32, so the sum stays below 2^40)
  if (threadIdx.x < kLimbs) {
    const int l = threadIdx.x;
    unsigned long long acc = 0;
    for (int e = 0; e < kBins; ++e) {
      const unsigned long long v = sb[e];
      const int r = (e > 0 ? e : 1) - 1 - 32 * l;   // bit of v that lands on the limb's bit 0 is -r
      if (v == 0 || r >= 32 || r <= -64) continue;
      acc += (r >= 0 ? (v << r) : (v >> -r)) & 0xFFFFFFFFull;
    }
    limb_sum[l] = acc;
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  uint32_t z[kLimbs];
  unsigned long long carry = 0;
  for (int i = 0; i < kLimbs; ++i) {
    const unsigned long long t = limb_sum[i] + carry;
    z[i] = static_cast<uint32_t>(t);
    carry = t >> 32;
  }
  // Long division Q = floor(Z / D), R = Z mod D.
  uint32_t q[kLimbs];
  unsigned long long R;
  if (D <= 0xFFFFFFFFull) {
    unsigned long long rem = 0;
    for (int i = kLimbs - 1; i >= 0; --i) {
      const unsigned long long cur = (rem << 32) | z[i];
      q[i] = static_cast<uint32_t>(cur / D);
      rem = cur % D;
    }
    R = rem;
  } else {
    unsigned __int128 rem = 0;
    for (int i = kLimbs - 1; i >= 0; --i) {
      const unsigned __int128 cur = (rem << 32) | z[i];
      q[i] = static_cast<uint32_t>(cur / D);
      rem = cur % D;
    }
    R = static_cast<unsigned long long>(rem);
  }
  const int L = big_bitlen(q);
  float result;
  if (L == 0) {
    // value * 2^149 = R/D < 1: rounds to 0 or to the smallest subnormal
    result = (2 * static_cast<unsigned __int128>(R) > D) ? __uint_as_float(1u) : 0.f;
  } else {
    // value = (Q + R/D) * 2^-149, top bit of Q at L-1 -> exponent L-1-149.
    // Keep 24 significant bits, or all bits down to 2^-149 when subnormal.
    const int shift = (L - 1 - 23 > 0) ? (L - 1 - 23) : 0;
    unsigned long long mant = big_window64(q, shift) & ((1ull << 25) - 1ull);
    bool up;
    if (shift == 0) {
      const unsigned __int128 twoR = 2 * static_cast<unsigned __int128>(R);
      up = twoR > D || (twoR == D && (mant & 1ull));
    } else {
      const uint32_t half = big_bit(q, shift - 1);
      const bool below = big_any_below(q, shift - 1) || R != 0;
      up = half && (below || (mant & 1ull));
    }
    mant += up ? 1ull : 0ull;
    int lsb_exp = shift - 149;  // value = mant * 2^lsb_exp
    if (mant >> 24) {           // carried into a new binade
      mant >>= 1;
      lsb_exp += 1;
    }
    if (mant >> 23) {
      const int biased = lsb_exp + 23 + 127;
      result = biased >= 255 ? __uint_as_float(0x7F800000u)
                             : __uint_as_float((static_cast<uint32_t>(biased) << 23) |
                                               static_cast<uint32_t>(mant & 0x7FFFFFu));
    } else {
      result = __uint_as_float(static_cast<uint32_t>(mant));  // subnormal: lsb_exp == -149
    }
  }
  *alpha = result;
}

// t = RoundClip(w / (alpha + eps), -1, 1) without the division.  With d = alpha + eps
// and h = d / 2 (exact while d >= 2^-125): rint(RN(|w|/d)) clipped to 1 is nonzero
// iff RN(|w|/d) > 1/2, iff |w|/d > 1/2 + 2^-25 (the tie at that midpoint rounds to
// the even 1/2), iff |w| > h * (1 + 2^-24).  Since h * 2^-24 < ulp(h), for an
// fp32 |w| that is the same as |w| > h.  So t = sign(w) * [|w| > h].  Smaller d
// (or an infinite one) keeps the IEEE division.
__device__ __forceinline__ int ternary_code(float w, float d, float h, bool fast) {
  if (fast) return fabsf(w) > h ? (w > 0.f ? 1 : -1) : 0;
  return round_clip(__fdiv_rn(w, d), -1.f, 1.f);
}

// t = RoundClip(w / (alpha + eps), -1, 1); 16 weights per thread-step.
//   WF = BL_W_T2:   4 bytes out (2-bit codes, element 4i in bits 0-1; 0->00, +1->01, -1->11)
//   WF = BL_W_I8:   16 bytes out
//   WF = BL_W_E2M1: 8 bytes out (E2M1 nibbles, element 2i in bits 0-3; 0->0x0, +1->0x2, -1->0xA)
template <int WF>
__global__ void __launch_bounds__(256) ternary_pack_kernel(const float* __restrict__ w, int64_t N, int K,
                                                           int64_t ldw, const float* __restrict__ alpha,
                                                           float eps, uint8_t* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const float d = __fadd_rn(ld_dep_f32(alpha), eps);
  const bool fast = d >= 0x1p-125f && d <= 0x1p+127f;   // d/2 exact and normal
  const float h = __fmul_rn(d, 0.5f);
  const int per_row = K >> 4;   // 16 weights per thread-step
  // rows strided over the grid's warps, 16-weight steps strided over lanes: no integer division
  const int lane = threadIdx.x & 31;
  const int64_t gwarp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t n = gwarp; n < N; n += nwarps) {
    // two 16-weight steps per lane and iteration: eight 16-byte loads in flight
    for (int q0 = lane; q0 < per_row; q0 += 64) {
      uint4 v[2][4];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int q = q0 + 32 * h2;
        const float* src = w + n * ldw + static_cast<int64_t>(q) * 16;
#pragma unroll
        for (int j = 0; j < 4; ++j) v[h2][j] = q < per_row ? ld_global_nc_v4(src + 4 * j) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int q = q0 + 32 * h2;
        if (q >= per_row) continue;
        int c[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          c[4 * j + 0] = ternary_code(__uint_as_float(v[h2][j].x), d, h, fast);
          c[4 * j + 1] = ternary_code(__uint_as_float(v[h2][j].y), d, h, fast);
          c[4 * j + 2] = ternary_code(__uint_as_float(v[h2][j].z), d, h, fast);
          c[4 * j + 3] = ternary_code(__uint_as_float(v[h2][j].w), d, h, fast);
        }
        if constexpr (WF == BL_W_T2) {
          uint32_t word = 0;
#pragma unroll
          for (int j = 0; j < 16; ++j) word |= (static_cast<uint32_t>(c[j]) & 3u) << (2 * j);
          reinterpret_cast<uint32_t*>(out + n * static_cast<int64_t>(K >> 2))[q] = word;
        } else if constexpr (WF == BL_W_E2M1) {
          uint32_t lo = 0, hi = 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            lo |= ((c[j] != 0 ? 2u : 0u) | (c[j] < 0 ? 8u : 0u)) << (4 * j);
            hi |= ((c[8 + j] != 0 ? 2u : 0u) | (c[8 + j] < 0 ? 8u : 0u)) << (4 * j);
          }
          reinterpret_cast<uint2*>(out + n * static_cast<int64_t>(K >> 1))[q] = make_uint2(lo, hi);
        } else {
          uint32_t wd[4];
#pragma unroll
          for (int j = 0; j < 4; ++j)
            wd[j] = (static_cast<uint32_t>(c[4 * j]) & 0xFFu) | ((static_cast<uint32_t>(c[4 * j + 1]) & 0xFFu) << 8) |
                    ((static_cast<uint32_t>(c[4 * j + 2]) & 0xFFu) << 16) | (static_cast<uint32_t>(c[4 * j + 3]) << 24);
          reinterpret_cast<uint4*>(out + n * static_cast<int64_t>(K))[q] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        }
      }
    }
  }
}

}  // namespace bl
