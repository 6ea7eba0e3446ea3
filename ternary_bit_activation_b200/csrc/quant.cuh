// Per-token activation quantizers of BitNet a4.8 (arXiv 2411.04965, §3.4):
//   quant_a4_kernel   -- INT4 absmean (Eq. 6-7) or FP4 E2M1 MinMax (Eq. 8-9)
//   topk_int8 kernels -- Top-K mask + INT8 absmax (Eq. 1), for the raw bf16
//                        input (sparsify_a8) and for h = up * relu(gate)^2
//                        (Eq. 5, relu2_glu)
// All are HBM-bound row kernels: one pass over coalesced 16-byte loads, the row
// held in registers, reductions by warp shuffles and a few shared words.
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

// Index of the nearest E2M1 magnitude {0,.5,1,1.5,2,3,4,6} to a (a >= 0),
// ties to the even index (the encoding with mantissa bit 0).  Each midpoint
// between an even and an odd index uses '>' (the tie stays on the even side
// below), each midpoint between an odd and an even index uses '>='.
__device__ __forceinline__ int e2m1_index(float a) {
  return (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
}

// ---------------------------------------------------------------------------
// quant_a4: 128 threads per row, 2 rows per 256-thread CTA.  Thread t of a row
// holds chunks c*128 + t (8 bf16 each) for c < CHUNKS.
// ---------------------------------------------------------------------------
constexpr int kQ4ThreadsPerRow = 128;

template <int CHUNKS, bool FP4, bool PACKED>
__global__ void __launch_bounds__(256) quant_a4_kernel(const uint16_t* __restrict__ x, int64_t M, int K,
                                                       int64_t ldx, float eps, uint8_t* __restrict__ codes,
                                                       float* __restrict__ scale) {
  __shared__ double s_sum[2][4];
  __shared__ uint32_t s_max[2][4];
  const int sub = threadIdx.x >> 7;
  const int t = threadIdx.x & 127;
  const int warp = t >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 2 + sub;
  const bool row_ok = row < M;
  const int nchunk = K >> 3;
  const uint16_t* xr = x + (row_ok ? row : 0) * ldx;

  uint4 v[CHUNKS];
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int idx = c * kQ4ThreadsPerRow + t;
    v[c] = (row_ok && idx < nchunk) ? ld_global_nc_v4(xr + static_cast<int64_t>(idx) * 8) : make_uint4(0, 0, 0, 0);
  }

  if constexpr (!FP4) {
    // beta = mean|x|: the fp64 sum of bf16 magnitudes is exact for in-contract
    // rows, so the reduction order does not change it.
    double acc = 0.0;
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      float f[8];
      unpack_bf16x8(v[c], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc += static_cast<double>(fabsf(f[e]));
    }
    acc = warp_sum_f64(acc);
    if (lane == 0) s_sum[sub][warp] = acc;
    __syncthreads();
    const double S = (s_sum[sub][0] + s_sum[sub][1]) + (s_sum[sub][2] + s_sum[sub][3]);
    const float beta = __double2float_rn(S / static_cast<double>(K));
    const float mult = __fdiv_rn(sqrt7_f32(), __fadd_rn(beta, eps));
    if (row_ok && t == 0) scale[row] = __fdiv_rn(beta, sqrt7_f32());
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      const int idx = c * kQ4ThreadsPerRow + t;
      if (!row_ok || idx >= nchunk) continue;
      float f[8];
      unpack_bf16x8(v[c], f);
      int q[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) q[e] = round_clip(__fmul_rn(f[e], mult), -8.f, 7.f);
      if constexpr (PACKED) {
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) word |= (static_cast<uint32_t>(q[e]) & 0xFu) << (4 * e);
        reinterpret_cast<uint32_t*>(codes + row * (K >> 1))[idx] = word;
      } else {
        uint2 w2;
        w2.x = (q[0] & 0xFF) | ((q[1] & 0xFF) << 8) | ((q[2] & 0xFF) << 16) | (static_cast<uint32_t>(q[3]) << 24);
        w2.y = (q[4] & 0xFF) | ((q[5] & 0xFF) << 8) | ((q[6] & 0xFF) << 16) | (static_cast<uint32_t>(q[7]) << 24);
        reinterpret_cast<uint2*>(codes + row * static_cast<int64_t>(K))[idx] = w2;
      }
    }
  } else {
    // MinMax FP4: max|x| as the largest 15-bit bf16 magnitude.
    uint32_t mk = 0;
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      uint32_t k[8];
      bf16x8_mag_keys(v[c], k);
#pragma unroll
      for (int e = 0; e < 8; ++e) mk = max(mk, k[e]);
    }
    mk = warp_max_u32(mk);
    if (lane == 0) s_max[sub][warp] = mk;
    __syncthreads();
    mk = max(max(s_max[sub][0], s_max[sub][1]), max(s_max[sub][2], s_max[sub][3]));
    const int p = fp4_scale_exponent(mk << 16);
    if (row_ok && t == 0) scale[row] = exact_pow2(PACKED ? p : p - 1);
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      const int idx = c * kQ4ThreadsPerRow + t;
      if (!row_ok || idx >= nchunk) continue;
      float f[8];
      unpack_bf16x8(v[c], f);
      uint32_t word = 0;
      uint2 w2 = make_uint2(0, 0);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float s = mul_pow2(f[e], -p);
        const int i = e2m1_index(fabsf(s));
        const bool neg = (s < 0.f) && (i != 0);
        if constexpr (PACKED) {
          word |= (static_cast<uint32_t>(i) | (neg ? 8u : 0u)) << (4 * e);
        } else {
          // twice the E2M1 value: {0,1,2,3,4,6,8,12}[i]
          const int tv = (i <= 4) ? i : (i == 5 ? 6 : (i == 6 ? 8 : 12));
          const uint32_t b = static_cast<uint32_t>(neg ? -tv : tv) & 0xFFu;
          if (e < 4) w2.x |= b << (8 * e); else w2.y |= b << (8 * (e - 4));
        }
      }
      if constexpr (PACKED) {
        reinterpret_cast<uint32_t*>(codes + row * (K >> 1))[idx] = word;
      } else {
        reinterpret_cast<uint2*>(codes + row * static_cast<int64_t>(K))[idx] = w2;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Top-K + INT8 (Eq. 1).  One 256-thread CTA per row; thread t holds chunks
// c*256 + t (8 elements each) for c < CHUNKS, as fp32 values.
// Threshold search: if the row has at most `keep` nonzero magnitudes, the
// threshold is 0 (every nonzero survives, zeros fill the rest in index order).
// Otherwise the keep-th largest magnitude key is found by an MSD radix select
// over the nonzero keys (zeros can no longer be the threshold), with one
// private shared-memory histogram per warp merged by warp 0.  Elements tied
// at the threshold key are taken in index order with a block prefix count.
//   F32KEY = false: values came from bf16, key = 15-bit bf16 magnitude.
//   F32KEY = true : values are fp32 (relu2_glu's h), key = 31-bit magnitude.
// ---------------------------------------------------------------------------
constexpr int kTkThreads = 256;
constexpr int kTkWarps = kTkThreads / 32;
constexpr int kTkListCap = 2048;   // candidates kept after the first radix pass

struct TopkSmem {
  uint32_t whist[kTkWarps][256];   // per-warp histograms, zero between passes
  uint32_t wmax[kTkWarps];
  uint32_t wnz[kTkWarps];
  uint32_t sel_digit, sel_above, sel_count;
  uint32_t list_n;
  int32_t tie_off[8][kTkWarps];    // exclusive tie prefix per (chunk, warp)
  int32_t tie_cnt[8][kTkWarps];
  uint32_t list_key[kTkListCap];   // keys of the candidates left after pass 0
};

template <bool F32KEY>
__device__ __forceinline__ uint32_t mag_key(float v) {
  return F32KEY ? (__float_as_uint(v) & 0x7FFFFFFFu) : ((__float_as_uint(v) >> 16) & 0x7FFFu);
}

// Digit layout of the MSD radix select: 8-bit digits from the top, 7 bits last.
template <bool F32KEY>
__device__ __forceinline__ int digit_shift(int pass) {
  return F32KEY ? 23 - 8 * pass : 7 - 7 * pass;   // fp32: 23, 15, 7, 0 (last clamps); bf16: 7, 0
}

// Warp 0: merge the per-warp histograms (zeroing them for the next pass) and
// find the digit d with  above(d) < r <= above(d) + hist[d], where above(d)
// counts candidates whose digit is greater than d.  Lane l owns bins l, l+32,
// ..., so every shared-memory access of the warp hits 32 distinct banks.
__device__ __forceinline__ void merge_select_digit(TopkSmem& sm, int nbins, uint32_t r) {
  const int lane = threadIdx.x & 31;
  const int slots = nbins / 32;  // 8 or 4
  uint32_t h[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = 0;
    if (i < slots) {
      const int b = 32 * i + lane;
#pragma unroll
      for (int w = 0; w < kTkWarps; ++w) {
        h[i] += sm.whist[w][b];
        sm.whist[w][b] = 0;
      }
    }
  }
  uint32_t above_slots = 0;   // candidates in slots above the current one
#pragma unroll
  for (int i = 7; i >= 0; --i) {
    if (i >= slots) continue;
    uint32_t inc = h[i];      // inclusive suffix sum over lanes >= lane within slot i
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t other = __shfl_down_sync(0xFFFFFFFFu, inc, o);
      if (lane + o < 32) inc += other;
    }
    const uint32_t above = above_slots + inc - h[i];
    if (above < r && r <= above + h[i]) {
      sm.sel_digit = static_cast<uint32_t>(32 * i + lane);
      sm.sel_above = above;
      sm.sel_count = h[i];
    }
    above_slots += __shfl_sync(0xFFFFFFFFu, inc, 0);   // the slot's total
  }
}

template <int CHUNKS, bool F32KEY>
__device__ __forceinline__ void topk_int8_row(const float (&val)[CHUNKS][8], int K, int keep, float eps,
                                              int64_t row, int8_t* __restrict__ codes,
                                              float* __restrict__ scale, uint32_t* __restrict__ mask,
                                              TopkSmem& sm) {
  const int t = threadIdx.x;
  const int lane = t & 31;
  const int warp = t >> 5;
  const int nchunk = K >> 3;
  constexpr int kPasses = F32KEY ? 4 : 2;

  // each warp clears its own histogram; the barrier below orders it
  for (int i = lane; i < 256; i += 32) sm.whist[warp][i] = 0;
  if (t == 0) sm.list_n = 0;

  // gamma = max |x| (largest key) and the number of nonzero magnitudes
  uint32_t mk = 0, nz = 0;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c)
    if (c * kTkThreads + t < nchunk)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t key = mag_key<F32KEY>(val[c][e]);
        mk = max(mk, key);
        nz += key != 0u;
      }
  mk = __reduce_max_sync(0xFFFFFFFFu, mk);
  nz = __reduce_add_sync(0xFFFFFFFFu, nz);
  if (lane == 0) {
    sm.wmax[warp] = mk;
    sm.wnz[warp] = nz;
  }
  __syncthreads();
  uint32_t gk = 0, nnz = 0;
#pragma unroll
  for (int w = 0; w < kTkWarps; ++w) {
    gk = max(gk, sm.wmax[w]);
    nnz += sm.wnz[w];
  }

  uint32_t thr, take, tie_total;
  if (nnz <= static_cast<uint32_t>(keep)) {
    thr = 0;                                   // every nonzero survives; zeros fill in index order
    take = static_cast<uint32_t>(keep) - nnz;
    tie_total = static_cast<uint32_t>(K) - nnz;
  } else {
    // MSD radix select of the keep-th largest nonzero key.
    uint32_t prefix = 0, fixed = 0, r = static_cast<uint32_t>(keep);
    tie_total = 0;
    bool listed = false;   // candidates compacted into sm.list_key after pass 0
#pragma unroll 1
    for (int pass = 0; pass < kPasses; ++pass) {
      const int shift = max(digit_shift<F32KEY>(pass), 0);
      const int width = shift == 0 ? 7 : 8;
      const uint32_t dmask = (1u << width) - 1u;
      uint32_t* hist = sm.whist[warp];
      if (listed) {
        const int n = static_cast<int>(sm.list_n);
        for (int i = t; i < n; i += kTkThreads) {
          const uint32_t key = sm.list_key[i];
          if ((key & fixed) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
        }
      } else {
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
          if (c * kTkThreads + t < nchunk) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const uint32_t key = mag_key<F32KEY>(val[c][e]);
              if (key != 0u && (key & fixed) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
            }
          }
        }
      }
      __syncthreads();
      if (warp == 0) merge_select_digit(sm, 1 << width, r);
      __syncthreads();
      const uint32_t d = sm.sel_digit;
      r -= sm.sel_above;
      tie_total = sm.sel_count;
      prefix |= d << shift;
      fixed |= dmask << shift;
      if (pass == 0 && pass + 1 < kPasses && tie_total <= static_cast<uint32_t>(kTkListCap)) {
        // compact the candidates left after the top digit; later passes read only them
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
          const bool chunk_ok = c * kTkThreads + t < nchunk;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t key = mag_key<F32KEY>(val[c][e]);
            const bool cand = chunk_ok && key != 0u && (key & fixed) == prefix;
            const uint32_t bal = __ballot_sync(0xFFFFFFFFu, cand);
            if (bal) {
              uint32_t base = 0;
              if (lane == __ffs(bal) - 1) base = atomicAdd(&sm.list_n, static_cast<uint32_t>(__popc(bal)));
              base = __shfl_sync(0xFFFFFFFFu, base, __ffs(bal) - 1);
              if (cand) sm.list_key[base + __popc(bal & ((1u << lane) - 1u))] = key;
            }
          }
        }
        __syncthreads();
        listed = true;
      }
    }
    thr = prefix;   // key of the keep-th largest element
    take = r;       // how many elements with key == thr survive (in index order)
  }

  // Index-ordered rank among the ties, needed only when some ties are dropped.
  int tie_base[CHUNKS];
  const bool partial = take < tie_total;
  if (partial) {
    int cnt[CHUNKS];
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      cnt[c] = 0;
      if (c * kTkThreads + t < nchunk)
#pragma unroll
        for (int e = 0; e < 8; ++e) cnt[c] += (mag_key<F32KEY>(val[c][e]) == thr);
      int inc = cnt[c];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int other = __shfl_up_sync(0xFFFFFFFFu, inc, o);
        if (lane >= o) inc += other;
      }
      tie_base[c] = inc - cnt[c];  // exclusive within the warp
      if (lane == 31) sm.tie_cnt[c][warp] = inc;
    }
    __syncthreads();
    if (t == 0) {
      int run = 0;
      for (int c = 0; c < CHUNKS; ++c)
        for (int w = 0; w < kTkWarps; ++w) {
          sm.tie_off[c][w] = run;
          run += sm.tie_cnt[c][w];
        }
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) tie_base[c] += sm.tie_off[c][warp];
  } else {
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) tie_base[c] = 0;
  }

  const float gamma = F32KEY ? __uint_as_float(gk) : __uint_as_float(gk << 16);
  const float mult = __fdiv_rn(127.f, __fadd_rn(gamma, eps));
  if (t == 0) scale[row] = __fdiv_rn(gamma, 127.f);

  const int mwords = (K + 31) >> 5;
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int q = c * kTkThreads + t;
    const bool ok = q < nchunk;
    uint32_t bits = 0;
    uint2 w2 = make_uint2(0, 0);
    int rank = tie_base[c];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t key = mag_key<F32KEY>(val[c][e]);
      bool keepit = key > thr;
      if (key == thr) {
        keepit = !partial || rank < static_cast<int>(take);
        ++rank;
      }
      keepit = keepit && ok;
      const int code = keepit ? round_clip(__fmul_rn(val[c][e], mult), -128.f, 127.f) : 0;
      bits |= (keepit ? 1u : 0u) << e;
      const uint32_t b = static_cast<uint32_t>(code) & 0xFFu;
      if (e < 4) w2.x |= b << (8 * e); else w2.y |= b << (8 * (e - 4));
    }
    if (ok) reinterpret_cast<uint2*>(codes + row * static_cast<int64_t>(K))[q] = w2;
    if (mask != nullptr) {
      // four consecutive chunks (lanes 4j..4j+3) make one 32-bit mask word
      const uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, bits, 1);
      const uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, bits, 2);
      const uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, bits, 3);
      if (ok && (t & 3) == 0) {
        const uint32_t word = bits | (b1 << 8) | (b2 << 16) | (b3 << 24);
        mask[row * mwords + (q >> 2)] = word;
      }
    }
  }
}

template <int CHUNKS>
__global__ void __launch_bounds__(kTkThreads, CHUNKS <= 2 ? 6 : 3) sparsify_a8_kernel(const uint16_t* __restrict__ x, int K, int64_t ldx,
                                                                 int keep, float eps, int8_t* __restrict__ codes,
                                                                 float* __restrict__ scale,
                                                                 uint32_t* __restrict__ mask) {
  __shared__ TopkSmem sm;
  const int64_t row = blockIdx.x;
  const int t = threadIdx.x;
  const int nchunk = K >> 3;
  const uint16_t* xr = x + row * ldx;
  float val[CHUNKS][8];
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int idx = c * kTkThreads + t;
    const uint4 v = idx < nchunk ? ld_global_nc_v4(xr + static_cast<int64_t>(idx) * 8) : make_uint4(0, 0, 0, 0);
    unpack_bf16x8(v, val[c]);
  }
  topk_int8_row<CHUNKS, false>(val, K, keep, eps, row, codes, scale, mask, sm);
}

// h = up * max(0, gate)^2 in fp32 (two roundings: g2 = g*g, h = up*g2), Eq. 5.
template <int CHUNKS>
__global__ void __launch_bounds__(kTkThreads) relu2_glu_kernel(const uint16_t* __restrict__ gate,
                                                               const uint16_t* __restrict__ up, int F, int64_t ld,
                                                               int keep, float eps, int8_t* __restrict__ codes,
                                                               float* __restrict__ scale,
                                                               uint32_t* __restrict__ mask) {
  __shared__ TopkSmem sm;
  const int64_t row = blockIdx.x;
  const int t = threadIdx.x;
  const int nchunk = F >> 3;
  const uint16_t* gr = gate + row * ld;
  const uint16_t* ur = up + row * ld;
  float val[CHUNKS][8];
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    const int idx = c * kTkThreads + t;
    uint4 gv = make_uint4(0, 0, 0, 0), uv = make_uint4(0, 0, 0, 0);
    if (idx < nchunk) {
      gv = ld_global_nc_v4(gr + static_cast<int64_t>(idx) * 8);
      uv = ld_global_nc_v4(ur + static_cast<int64_t>(idx) * 8);
    }
    float g[8], u[8];
    unpack_bf16x8(gv, g);
    unpack_bf16x8(uv, u);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float rg = g[e] > 0.f ? g[e] : 0.f;
      val[c][e] = __fmul_rn(u[e], __fmul_rn(rg, rg));
    }
  }
  topk_int8_row<CHUNKS, true>(val, F, keep, eps, row, codes, scale, mask, sm);
}

// ReLU^2-GLU + Top-K + INT8, persistent: each CTA walks rows blockIdx.x,
// blockIdx.x + gridDim.x, ...  Every thread copies its own chunks of the next
// row's gate and up into shared memory with cp.async while the current row is
// selected, so each CTA always has a row load in flight.  A thread overwrites a
// chunk only after pulling it into registers, so no barrier guards the buffer.
template <int CHUNKS>
__global__ void __launch_bounds__(kTkThreads, 3) relu2_glu_persistent_kernel(
    const uint16_t* __restrict__ gate, const uint16_t* __restrict__ up, int64_t M, int F, int64_t ld, int keep,
    float eps, int8_t* __restrict__ codes, float* __restrict__ scale, uint32_t* __restrict__ mask) {
  __shared__ TopkSmem sm;
  extern __shared__ uint4 rowbuf[];        // [CHUNKS][256] gate words, then [CHUNKS][256] up words
  const int t = threadIdx.x;
  const int nchunk = F >> 3;
  uint4* gbuf = rowbuf;
  uint4* ubuf = rowbuf + CHUNKS * kTkThreads;

  auto prefetch = [&](int64_t row) {
    const uint16_t* gr = gate + row * ld;
    const uint16_t* ur = up + row * ld;
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      const int idx = c * kTkThreads + t;
      if (idx < nchunk) {
        cp_async_16(&gbuf[c * kTkThreads + t], gr + static_cast<int64_t>(idx) * 8);
        cp_async_16(&ubuf[c * kTkThreads + t], ur + static_cast<int64_t>(idx) * 8);
      }
    }
    cp_async_commit();
  };

  int64_t row = blockIdx.x;
  if (row < M) prefetch(row);
  for (; row < M; row += gridDim.x) {
    cp_async_wait_all();
    float val[CHUNKS][8];
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
      const int idx = c * kTkThreads + t;
      uint4 gv = make_uint4(0, 0, 0, 0), uv = make_uint4(0, 0, 0, 0);
      if (idx < nchunk) {
        gv = gbuf[c * kTkThreads + t];
        uv = ubuf[c * kTkThreads + t];
      }
      float g[8], u[8];
      unpack_bf16x8(gv, g);
      unpack_bf16x8(uv, u);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float rg = g[e] > 0.f ? g[e] : 0.f;
        val[c][e] = __fmul_rn(u[e], __fmul_rn(rg, rg));
      }
    }
    const int64_t next = row + gridDim.x;
    if (next < M) prefetch(next);
    topk_int8_row<CHUNKS, true>(val, F, keep, eps, row, codes, scale, mask, sm);
    __syncthreads();   // all threads finish this row's shared-memory use before the next row starts
  }
}

}  // namespace bl