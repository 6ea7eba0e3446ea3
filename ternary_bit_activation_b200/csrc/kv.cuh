// Post-RoPE low-bit KV-cache quantizer (BitNet a4.8, §3.4 "Low-Bit KV Cache
// Quantization"): absmax per (position, head) vector to unsigned b-bit codes;
// for 3-bit caches the beginning-of-sequence position is kept at 4 bits.
//   Q = 2^(b-1) - 1,  c = RoundClip(Q/(gamma+eps) * x, -Q-1, Q),  stored c + 2^(b-1)
// One vector of D values is handled by D/32 threads (32 values per thread, four
// 16-byte loads), so the two divisions and the max reduction of a vector are
// shared by 32 values a thread.  The grid is persistent: each thread group takes kKvItems
// vectors per round and loads the next round's vectors before it quantizes the
// current ones; (position, head) of a group's vectors advance by a fixed step,
// so no integer division is needed.  3-bit output: a thread's 32 codes are
// three 32-bit words (12 bytes); 4-bit output is one 16-byte word a thread.
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kKvItems = 1;  // vectors per thread group and round

// A vector's (position, head) and linear index, advanced by `step` vectors.
struct KvPos {
  uint32_t t, h, vec;
  __device__ __forceinline__ void advance(uint32_t dt, uint32_t dh, uint32_t step, uint32_t H) {
    vec += step;
    t += dt;
    h += dh;
    if (h >= H) {
      h -= H;
      ++t;
    }
  }
};

template <int TPV>
__device__ __forceinline__ void kv_load(const uint16_t* kv, KvPos p, uint32_t dt, uint32_t dh, uint32_t step,
                                        uint32_t H, uint32_t nvec, int64_t ldt, int sub, uint4 (&v)[kKvItems][4]) {
  constexpr int D = TPV * 32;
#pragma unroll
  for (int it = 0; it < kKvItems; ++it) {
#pragma unroll
    for (int j = 0; j < 4; ++j) v[it][j] = make_uint4(0, 0, 0, 0);
    if (p.vec < nvec) {
      const uint16_t* src = kv + static_cast<int64_t>(p.t) * ldt + static_cast<int64_t>(p.h) * D + sub * 32;
#pragma unroll
      for (int j = 0; j < 4; ++j) v[it][j] = ld_global_nc_v4(src + 8 * j);
    }
    p.advance(dt, dh, step, H);
  }
}

template <int TPV>  // threads per vector = D / 32, one of 1, 2, 4, 8
__global__ void __launch_bounds__(256) kv_quant_kernel(const uint16_t* __restrict__ kv, int64_t T, int H,
                                                       int64_t ldt, int bits, int64_t bos_pos, float eps,
                                                       uint8_t* __restrict__ codes, float* __restrict__ scale,
                                                       uint8_t* __restrict__ bos_codes) {
  constexpr int D = TPV * 32;
  const int lane = threadIdx.x & 31;
  const int sub = lane % TPV;  // position inside the vector's thread group
  // the host keeps T * H below 2^31, so vector indices fit 32-bit arithmetic
  const uint32_t group = (blockIdx.x * blockDim.x + threadIdx.x) / TPV;
  const uint32_t ngroups = gridDim.x * blockDim.x / TPV;
  const uint32_t nvec = static_cast<uint32_t>(T) * static_cast<uint32_t>(H);
  const uint32_t uh = static_cast<uint32_t>(H);
  // vectors of a group: group + i * ngroups, i = 0, 1, ...
  const uint32_t dt = ngroups / uh, dh = ngroups - (ngroups / uh) * uh;

  KvPos p;
  p.vec = group;
  p.t = group / uh;
  p.h = group - p.t * uh;
  uint4 v[kKvItems][4];
  pdl_wait();
  pdl_trigger();
  kv_load<TPV>(kv, p, dt, dh, ngroups, uh, nvec, ldt, sub, v);
  // rounds continue while the warp's first group has a vector left, so every
  // lane takes part in every shuffle (lanes past the end only skip their stores)
  uint32_t warp_vec = (blockIdx.x * blockDim.x + (threadIdx.x & ~31u)) / TPV;
  for (; warp_vec < nvec; warp_vec += ngroups * kKvItems) {
    KvPos nx_p = p;
#pragma unroll
    for (int it = 0; it < kKvItems; ++it) nx_p.advance(dt, dh, ngroups, uh);
    uint4 nx[kKvItems][4];
    kv_load<TPV>(kv, nx_p, dt, dh, ngroups, uh, nvec, ldt, sub, nx);
#pragma unroll
    for (int it = 0; it < kKvItems; ++it) {
      const bool ok = p.vec < nvec;
      uint32_t mk = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t k[8];
        bf16x8_mag_keys(v[it][j], k);
#pragma unroll
        for (int e = 0; e < 8; ++e) mk = max(mk, k[e]);
      }
#pragma unroll
      for (int o = TPV / 2; o > 0; o >>= 1) mk = max(mk, __shfl_xor_sync(0xFFFFFFFFu, mk, o));
      const float gamma = __uint_as_float(mk << 16);

      const bool is_bos = (bits == 3) && (static_cast<int64_t>(p.t) == bos_pos);
      const int b = is_bos ? 4 : bits;
      const float qmax = static_cast<float>((1 << (b - 1)) - 1);
      const float denom = __fadd_rn(gamma, eps);
      const float mult = denom > 0.f ? __fdiv_rn(qmax, denom) : 0.f;
      if (ok && sub == 0) scale[p.vec] = __fdiv_rn(gamma, qmax);

      // |x * mult| <= qmax, so RoundClip needs no clip: rint_even by adding
      // 1.5*2^23 plus the (even) unsigned offset 2^(b-1); the code sits in the
      // low bits of the sum's bit pattern
      const float magic = 12582912.0f + static_cast<float>(1 << (b - 1));
      uint32_t u[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float f[8];
        unpack_bf16x8(v[it][j], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) u[8 * j + e] = __float_as_uint(__fadd_rn(__fmul_rn(f[e], mult), magic)) & 0xFu;
      }

      if (b == 4) {
        uint4 w4 = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          w4.x |= u[e] << (4 * e);
          w4.y |= u[8 + e] << (4 * e);
          w4.z |= u[16 + e] << (4 * e);
          w4.w |= u[24 + e] << (4 * e);
        }
        if (ok) {
          uint8_t* dst = is_bos ? bos_codes + static_cast<int64_t>(p.h) * (D / 2)
                                : codes + static_cast<int64_t>(p.vec) * (D / 2);
          reinterpret_cast<uint4*>(dst)[sub] = w4;
        }
      }
      // 3-bit layout (also zero-fills the BOS row's 3-bit slot): a thread's 32
      // codes are exactly three 32-bit words
      if (bits == 3 && ok) {
        uint32_t w0 = 0, w1 = 0, w2 = 0;
        if (!is_bos) {
          uint64_t a = 0, c = 0;   // codes 0-15 and 16-31, 48 bits each
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            a |= static_cast<uint64_t>(u[e]) << (3 * e);
            c |= static_cast<uint64_t>(u[16 + e]) << (3 * e);
          }
          w0 = static_cast<uint32_t>(a);
          w1 = static_cast<uint32_t>(a >> 32) | (static_cast<uint32_t>(c) << 16);
          w2 = static_cast<uint32_t>(c >> 16);
        }
        uint32_t* dst = reinterpret_cast<uint32_t*>(codes + static_cast<int64_t>(p.vec) * (D * 3 / 8) + sub * 12);
        dst[0] = w0;
        dst[1] = w1;
        dst[2] = w2;
      }
      p.advance(dt, dh, ngroups, uh);
    }
#pragma unroll
    for (int it = 0; it < kKvItems; ++it)
#pragma unroll
      for (int j = 0; j < 4; ++j) v[it][j] = nx[it][j];
  }
}

}  // namespace bl
