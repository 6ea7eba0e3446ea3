// Post-RoPE low-bit KV-cache quantizer (BitNet a4.8, §3.4 "Low-Bit KV Cache
// Quantization"): absmax per (position, head) vector to unsigned b-bit codes;
// for 3-bit caches the beginning-of-sequence position is kept at 4 bits.
//   Q = 2^(b-1) - 1,  c = RoundClip(Q/(gamma+eps) * x, -Q-1, Q),  stored c + 2^(b-1)
// One vector of D values is handled by D/16 threads (16 values per thread, two
// 16-byte loads).  The grid is persistent: each thread group takes kKvItems
// vectors per round and loads the next round's vectors before it quantizes the
// current ones; (position, head) of a group's vectors advance by a fixed step,
// so no integer division is needed.  3-bit output: each thread's 16 codes form
// a 48-bit word and two neighbouring threads (32 codes = 12 bytes) are stored
// by the first as three 32-bit words; 4-bit output is one 64-bit word a thread.
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kKvItems = 2;  // vectors per thread group and round

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
                                        uint32_t H, uint32_t nvec, int64_t ldt, int sub, uint4 (&v)[kKvItems][2]) {
  constexpr int D = TPV * 16;
#pragma unroll
  for (int it = 0; it < kKvItems; ++it) {
    v[it][0] = v[it][1] = make_uint4(0, 0, 0, 0);
    if (p.vec < nvec) {
      const uint16_t* src = kv + static_cast<int64_t>(p.t) * ldt + static_cast<int64_t>(p.h) * D + sub * 16;
      v[it][0] = ld_global_nc_v4(src);
      v[it][1] = ld_global_nc_v4(src + 8);
    }
    p.advance(dt, dh, step, H);
  }
}

template <int TPV>  // threads per vector = D / 16, one of 2, 4, 8, 16
__global__ void __launch_bounds__(256) kv_quant_kernel(const uint16_t* __restrict__ kv, int64_t T, int H,
                                                       int64_t ldt, int bits, int64_t bos_pos, float eps,
                                                       uint8_t* __restrict__ codes, float* __restrict__ scale,
                                                       uint8_t* __restrict__ bos_codes) {
  constexpr int D = TPV * 16;
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
  uint4 v[kKvItems][2];
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
    uint4 nx[kKvItems][2];
    kv_load<TPV>(kv, nx_p, dt, dh, ngroups, uh, nvec, ldt, sub, nx);
#pragma unroll
    for (int it = 0; it < kKvItems; ++it) {
      const bool ok = p.vec < nvec;
      uint32_t k[16];
      bf16x8_mag_keys(v[it][0], *reinterpret_cast<uint32_t(*)[8]>(&k[0]));
      bf16x8_mag_keys(v[it][1], *reinterpret_cast<uint32_t(*)[8]>(&k[8]));
      uint32_t mk = 0;
#pragma unroll
      for (int e = 0; e < 16; ++e) mk = max(mk, k[e]);
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
      float f[16];
      unpack_bf16x8(v[it][0], *reinterpret_cast<float(*)[8]>(&f[0]));
      unpack_bf16x8(v[it][1], *reinterpret_cast<float(*)[8]>(&f[8]));
      uint32_t u[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) u[e] = __float_as_uint(__fadd_rn(__fmul_rn(f[e], mult), magic)) & 0xFu;

      if (b == 4) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          lo |= u[e] << (4 * e);
          hi |= u[8 + e] << (4 * e);
        }
        if (ok) {
          uint8_t* dst = is_bos ? bos_codes + static_cast<int64_t>(p.h) * (D / 2)
                                : codes + static_cast<int64_t>(p.vec) * (D / 2);
          reinterpret_cast<uint2*>(dst)[sub] = make_uint2(lo, hi);
        }
      }
      // 3-bit layout (also zero-fills the BOS row's 3-bit slot).  All lanes take
      // part in the shuffles; the launch-uniform condition keeps them converged.
      if (bits == 3) {
        uint32_t w0 = 0, w1 = 0;   // 48 bits: codes 0-10 (and bit 0-1 of 10) / the rest
        if (!is_bos) {
          uint64_t w48 = 0;
#pragma unroll
          for (int e = 0; e < 16; ++e) w48 |= static_cast<uint64_t>(u[e]) << (3 * e);
          w0 = static_cast<uint32_t>(w48);
          w1 = static_cast<uint32_t>(w48 >> 32);
        }
        const uint32_t n0 = __shfl_down_sync(0xFFFFFFFFu, w0, 1);
        const uint32_t n1 = __shfl_down_sync(0xFFFFFFFFu, w1, 1);
        if (ok && (sub & 1) == 0) {
          uint32_t* dst = reinterpret_cast<uint32_t*>(codes + static_cast<int64_t>(p.vec) * (D * 3 / 8) + (sub / 2) * 12);
          // bits 0-47: this thread, bits 48-95: the next one
          dst[0] = w0;
          dst[1] = (w1 & 0xFFFFu) | (n0 << 16);
          dst[2] = (n0 >> 16) | (n1 << 16);
        }
      }
      p.advance(dt, dh, ngroups, uh);
    }
#pragma unroll
    for (int it = 0; it < kKvItems; ++it) {
      v[it][0] = nx[it][0];
      v[it][1] = nx[it][1];
    }
  }
}

}  // namespace bl
