// Post-RoPE low-bit KV-cache quantizer (BitNet a4.8, §3.4 "Low-Bit KV Cache
// Quantization"): absmax per (position, head) vector to unsigned b-bit codes;
// for 3-bit caches the beginning-of-sequence position is kept at 4 bits.
//   Q = 2^(b-1) - 1,  c = RoundClip(Q/(gamma+eps) * x, -Q-1, Q),  stored c + 2^(b-1)
// One vector of D values is handled by D/8 threads (8 values per thread, one
// 16-byte load); each thread group handles kKvItems vectors.  3-bit output: each thread's 8 codes form a 24-bit word, and
// four neighbouring threads (32 codes = 12 bytes) are stored by the first as
// three 32-bit words.
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kKvItems = 4;  // vectors per thread group, loaded before any is processed

template <int TPV>  // threads per vector = D / 8, one of 4, 8, 16, 32
__global__ void __launch_bounds__(256) kv_quant_kernel(const uint16_t* __restrict__ kv, int64_t T, int H,
                                                       int64_t ldt, int bits, int64_t bos_pos, float eps,
                                                       uint8_t* __restrict__ codes, float* __restrict__ scale,
                                                       uint8_t* __restrict__ bos_codes) {
  constexpr int D = TPV * 8;
  const int lane = threadIdx.x & 31;
  const int sub = lane % TPV;  // position inside the vector's thread group
  // the host keeps T * H below 2^31, so vector indices fit 32-bit arithmetic
  const uint32_t group = (blockIdx.x * blockDim.x + threadIdx.x) / TPV;
  const uint32_t ngroups = gridDim.x * blockDim.x / TPV;
  const uint32_t nvec = static_cast<uint32_t>(T) * static_cast<uint32_t>(H);
  const uint32_t uh = static_cast<uint32_t>(H);

  // group g handles vectors g, g + ngroups, ... so neighbouring groups read
  // neighbouring vectors in every round
  uint4 v[kKvItems];
#pragma unroll
  for (int it = 0; it < kKvItems; ++it) {
    const uint32_t vec = group + it * ngroups;
    v[it] = make_uint4(0, 0, 0, 0);
    if (vec < nvec) {
      const uint32_t t = vec / uh;
      const uint32_t h = vec - t * uh;
      v[it] = ld_global_nc_v4(kv + static_cast<int64_t>(t) * ldt + static_cast<int64_t>(h) * D + sub * 8);
    }
  }

#pragma unroll
  for (int it = 0; it < kKvItems; ++it) {
    const uint32_t vec = group + it * ngroups;
    const bool ok = vec < nvec;
    const uint32_t t = ok ? vec / uh : 0u;
    const uint32_t h = ok ? vec - t * uh : 0u;

    uint32_t k[8];
    bf16x8_mag_keys(v[it], k);
    uint32_t mk = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) mk = max(mk, k[e]);
#pragma unroll
    for (int o = TPV / 2; o > 0; o >>= 1) mk = max(mk, __shfl_xor_sync(0xFFFFFFFFu, mk, o));
    const float gamma = __uint_as_float(mk << 16);

    const bool is_bos = (bits == 3) && (static_cast<int64_t>(t) == bos_pos);
    const int b = is_bos ? 4 : bits;
    const float qmax = static_cast<float>((1 << (b - 1)) - 1);
    const float mult = __fdiv_rn(qmax, __fadd_rn(gamma, eps));
    if (ok && sub == 0) scale[vec] = __fdiv_rn(gamma, qmax);

    float f[8];
    unpack_bf16x8(v[it], f);
    uint32_t u[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      u[e] = static_cast<uint32_t>(round_clip(__fmul_rn(f[e], mult), -qmax - 1.f, qmax) + (1 << (b - 1)));

    if (b == 4) {
      uint32_t word = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) word |= u[e] << (4 * e);
      if (ok) {
        if (is_bos) {
          reinterpret_cast<uint32_t*>(bos_codes + static_cast<int64_t>(h) * (D / 2))[sub] = word;
        } else {
          reinterpret_cast<uint32_t*>(codes + static_cast<int64_t>(vec) * (D / 2))[sub] = word;
        }
      }
    }
    // 3-bit layout (also zero-fills the BOS row's 3-bit slot).  All lanes take
    // part in the shuffles; the launch-uniform condition keeps them converged.
    if (bits == 3) {
      uint32_t w24 = 0;
      if (!is_bos) {
#pragma unroll
        for (int e = 0; e < 8; ++e) w24 |= u[e] << (3 * e);
      }
      const uint32_t w1 = __shfl_down_sync(0xFFFFFFFFu, w24, 1);
      const uint32_t w2 = __shfl_down_sync(0xFFFFFFFFu, w24, 2);
      const uint32_t w3 = __shfl_down_sync(0xFFFFFFFFu, w24, 3);
      if (ok && (sub & 3) == 0) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(codes + static_cast<int64_t>(vec) * (D * 3 / 8) + (sub / 4) * 12);
        dst[0] = w24 | (w1 << 24);
        dst[1] = (w1 >> 8) | (w2 << 16);
        dst[2] = (w2 >> 16) | (w3 << 8);
      }
    }
  }
}

}  // namespace bl
