// Top-K + INT8 absmax quantization of token rows (BitNet a4.8, arXiv 2411.04965,
// §3.4, Eq. 1 with Q_INT8), for the raw bf16 inputs (sparsify_a8) and for the
// ReLU^2-GLU output h = up * max(0, gate)^2 in fp32 (Eq. 5, relu2_glu).
//
// One 256-thread CTA owns one row at a time (persistent over rows).  Rows stream
// through a shared-memory stage (cp.async, 16 B per copy), so HBM is read once
// per element.  bf16 rows are double-buffered: the next row is in flight while
// the current one is ranked and quantized.  ReLU^2 rows (gate and up, 44 KB at
// the 7B FFN width) take a single stage so that three CTAs fit on an SM; the
// other CTAs' ranking covers each row's load.  For ReLU^2 rows the first sweep
// writes h over the staged gate/up values of its own chunk, so later sweeps read h.
//
// Selection: exactly `keep` survivors ranked by magnitude, ties to the lower
// index.  The keep-th largest magnitude key is found by an MSD radix select:
// bf16 keys (15 bits) take an 8-bit then a 7-bit digit (the first counted in the
// same sweep that finds the row maximum); fp32 keys (31 bits) take 8, 8, 8 and
// 7 bits, and once two digits are fixed the few candidates left go to a short
// list that the last passes read.  A full-row pass counts digits with shared
// atomics into lane-private counter words (word bin*32 + lane for bf16, two
// 16-bit bins per word for fp32), so a warp's 32 lanes always hit 32 different
// banks; thread t then sums bin t over the 32 lane columns.  ReLU^2 rows with
// at most `keep` nonzero values need no pass: every nonzero survives and zeros
// fill the rest in index order.
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kTkThreads = 256;            // one row per CTA
constexpr int kTkMaxSlots = 8;             // chunks of 8 values per thread and row (K <= 16384)
constexpr int kTkListCap = 1024;           // fp32 candidates once two digits are fixed

template <bool F32>
struct __align__(16) TkShared {
  uint32_t cnt[F32 ? 2048 : 4096];         // 256 bins x 16 columns (u32, or u16 pairs for fp32)
  uint32_t tot[256];                       // bin totals of the current pass
  uint32_t red[8][2];                      // per-warp max key / nonzero count
  uint32_t scan[8];                        // per-warp tie counts (rank scan)
  uint32_t sel[4];                         // selected digit, count above it, its count
  uint32_t hist[2][F32 ? 256 : 1];         // list passes (fp32 keys)
  uint32_t list_n;
  uint32_t list[F32 ? kTkListCap : 1];
  uint32_t maskw[kTkMaxSlots * kTkThreads / 4];   // mask bits of the row, 8 per chunk
  uint16_t tiec[F32 ? kTkMaxSlots * kTkThreads : 2];   // fp32 rows: ties per chunk, then their prefix
};

// Bytes of dynamic shared memory for rows of K values.
// Row stages per CTA (see above).
template <bool F32>
constexpr int kTkStages = F32 ? 1 : 2;

template <bool F32>
inline size_t tk_smem_bytes(int K) {
  return sizeof(TkShared<F32>) + kTkStages<F32> * static_cast<size_t>(F32 ? 2 : 1) * static_cast<size_t>(K) * 2;
}

// Counter update: `inc` (0 or 1) for digit `bin`.  Lanes l and l+16 share a
// counter column; a warp's other lanes hit 16 different banks.
template <bool F32>
__device__ __forceinline__ void tk_count(uint32_t* cnt, uint32_t bin, int col, uint32_t inc) {
  if constexpr (F32) {
    atomicAdd(&cnt[((bin >> 1) << 4) + col], inc << ((bin & 1u) << 4));   // two 16-bit bins per word
  } else {
    atomicAdd(&cnt[(bin << 4) + col], inc);
  }
}

// Sum of bin b over the 16 counter columns: four 16-byte loads, the quarter
// order rotated by (lane / 2) % 4 so that each 8-lane phase of a load covers 8
// different 4-bank groups (lanes 2m and 2m+1 read the same words for fp32).
template <bool F32>
__device__ __forceinline__ uint32_t tk_bin_total(const uint32_t* cnt, uint32_t b, int lane) {
  const int rot = (lane >> 1) & 3;
  const uint4* w = reinterpret_cast<const uint4*>(cnt + ((F32 ? (b >> 1) : b) << 4));
  uint32_t s = 0;
  if constexpr (F32) {
    const int sh = (b & 1u) ? 16 : 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 v = w[(rot + j) & 3];
      s += ((v.x >> sh) & 0xFFFFu) + ((v.y >> sh) & 0xFFFFu) + ((v.z >> sh) & 0xFFFFu) + ((v.w >> sh) & 0xFFFFu);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 v = w[(rot + j) & 3];
      s += (v.x + v.y) + (v.z + v.w);
    }
  }
  return s;
}

// Within one warp: the digit d with above(d) < r <= above(d) + count(d),
// counting from the largest digit; t[i] = count of bin 8*lane + i.
// Lane 0 of the warp returns the result in out[0..2].
__device__ __forceinline__ void tk_select(const uint32_t (&t)[8], uint32_t r, int lane, uint32_t* out) {
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += t[i];
  uint32_t incl = s;                       // sum over lanes >= lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, incl, o);
    if (lane + o < 32) incl += v;
  }
  uint32_t above = incl - s;
#pragma unroll
  for (int i = 7; i >= 0; --i) {
    if (above < r && r <= above + t[i]) {
      out[0] = static_cast<uint32_t>(8 * lane + i);
      out[1] = above;
      out[2] = t[i];
    }
    above += t[i];
  }
}

// Low byte of the bits of RN(RN(v*mult) + 1.5*2^23): the code RoundClip(v*mult)
// for |v*mult| <= 127 (the sum's ulp is 1, so it rounds half to even; the
// product is rounded first, as the quantizer prescribes).
__device__ __forceinline__ uint32_t tk_code_bits(float v, float mult) {
  return __float_as_uint(__fadd_rn(__fmul_rn(v, mult), 12582912.0f));
}

// Bytes e of lo/hi = code of value e when bit e of `bits` is set, else 0.
__device__ __forceinline__ uint2 tk_pack_codes(const uint32_t (&cb)[8], uint32_t bits) {
  const uint32_t lo = __byte_perm(__byte_perm(cb[0], cb[1], 0x0040), __byte_perm(cb[2], cb[3], 0x0040), 0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(cb[4], cb[5], 0x0040), __byte_perm(cb[6], cb[7], 0x0040), 0x5410);
  // spread 4 mask bits to 4 bytes of 0x01, then to 0xFF
  const uint32_t ml = ((((bits & 0xFu) * 0x00204081u) & 0x01010101u) * 0xFFu);
  const uint32_t mh = (((((bits >> 4) & 0xFu) * 0x00204081u) & 0x01010101u) * 0xFFu);
  return make_uint2(lo & ml, hi & mh);
}

template <bool F32>
__device__ __forceinline__ void tk_keys(const uint4* st, int q, int row_words, uint32_t (&k)[8], float (&f)[8]) {
  if constexpr (F32) {
    const uint4 a = st[q], b = st[row_words + q];   // h written in place: values 0-3, then 4-7
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      f[e] = __uint_as_float(w[e]);
      k[e] = w[e] & 0x7FFFFFFFu;
    }
  } else {
    const uint4 v = st[q];
    unpack_bf16x8(v, f);
    bf16x8_mag_keys(v, k);
  }
}

template <bool F32>
__global__ void __launch_bounds__(kTkThreads, F32 ? 3 : 6) topk_rows_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ up, int64_t M, int K, int64_t ldx, int keep,
    float eps, int8_t* __restrict__ codes, float* __restrict__ scale, uint32_t* __restrict__ mask) {
  extern __shared__ __align__(16) uint8_t tk_dyn[];
  TkShared<F32>& sm = *reinterpret_cast<TkShared<F32>*>(tk_dyn);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int wig = tid >> 5;
  const int nchunk = K >> 3;                       // 16-byte bf16 words per input row
  const int row_words = nchunk;
  const int stage_words = F32 ? 2 * row_words : row_words;
  uint4* stages = reinterpret_cast<uint4*>(tk_dyn + sizeof(TkShared<F32>));
  // bf16 rows: thread t owns the contiguous chunks [q_begin, q_end), a run of the
  // row in index order, so a tie's rank is one scan over threads.  fp32 rows
  // (six or more chunks per thread at the FFN width) stride their chunks over
  // the threads instead, which keeps the 16-byte shared-memory accesses free of
  // bank conflicts; their rare tie ranks come from a scan in chunk order.
  const int slots = (nchunk + kTkThreads - 1) / kTkThreads;
  const int q_begin = F32 ? tid : min(tid * slots, nchunk);
  const int q_end = F32 ? nchunk : min(q_begin + slots, nchunk);
  constexpr int q_step = F32 ? kTkThreads : 1;
  const int mwords = (K + 31) >> 5;
  constexpr int kCntWords = F32 ? 2048 : 4096;
  const int col = lane & 15;
  uint8_t* maskb = reinterpret_cast<uint8_t*>(sm.maskw);

  auto prefetch = [&](int64_t r, int buf) {
    if (r < M) {
      uint4* dst = stages + buf * stage_words;
      const uint16_t* src = x + r * ldx;
      for (int i = tid; i < row_words; i += kTkThreads) cp_async_16(dst + i, src + static_cast<int64_t>(i) * 8);
      if constexpr (F32) {
        const uint16_t* usrc = up + r * ldx;
        for (int i = tid; i < row_words; i += kTkThreads)
          cp_async_16(dst + row_words + i, usrc + static_cast<int64_t>(i) * 8);
      }
    }
    cp_async_commit();
  };
  auto zero_counters = [&]() {
    for (int i = tid; i < kCntWords / 4; i += kTkThreads) reinterpret_cast<uint4*>(sm.cnt)[i] = make_uint4(0, 0, 0, 0);
  };

  zero_counters();
  pdl_wait();
  pdl_trigger();
  int64_t row = blockIdx.x;
  prefetch(row, 0);
  int buf = 0;
  for (; row < M; row += gridDim.x, buf ^= kTkStages<F32> - 1) {
    if constexpr (kTkStages<F32> == 2) {
      prefetch(row + gridDim.x, buf ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    uint4* st = stages + buf * stage_words;

    // ---- sweep 1: max key; bf16 counts its first digit, fp32 writes h and counts nonzeros ----
    uint32_t mk = 0, nz = 0;
    for (int q = q_begin; q < q_end; q += q_step) {
      if constexpr (F32) {
        const uint4 gv = st[q], uv = st[row_words + q];
        float g[8], u[8];
        unpack_bf16x8(gv, g);
        unpack_bf16x8(uv, u);
        uint32_t hb[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float rg = fmaxf(g[e], 0.f);
          hb[e] = __float_as_uint(__fmul_rn(u[e], __fmul_rn(rg, rg)));
          const uint32_t key = hb[e] & 0x7FFFFFFFu;
          mk = max(mk, key);
          nz += key != 0u ? 1u : 0u;
        }
        st[q] = make_uint4(hb[0], hb[1], hb[2], hb[3]);
        st[row_words + q] = make_uint4(hb[4], hb[5], hb[6], hb[7]);
      } else {
        const uint4 v = st[q];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t klo = w[i] & 0x7FFFu, khi = (w[i] >> 16) & 0x7FFFu;
          mk = max(mk, max(klo, khi));
          tk_count<false>(sm.cnt, klo >> 7, col, 1u);
          tk_count<false>(sm.cnt, khi >> 7, col, 1u);
        }
      }
    }
    mk = __reduce_max_sync(0xFFFFFFFFu, mk);
    nz = __reduce_add_sync(0xFFFFFFFFu, nz);
    if (lane == 0) {
      sm.red[wig][0] = mk;
      sm.red[wig][1] = nz;
    }
    __syncthreads();
    mk = 0;
    nz = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      mk = max(mk, sm.red[w][0]);
      nz += sm.red[w][1];
    }

    // ---- threshold key `thr`; the first `take` (index order) of its ties survive ----
    uint32_t thr = 0, take = 0, tie_total = 0;
    const bool all_kept = keep >= K;
    bool counted = !F32;                         // counters hold this row's first digit
    if (all_kept) {
      // every element survives
    } else if (F32 && nz <= static_cast<uint32_t>(keep)) {
      take = static_cast<uint32_t>(keep) - nz;
      tie_total = static_cast<uint32_t>(K) - nz;
    } else {
      uint32_t prefix = 0, fixed = 0, r = static_cast<uint32_t>(keep);
      constexpr int kPasses = F32 ? 4 : 2;
      bool listed = false;
#pragma unroll 1
      for (int pass = 0; pass < kPasses; ++pass) {
        const int shift = F32 ? (pass == 3 ? 0 : 23 - 8 * pass) : (pass == 0 ? 7 : 0);
        const uint32_t dmask = shift == 0 ? 0x7Fu : 0xFFu;
        if (!listed) {
          if (!counted) {
            // the candidates (keys with the digits fixed so far) count 1, the
            // others 0: one branch-free atomic per value
            for (int q = q_begin; q < q_end; q += q_step) {
              uint32_t k[8];
              float f[8];
              tk_keys<F32>(st, q, row_words, k, f);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                tk_count<F32>(sm.cnt, (k[e] >> shift) & dmask, col, (k[e] & fixed) == prefix ? 1u : 0u);
            }
            __syncthreads();
          }
          sm.tot[tid] = tk_bin_total<F32>(sm.cnt, static_cast<uint32_t>(tid), lane);
          __syncthreads();
          // warp 0 picks the digit while the others clear the counters
          if (wig == 0) {
            uint32_t t[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) t[i] = sm.tot[8 * lane + i];
            tk_select(t, r, lane, sm.sel);
          } else {
            for (int i = tid - 32; i < kCntWords / 4; i += kTkThreads - 32)
              reinterpret_cast<uint4*>(sm.cnt)[i] = make_uint4(0, 0, 0, 0);
          }
          counted = false;
        } else {
          // candidates in the list: a shared histogram
          uint32_t* h = sm.hist[pass & 1];
          const int n = static_cast<int>(sm.list_n);
          for (int i = tid; i < n; i += kTkThreads) {
            const uint32_t key = sm.list[i];
            if ((key & fixed) == prefix) atomicAdd(&h[(key >> shift) & dmask], 1u);
          }
          __syncthreads();
          if (wig == 0) {
            uint32_t t[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) t[i] = h[8 * lane + i];
            tk_select(t, r, lane, sm.sel);
          } else {
            // the other histogram (last used a pass ago) is cleared for the next pass
            uint32_t* h2 = sm.hist[(pass + 1) & 1];
            for (int i = tid - 32; i < 256; i += kTkThreads - 32) h2[i] = 0;
          }
        }
        __syncthreads();
        r -= sm.sel[1];
        tie_total = sm.sel[2];
        prefix |= sm.sel[0] << shift;
        fixed |= dmask << shift;
        if (F32 && !listed && pass < kPasses - 1 && tie_total <= static_cast<uint32_t>(kTkListCap)) {
          // few candidates left (ReLU^2 rows usually cut among their smallest
          // nonzero values, one exponent bucket): they go to a list, and the
          // remaining digits are counted over the list only
          if (tid == 0) sm.list_n = 0;
          for (int i = tid; i < 512; i += kTkThreads) (&sm.hist[0][0])[i] = 0;
          __syncthreads();
          for (int q = q_begin; q < q_end; q += q_step) {
            uint32_t k[8];
            float f[8];
            tk_keys<F32>(st, q, row_words, k, f);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if ((k[e] & fixed) == prefix) sm.list[atomicAdd(&sm.list_n, 1u)] = k[e];
          }
          __syncthreads();
          listed = true;
        }
      }
      thr = prefix;
      take = r;
    }
    if (counted) {
      // a bf16 row that needed no selection: its first-digit counts are discarded
      __syncthreads();
      zero_counters();
    }
    // Ranks among the ties are needed only when some are dropped -- and not when
    // the tied key is 0 without a mask: a kept zero and a dropped one both get code 0.
    const bool partial = !all_kept && take < tie_total && (thr != 0u || mask != nullptr);

    // ---- ties before this thread's values (bf16: before its run) ----
    uint32_t before = 0;
    auto block_exclusive_scan = [&](uint32_t n) {
      uint32_t inc = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, inc, o);
        if (lane >= o) inc += v;
      }
      if (lane == 31) sm.scan[wig] = inc;
      __syncthreads();
      uint32_t wb = 0;
#pragma unroll
      for (int w = 0; w < 8; ++w) wb += w < wig ? sm.scan[w] : 0u;
      return wb + inc - n;
    };
    if (partial) {
      if constexpr (F32) {
        // ties per chunk, an exclusive scan in chunk (= index) order, read back per chunk
        for (int q = q_begin; q < q_end; q += q_step) {
          uint32_t k[8];
          float f[8];
          tk_keys<F32>(st, q, row_words, k, f);
          uint32_t n = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) n += k[e] == thr ? 1u : 0u;
          sm.tiec[q] = static_cast<uint16_t>(n);
        }
        __syncthreads();
        const int c0 = min(tid * slots, nchunk), c1 = min(c0 + slots, nchunk);
        uint32_t n = 0;
        for (int c = c0; c < c1; ++c) n += sm.tiec[c];
        uint32_t run = block_exclusive_scan(n);
        for (int c = c0; c < c1; ++c) {
          const uint32_t t = sm.tiec[c];
          sm.tiec[c] = static_cast<uint16_t>(run);   // ties before chunk c (< 2^16: K <= 16384)
          run += t;
        }
        __syncthreads();
      } else {
        uint32_t n = 0;
        for (int q = q_begin; q < q_end; q += q_step) {
          uint32_t k[8];
          float f[8];
          tk_keys<F32>(st, q, row_words, k, f);
#pragma unroll
          for (int e = 0; e < 8; ++e) n += k[e] == thr ? 1u : 0u;
        }
        before = block_exclusive_scan(n);
      }
    }

    // ---- codes and mask ----
    const float gamma = F32 ? __uint_as_float(mk) : __uint_as_float(mk << 16);
    const float denom = __fadd_rn(gamma, eps);
    const float mult = denom > 0.f ? __fdiv_rn(127.f, denom) : 0.f;
    if (tid == 0) scale[row] = __fdiv_rn(gamma, 127.f);
    for (int q = q_begin; q < q_end; q += q_step) {
      uint32_t k[8];
      float f[8];
      tk_keys<F32>(st, q, row_words, k, f);
      uint32_t bits = 0;
      if (!partial) {
#pragma unroll
        for (int e = 0; e < 8; ++e) bits |= (k[e] >= thr ? 1u : 0u) << e;
      } else {
        if constexpr (F32) before = sm.tiec[q];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t eq = k[e] == thr ? 1u : 0u;
          const uint32_t kp = (k[e] > thr ? 1u : 0u) | (eq & (before < take ? 1u : 0u));
          before += eq;
          bits |= kp << e;
        }
      }
      uint32_t cb[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) cb[e] = tk_code_bits(f[e], mult);
      reinterpret_cast<uint2*>(codes + row * static_cast<int64_t>(K))[q] = tk_pack_codes(cb, bits);
      if (mask != nullptr) maskb[q] = static_cast<uint8_t>(bits);
    }
    if (mask != nullptr) {
      __syncthreads();
      for (int w = tid; w < mwords; w += kTkThreads) {
        uint32_t v = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b)
          if (4 * w + b < nchunk) v |= static_cast<uint32_t>(maskb[4 * w + b]) << (8 * b);
        mask[row * mwords + w] = v;
      }
    }
    __syncthreads();   // the stage and the shared state are reused
    if constexpr (kTkStages<F32> == 1) prefetch(row + gridDim.x, 0);
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

}  // namespace bl
