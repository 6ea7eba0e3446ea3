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

namespace bl {

// ---------------------------------------------------------------------------
// Top-K + INT8 for bf16 rows of up to 4096 values: one warp per row, the row in
// registers (lane l holds the 16-byte chunks 32q + l, q < C), no shared memory
// and no block barrier.
//
// The keep-th largest magnitude key thr is found by counting probes: count(t) =
// #{|x| >= t} over the row, one packed bf16x2 comparison per two values
// (set.ge.u32.bf16x2 writes 0xFFFF per true half; the sum of those masks over a
// lane's words still tells how many low and how many high halves were true),
// summed over the warp.  count(0) = K and count(max + 1) = 0 bracket thr; the
// first probes come from a sorted sample of 32 values at the target quantile,
// the next ones interpolate the counts linearly between the bracket's ends, and
// a probe that fails to halve the bracket makes the next one a bisection, so the
// search ends (at most two probes per halving of the 15-bit key range) with
// count(thr) >= keep > count(thr + 1).  Values above thr survive; of the values
// equal to thr the first keep - count(thr + 1) in index order survive, ranked
// by a warp scan over the chunks in index order.  Values past K (a ragged last
// chunk round) are a bf16 NaN, which no comparison counts.
// ---------------------------------------------------------------------------
constexpr int kTwWarps = 4;                  // rows in flight per CTA
constexpr int kTwMaxK = 4096;                // 16 chunks of 8 values per lane

// Dynamic shared memory of topk_warp_kernel<C>: a row buffer per warp and its
// mbarrier.
template <int C>
constexpr size_t tw_smem_bytes() {
  return static_cast<size_t>(kTwWarps) * C * 32 * 16 + kTwWarps * 8;
}

// 0xFFFF in each 16-bit half where a >= b as bf16 values (a, b finite or NaN).
__device__ __forceinline__ uint32_t bf2_ge_mask(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.ge.u32.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf2_gt_mask(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.gt.u32.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf2_eq_mask(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.eq.u32.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// 1.0 in each bf16 half where a >= b, else +0 (a, b finite or NaN).
__device__ __forceinline__ uint32_t bf2_ge_one(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.ge.bf16x2.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// Per-half bf16 sum (round to nearest; exact for the small counts added here).
__device__ __forceinline__ uint32_t bf2_add(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// Per-half bf16 maximum of two non-negative values.
__device__ __forceinline__ uint32_t bf2_max(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// 1.0 in each bf16 half where a > b / a == b, else +0.
__device__ __forceinline__ uint32_t bf2_gt_one(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.gt.bf16x2.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// |a| per bf16 half (sign bits cleared; runs on the FMA pipe, not the ALU).
__device__ __forceinline__ uint32_t bf2_abs(uint32_t a) {
  uint32_t d;
  asm("abs.bf16x2 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}
// x * k - 0 in fp32 for the low (HI = false) or high bf16 halves of x and k:
// with k = 1.0 or +0 this is x converted exactly, or a zero (one FMA-pipe
// instruction for the conversion and the mask).
template <bool HI>
__device__ __forceinline__ float bf16_times_f32(uint32_t x, uint32_t k) {
  float d;
  if constexpr (HI)
    asm("{\n\t.reg .b16 xl, xh, kl, kh;\n\tmov.b32 {xl, xh}, %1;\n\tmov.b32 {kl, kh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, xh, kh, 0f80000000;\n\t}"
        : "=f"(d) : "r"(x), "r"(k));
  else
    asm("{\n\t.reg .b16 xl, xh, kl, kh;\n\tmov.b32 {xl, xh}, %1;\n\tmov.b32 {kl, kh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, xl, kl, 0f80000000;\n\t}"
        : "=f"(d) : "r"(x), "r"(k));
  return d;
}
// Four codes as bytes from the bit patterns b_i = bits(c_i + 1.5 * 2^23)
// = 0x4B400000 + c_i (|c_i| <= 127): the sum of (c_i + 128) * 256^i has no carry
// between bytes, and XOR 0x80 turns each c + 128 back into c's two's
// complement byte.  Multiply-adds, so the work stays off the ALU.
__device__ __forceinline__ uint32_t tw_pack4(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  constexpr uint32_t kBias = 0u - 0x4B3FFF80u * 0x01010101u;   // -sum_i (0x4B400000 - 128) * 256^i
  uint32_t wd = b0 + kBias;
  wd = b1 * 0x100u + wd;
  wd = b2 * 0x10000u + wd;
  wd = b3 * 0x1000000u + wd;
  return wd ^ 0x80808080u;
}

// PRMT with the selector's replicate bit: a selector nibble 8 + b yields 0xFF
// if byte b of {b:a} has its top bit set, else 0 (__byte_perm ignores that bit).
__device__ __forceinline__ uint32_t prmt_sign(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// s = the 32-bit sum of n per-half masks (each 0, 0xFFFF, 0xFFFF0000 or
// 0xFFFFFFFF), n < 2^15: the number of true halves.  With A true low halves and
// B true high halves, s = (A - B) * 2^16 - A (mod 2^32), so A = -s mod 2^16 and
// A - B is the signed high half of s + A.
__device__ __forceinline__ int tw_true_halves(uint32_t s) {
  const uint32_t a = (0u - s) & 0xFFFFu;
  const int d = static_cast<int16_t>(static_cast<uint16_t>((s + a) >> 16));
  return 2 * static_cast<int>(a) - d;
}

// 16-byte load that bypasses L1 (volatile: stays behind pdl_wait).
__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// Four bytes that are 0 or 0xFF -> four bits (byte i -> bit i).
__device__ __forceinline__ uint32_t tw_byte_bits(uint32_t m) { return ((m & 0x01010101u) * 0x01020408u) >> 24; }

template <int C>
__global__ void __launch_bounds__(32 * kTwWarps) topk_warp_kernel(
    const uint16_t* __restrict__ x, int64_t M, int K, int64_t ldx, int keep, float eps,
    int8_t* __restrict__ codes, float* __restrict__ scale, uint32_t* __restrict__ mask) {
  constexpr uint32_t kPadNaN = 0x7FC07FC0u;
  // One row buffer per warp, filled by a 1-D bulk copy.  The code pass reads the
  // signed row from it in a rolled loop (an unrolled one overflows the
  // instruction cache); the probes read the |x| words from registers.  The
  // next row is prefetched into L2 when a row starts and copied in as soon as
  // the code pass is done: a row keeps a warp busy far longer than a copy
  // takes, and one buffer per warp leaves room for more warps per SM.
  extern __shared__ __align__(128) uint4 tw_dyn[];
  uint4 (*rowbuf)[C * 32] = reinterpret_cast<uint4 (*)[C * 32]>(tw_dyn);
  uint64_t* rowbar = reinterpret_cast<uint64_t*>(tw_dyn + kTwWarps * C * 32);
  const int lane = threadIdx.x & 31;
  const int wig = threadIdx.x >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kTwWarps;
  const int nchunk = K >> 3;
  const int mbytes = ((K + 31) >> 5) * 4;
  const uint32_t row_bytes = static_cast<uint32_t>(2 * K);
  // the sample: word 0 of chunk round (lane % C), low half
  const int qs = lane % C;
  if (lane == 0) {
    mbar_init(&rowbar[wig], 1);
    fence_mbarrier_init();
  }
  __syncwarp();
  pdl_wait();
  pdl_trigger();
  int64_t row = static_cast<int64_t>(blockIdx.x) * kTwWarps + wig;
  if (lane == 0 && row < M) {
    mbar_arrive_expect_tx(&rowbar[wig], row_bytes);
    bulk_load_1d(rowbuf[wig], x + row * ldx, row_bytes, &rowbar[wig]);
  }
  uint32_t phase = 0;
  bool aborted = false;
  const uint4* rb = rowbuf[wig];
  for (; row < M; row += nwarps) {
    if (lane == 0 && row + nwarps < M) bulk_prefetch_l2(x + (row + nwarps) * ldx, row_bytes);
    // every lane waits for the copy; giving up is decided for the whole warp
    if (__any_sync(0xFFFFFFFFu, !mbar_wait_bounded(&rowbar[wig], phase))) {
      aborted = true;
      break;
    }
    phase ^= 1u;
    // |x| words in registers (the probes' operand), NaN past K
    uint32_t w[C][4];
#pragma unroll
    for (int q = 0; q < C; ++q) {
      uint4 v = make_uint4(kPadNaN, kPadNaN, kPadNaN, kPadNaN);
      if (32 * q + lane < nchunk) v = rb[32 * q + lane];
      w[q][0] = bf2_abs(v.x);
      w[q][1] = bf2_abs(v.y);
      w[q][2] = bf2_abs(v.z);
      w[q][3] = bf2_abs(v.w);
    }
    // row maximum of |x| (bf16 maxima of non-negative values order like the
    // 15-bit keys; NaN padding excluded) and the sample; four independent
    // partial results per lane keep the dependency chains short
    uint32_t mxp[4] = {0, 0, 0, 0}, smp = 0;
#pragma unroll
    for (int q = 0; q < C; ++q) {
      if (32 * q + lane < nchunk) {
#pragma unroll
        for (int j = 0; j < 4; ++j) mxp[j] = bf2_max(mxp[j], w[q][j]);
        if (q == qs) smp = w[q][0] & 0x7FFFu;
      }
    }
    const uint32_t mx = bf2_max(bf2_max(mxp[0], mxp[1]), bf2_max(mxp[2], mxp[3]));
    const uint32_t maxkey = __reduce_max_sync(0xFFFFFFFFu, max(mx & 0xFFFFu, mx >> 16));

    // ---- threshold: count(thr) >= keep > count(thr + 1) ----
    uint32_t lo = 0, hi = maxkey + 1;
    int clo = K, chi = 0;
    if (keep < K) {
      // sorted sample (ascending over lanes, bitonic)
#pragma unroll
      for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
          const uint32_t o = __shfl_xor_sync(0xFFFFFFFFu, smp, j);
          const bool take_min = ((lane & j) == 0) == ((lane & k) == 0);
          smp = take_min ? min(smp, o) : max(smp, o);
        }
      }
      // the target's position among 32 descending samples, and two steps either side
      const int rs = static_cast<int>(((2 * static_cast<int64_t>(keep) - 1) * 32) / (2 * static_cast<int64_t>(K)));
      const int ai = 31 - rs;
      const uint32_t t_hi = __shfl_sync(0xFFFFFFFFu, smp, min(ai + 2, 31));
      const uint32_t t_lo = __shfl_sync(0xFFFFFFFFu, smp, max(ai - 2, 0));
      // count(t) for one or two thresholds in one pass over the row: packed
      // compares give 1.0 / 0 per half, summed in bf16 on the FMA pipe in
      // independent partial sums (at most C per half and partial sum, 4C <= 64
      // per lane: exact); the counts leave the bf16 sums through fp32 (exact)
      // and the 2^23 trick
      auto bf2_count = [](uint32_t a, uint32_t b) -> uint32_t {
        const uint32_t sa = bf2_add(a, b);
        const float f = __fadd_rn(__fadd_rn(__uint_as_float(sa << 16), __uint_as_float(sa & 0xFFFF0000u)), 8388608.f);
        return static_cast<uint32_t>(__float_as_int(f) - 0x4B000000);
      };
      auto counts2 = [&](uint32_t t0, uint32_t t1, int& c0, int& c1) {
        const uint32_t u0 = t0 | (t0 << 16), u1 = t1 | (t1 << 16);
        uint32_t a[4] = {0, 0, 0, 0}, b[4] = {0, 0, 0, 0};
#pragma unroll
        for (int q = 0; q < C; ++q)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            a[j] = bf2_add(a[j], bf2_ge_one(w[q][j], u0));
            b[j] = bf2_add(b[j], bf2_ge_one(w[q][j], u1));
          }
        const uint32_t r = __reduce_add_sync(0xFFFFFFFFu, (bf2_count(a[0], a[1]) + bf2_count(a[2], a[3])) |
                                                              ((bf2_count(b[0], b[1]) + bf2_count(b[2], b[3])) << 16));
        c0 = static_cast<int>(r & 0xFFFFu);   // two 16-bit sums (K <= 4096)
        c1 = static_cast<int>(r >> 16);
      };
      auto count1 = [&](uint32_t t0) -> int {
        const uint32_t u0 = t0 | (t0 << 16);
        uint32_t a[4] = {0, 0, 0, 0};
#pragma unroll
        for (int q = 0; q < C; ++q)
#pragma unroll
          for (int j = 0; j < 4; ++j) a[j] = bf2_add(a[j], bf2_ge_one(w[q][j], u0));
        return static_cast<int>(
            __reduce_add_sync(0xFFFFFFFFu, bf2_count(a[0], a[1]) + bf2_count(a[2], a[3])));
      };
      auto update = [&](uint32_t t, int c) {
        if (t <= lo || t >= hi) return;
        if (c >= keep) {
          lo = t;
          clo = c;
        } else {
          hi = t;
          chi = c;
        }
      };
      // the sample's two guesses in one pass
      {
        int c0, c1;
        counts2(t_hi, t_lo, c0, c1);
        update(t_hi, c0);
        update(t_lo, c1);
      }
      bool bisect = false;
#pragma unroll 1
      while (hi - lo > 1) {
        if (hi - lo == 3) {
          // the last two candidates in one pass
          int c0, c1;
          const uint32_t t0 = lo + 1, t1 = lo + 2;
          counts2(t0, t1, c0, c1);
          update(t0, c0);
          update(t1, c1);
          continue;
        }
        uint32_t t;
        if (bisect) {
          t = (lo + hi) >> 1;
        } else {
          // linear interpolation of the counts (any guess inside the bracket is correct)
          const float f = __fdividef(static_cast<float>(clo) - (static_cast<float>(keep) - 0.5f),
                                     static_cast<float>(clo - chi));
          t = lo + static_cast<uint32_t>(__float2int_rn(f * static_cast<float>(hi - lo)));
          t = min(max(t, lo + 1), hi - 1);
        }
        const uint32_t before = hi - lo;
        update(t, count1(t));
        bisect = 2 * (hi - lo) > before;
      }
    }
    const uint32_t thr = lo;
    const int take = keep - chi;            // ties at thr that survive
    const bool partial = keep < K && take < clo - chi && (thr != 0u || mask != nullptr);

    // ---- codes and mask, chunk rounds in index order ----
    const float gamma = __uint_as_float(maxkey << 16);
    const float denom = __fadd_rn(gamma, eps);
    const float mult = denom > 0.f ? __fdiv_rn(127.f, denom) : 0.f;
    if (lane == 0) scale[row] = __fdiv_rn(gamma, 127.f);
    const uint32_t tt = thr | (thr << 16);
    // the code of +thr and of -thr, four times over: every surviving tie has
    // magnitude thr, so its code depends only on its sign
    const uint32_t ct = tk_code_bits(__uint_as_float(thr << 16), mult) & 0xFFu;
    const uint32_t ct_pos = ct * 0x01010101u, ct_neg = ((0u - ct) & 0xFFu) * 0x01010101u;
    int8_t* crow = codes + row * static_cast<int64_t>(K);
    uint8_t* mrow = mask != nullptr ? reinterpret_cast<uint8_t*>(mask) + row * static_cast<int64_t>(mbytes) : nullptr;
    int running = 0;                         // ties in the rounds before
#pragma unroll 2
    for (int q = 0; q < C; ++q) {
      const int c = 32 * q + lane;
      const uint4 v = rb[c];
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
      uint32_t av[4], kp[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        av[j] = bf2_abs(wv[j]);
        // 1.0 where the value survives for sure: above thr, or at thr when every tie does
        kp[j] = partial ? bf2_gt_one(av[j], tt) : bf2_ge_one(av[j], tt);
      }
      // codes of the surviving values, zeros elsewhere (x * 1 or x * 0 in one instruction)
      uint32_t cb[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        cb[2 * j] = tk_code_bits(bf16_times_f32<false>(wv[j], kp[j]), mult);
        cb[2 * j + 1] = tk_code_bits(bf16_times_f32<true>(wv[j], kp[j]), mult);
      }
      uint32_t lo4 = tw_pack4(cb[0], cb[1], cb[2], cb[3]);
      uint32_t hi4 = tw_pack4(cb[4], cb[5], cb[6], cb[7]);
      uint32_t sel_lo = 0, sel_hi = 0;
      if (partial && running < take) {
        // ties at thr, taken in index order until `take` have survived
        uint32_t eq[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) eq[j] = bf2_eq_mask(av[j], tt);
        const uint32_t tl = __byte_perm(eq[0], eq[1], 0x6420), th = __byte_perm(eq[2], eq[3], 0x6420);
        const int n = (__popc(tl) + __popc(th)) >> 3;
        if (__ballot_sync(0xFFFFFFFFu, n != 0) != 0u) {
          const int tot = static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<uint32_t>(n)));
          if (running + tot <= take) {
            sel_lo = tl;                       // every tie of this round survives
            sel_hi = th;
          } else {
            // the round where the cut falls: ranks by a scan over the lanes
            int incl = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
              if (lane >= o) incl += u;
            }
            int nt = min(max(take - (running + incl - n), 0), n);
            // the first nt tie bytes in element order
            uint64_t tb = (static_cast<uint64_t>(th) << 32) | tl;
            uint64_t sel = 0;
            for (; nt > 0; --nt) {
              const uint64_t byte = (tb & (0ull - tb)) * 0xFFull;
              sel |= byte;
              tb &= ~byte;
            }
            sel_lo = static_cast<uint32_t>(sel);
            sel_hi = static_cast<uint32_t>(sel >> 32);
          }
          running += tot;
          if ((sel_lo | sel_hi) != 0u) {
            // sign bytes (0xFF where negative) pick the tie code
            const uint32_t sg_lo = prmt_sign(wv[0], wv[1], 0xFDB9u), sg_hi = prmt_sign(wv[2], wv[3], 0xFDB9u);
            lo4 |= ((sg_lo & ct_neg) | (~sg_lo & ct_pos)) & sel_lo;
            hi4 |= ((sg_hi & ct_neg) | (~sg_hi & ct_pos)) & sel_hi;
          }
        }
      }
      if (c < nchunk) {
        *reinterpret_cast<uint2*>(crow + 8 * c) = make_uint2(lo4, hi4);
        if (mrow != nullptr) {
          // kept: the 1.0 halves (byte 1 of a half is 0x3F) and the selected ties
          const uint32_t kl = (((__byte_perm(kp[0], kp[1], 0x7531) + 0x7F7F7F7Fu) >> 7) & 0x01010101u) * 0xFFu | sel_lo;
          const uint32_t kh = (((__byte_perm(kp[2], kp[3], 0x7531) + 0x7F7F7F7Fu) >> 7) & 0x01010101u) * 0xFFu | sel_hi;
          mrow[c] = static_cast<uint8_t>(tw_byte_bits(kl) | (tw_byte_bits(kh) << 4));
        }
      } else if (mrow != nullptr && c < mbytes) {
        mrow[c] = 0;                         // bits past K
      }
    }
    __syncwarp();                            // the code pass is done with the buffer
    if (lane == 0 && row + nwarps < M) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive_expect_tx(&rowbar[wig], row_bytes);
      bulk_load_1d(rowbuf[wig], x + (row + nwarps) * ldx, row_bytes, &rowbar[wig]);
    }
  }
  if (aborted) {
    // a copy may still be in flight into this warp's buffers: let it land
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) {
    }
  }
}

}  // namespace bl
