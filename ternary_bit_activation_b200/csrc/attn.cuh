// Low-bit attention: 4-bit queries over a 3- or 4-bit key/value cache
// (BitNet a4.8, §3.4 "Low-Bit KV Cache Quantization": post-RoPE Q, K and V
// quantized by absmax to unsigned integers; Table 3's "4-bit Q, 3-bit KV" and
// "4-bit QKV" rows).  Reading: softmax attention over the dequantized codes,
//   s_t = softmax_scale * <(q - 8) q_scale, (k_t - 2^(b-1)) k_scale_t>,
//   o = sum_t softmax(s)_t (v_t - 2^(b-1)) v_scale_t,
// the BOS position of a 3-bit cache at 4 bits; the M queries are the cache's
// last M positions (query m at T - M + m, attending positions 0 .. T - M + m).
//
// Split over positions and heads (decode reads every K and V code once, so the
// grid spreads the cache over all SMs):
//  * attn_partial_kernel: CTA (chunk, head group, query group) takes a
//    contiguous range of positions for HG heads.  Blocks of 512/HG positions
//    arrive in shared memory as four 2-D TMA tiles (K and V codes, K and V
//    scales), two blocks in flight, each completing on an mbarrier whose wait
//    is bounded.  One thread per
//    (position, head) forms the exact integer <q, k> with dp4a straight from the
//    packed codes (3-bit fields masked in place, one field per byte lane, the
//    lane's shift folded into the query's weight bytes); then one thread per
//    (query, head, 32-value segment) and position phase keeps an online softmax
//    and 32 fp32 sums of the weights times the V codes.  A V code becomes a
//    float without a conversion: the field, masked where it lies in its word (a
//    word's high fields after one shared shift), is the mantissa of a subnormal
//    float u * 2^(o - 149); the weights carry a 2^64 factor (taken into the
//    exponent: 2^(s - m + 64)) so the products stay normal, and the powers of
//    two come off once at the end.  Pairs of sums use
//    the packed fp32x2 FMA.
//  * attn_combine_kernel: per (query, head), the chunks' partial results are
//    merged in the log-sum-exp way, the BOS position of a 3-bit cache is added
//    from its 4-bit codes, and the output is rounded to bf16.
#pragma once

#include <utility>

#include "common.cuh"

namespace bl {

constexpr int kAttnThreads = 256;     // threads per CTA (two (position, head) pairs of a block each)
constexpr int kAttnMaxGroup = 8;      // queries per CTA
constexpr int kAttnMaxChunks = 512;   // position chunks per (query group, head group)
constexpr int kAttnAcc = 34;          // per V thread: 32 sums, the weight sum, the probability sum
constexpr int kAttnWScale = 64;       // the weights' 2^64 factor
// lanes 0-3 of a word hold the 3-bit fields at bits 0-2, 9-11, 18-20, 27-29
constexpr uint32_t kAttn3Mask = 0x381C0E07u;

template <int D, int BITS>
struct AttnShape {
  static constexpr int kSeg = D / 32;                      // 32-code segments per vector
  static constexpr int kSegWords = BITS;                   // 3 or 4 words per segment
  static constexpr int kVecWords = kSeg * kSegWords;       // words per (position, head) vector
  static constexpr int kVecBytes = 4 * kVecWords;
  static constexpr int kWordsPerSeg = BITS == 3 ? 9 : 8;   // query weight words per segment
  static constexpr int kQWords = kSeg * kWordsPerSeg;
  static constexpr int kDotScale = BITS == 3 ? 8 : 1;      // the dp4a sums give kDotScale * <q, u>
  static constexpr int kOffset = 1 << (BITS - 1);          // stored u = c + kOffset
};

struct AttnParams {
  const uint8_t* q;    // [M x H x D/2] 4-bit codes (c + 8), nibble layout
  const float* qs;     // [M x H]
  const uint8_t* k;    // [T x H x D*BITS/8]
  const float* ks;     // [T x H]
  const uint8_t* v;
  const float* vs;
  const uint8_t* kbos; // [H x D/2] (3-bit caches with a BOS position)
  const uint8_t* vbos;
  int M, T, H, bos;    // bos = -1: none (always -1 for 4-bit caches)
  float coef;          // softmax_scale * log2(e): scores are kept in base-2 units
  int group;           // queries per CTA
  int chunk;           // positions per CTA (a multiple of the block size)
  int nchunks;
  float* part;         // [nchunks x M x H x (D + 4)]: max, probability sum, 0, 0, D sums
  uint16_t* out;       // [M x ldo] bf16, element h*D + d of row m
  int64_t ldo;
};

// 4-bit query code d of a (query, head) row, as a signed value c = code - 8
template <int D>
__device__ __forceinline__ int attn_q_code(const uint8_t* q, int row, int d) {
  const uint32_t b = q[static_cast<int64_t>(row) * (D / 2) + (d >> 1)];
  return static_cast<int>((d & 1) ? (b >> 4) : (b & 15u)) - 8;
}

// The query's dp4a weight word `w` of a (query, head) row.
// 3-bit: a segment's 32 codes are 96 bits; words x = (bits from base 0, 36, 72)
// shifted by 0, 3 and 6 and masked with kAttn3Mask hold codes 12W + S + 3l in
// lane l, scaled by 2^l; the weight byte q * 2^(3-l) makes every product 8 q u.
// 4-bit: even and odd nibbles of each word, weight q.
template <int D, int BITS>
__device__ __forceinline__ uint32_t attn_q_word(const uint8_t* q, int row, int w) {
  using S = AttnShape<D, BITS>;
  const int seg = w / S::kWordsPerSeg, i = w % S::kWordsPerSeg;
  uint32_t word = 0;
#pragma unroll
  for (int l = 0; l < 4; ++l) {
    int j, shift;
    if constexpr (BITS == 3) {
      j = 12 * (i / 3) + (i % 3) + 3 * l;
      shift = 3 - l;
    } else {
      j = 8 * (i >> 1) + 2 * l + (i & 1);
      shift = 0;
    }
    int byte = 0;
    if (j < 32) byte = attn_q_code<D>(q, row, 32 * seg + j) * (1 << shift);
    word |= (static_cast<uint32_t>(byte) & 0xFFu) << (8 * l);
  }
  return word;
}

// kDotScale * <q, u> over one (position, head) vector; kw: its code words,
// qw(i): the query's weight word i
template <int D, int BITS, typename QW>
__device__ __forceinline__ int attn_dot(const uint32_t (&kw)[AttnShape<D, BITS>::kVecWords], QW qw) {
  using S = AttnShape<D, BITS>;
  int part[S::kSeg];   // one dependency chain per segment
#pragma unroll
  for (int s = 0; s < S::kSeg; ++s) {
    const int b = s * S::kWordsPerSeg;
    int acc = 0;
    if constexpr (BITS == 3) {
      const uint32_t w0 = kw[3 * s], w1 = kw[3 * s + 1], w2 = kw[3 * s + 2];
      acc = __dp4a(static_cast<int>(w0 & kAttn3Mask), qw(b + 0), acc);
      acc = __dp4a(static_cast<int>(__funnelshift_r(w0, w1, 3) & kAttn3Mask), qw(b + 1), acc);
      acc = __dp4a(static_cast<int>(__funnelshift_r(w0, w1, 6) & kAttn3Mask), qw(b + 2), acc);
      acc = __dp4a(static_cast<int>(__funnelshift_r(w1, w2, 4) & kAttn3Mask), qw(b + 3), acc);
      acc = __dp4a(static_cast<int>(__funnelshift_r(w1, w2, 7) & kAttn3Mask), qw(b + 4), acc);
      acc = __dp4a(static_cast<int>(__funnelshift_r(w1, w2, 10) & kAttn3Mask), qw(b + 5), acc);
      acc = __dp4a(static_cast<int>((w2 >> 8) & kAttn3Mask), qw(b + 6), acc);
      acc = __dp4a(static_cast<int>((w2 >> 11) & kAttn3Mask), qw(b + 7), acc);
      acc = __dp4a(static_cast<int>((w2 >> 14) & kAttn3Mask), qw(b + 8), acc);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t w = kw[4 * s + i];
        acc = __dp4a(static_cast<int>(w & 0x0F0F0F0Fu), qw(b + 2 * i), acc);
        acc = __dp4a(static_cast<int>((w >> 4) & 0x0F0F0F0Fu), qw(b + 2 * i + 1), acc);
      }
    }
    part[s] = acc;
  }
  int acc = 0;
#pragma unroll
  for (int s = 0; s < S::kSeg; ++s) acc += part[s];
  return acc;
}

// V code J of a 32-code segment: where its field lies after the word's
// preparation.  Fields that end at bit 22 or below stay in place; a word's
// higher fields are read from the word shifted right by 11 (one shift shared by
// them); a field that crosses into the next word is read from a funnel shift by
// 16.  kOff is the field's final bit offset (the field ends at bit 22 or below,
// so the masked word is a subnormal float of value u * 2^(kOff - 149)).
template <int BITS, int J>
struct AttnVField {
  static constexpr int kBit = BITS * J, kWord = kBit / 32, kAt = kBit % 32;
  static constexpr int kKind = kAt + BITS <= 23 ? 0 : (kAt + BITS <= 32 ? 1 : 2);   // in place, shifted, crossing
  static constexpr int kOff = kKind == 0 ? kAt : (kKind == 1 ? kAt - 11 : kAt - 16);
  static constexpr uint32_t kMask = ((1u << BITS) - 1u) << kOff;
};

template <int BITS, int J>
__device__ __forceinline__ float attn_v_code(const uint32_t (&w)[BITS], const uint32_t (&hi)[BITS],
                                             const uint32_t (&cross)[BITS]) {
  using F = AttnVField<BITS, J>;
  if constexpr (F::kKind == 0)
    return __uint_as_float(w[F::kWord] & F::kMask);
  else if constexpr (F::kKind == 1)
    return __uint_as_float(hi[F::kWord] & F::kMask);
  else
    return __uint_as_float(cross[F::kWord] & F::kMask);
}

// acc[i] += wt * (code 2i, code 2i+1) over the segment's 32 codes
template <int BITS, int... I>
__device__ __forceinline__ void attn_v_acc(float2 (&acc)[16], const uint32_t (&w)[BITS], float wt,
                                           std::integer_sequence<int, I...>) {
  uint32_t hi[BITS], cross[BITS];
#pragma unroll
  for (int i = 0; i < BITS; ++i) {
    hi[i] = w[i] >> 11;
    cross[i] = __funnelshift_r(w[i], w[i + 1 < BITS ? i + 1 : i], 16);   // the last word's is never read
  }
  const float2 ww = make_float2(wt, wt);
  ((acc[I] = __ffma2_rn(make_float2(attn_v_code<BITS, 2 * I>(w, hi, cross),
                                    attn_v_code<BITS, 2 * I + 1>(w, hi, cross)),
                        ww, acc[I])),
   ...);
}

// code J's power of two: sum_t w_t u_t = acc_J * 2^(149 - kAttnWScale - kOff)
template <int BITS, int... J>
__device__ __forceinline__ void attn_v_scales(float (&sc)[32], std::integer_sequence<int, J...>) {
  ((sc[J] = __uint_as_float(static_cast<uint32_t>(127 + 149 - kAttnWScale - AttnVField<BITS, J>::kOff) << 23)),
   ...);
}

// Shared-memory layout of attn_partial_kernel for `group` queries (bytes from a
// 128-byte aligned base): kStages stages of [K codes | V codes | K scales | V
// scales] of a block (the TMA tiles, each a multiple of 128 bytes); the
// queries' codes, weight words ([g][word][head]), offsets and coefficients; the
// block's scores ([g][pair]); the per-warp maxima ([g][warp][head]); one
// mbarrier per stage.  The position phases' final reduction reuses the stage
// area.
template <int D, int BITS, int HG>
struct AttnSmem {
  static constexpr int kPairs = 2 * kAttnThreads;   // (position, head) pairs per block: two a thread
  static constexpr int kPos = kPairs / HG;          // positions per block
  static constexpr int kStages = 2;
  static constexpr size_t kCodes = static_cast<size_t>(kPairs) * AttnShape<D, BITS>::kVecBytes;
  static constexpr size_t kScales = static_cast<size_t>(kPairs) * 4;
  static constexpr size_t kStage = 2 * kCodes + 2 * kScales;
  size_t qc, qw, qoff, qcoef, scores, wmax, bars, total;
  __host__ __device__ explicit AttnSmem(int group) {
    using S = AttnShape<D, BITS>;
    auto up = [](size_t x) { return (x + 15) & ~size_t{15}; };
    const size_t g = static_cast<size_t>(group);
    const size_t red = static_cast<size_t>(kAttnThreads) * kAttnAcc * 4;
    qc = kStages * kStage > red ? kStages * kStage : red;
    qw = qc + up(g * HG * (D / 2));
    qoff = qw + up(g * S::kQWords * HG * 4);
    qcoef = qoff + up(g * HG * 4);
    scores = qcoef + up(g * HG * 4);
    wmax = scores + up(g * kPairs * 4);
    bars = wmax + up(g * (kAttnThreads / 32) * HG * 4);
    total = bars + kStages * 8 + 128;   // + the base's alignment slack
  }
};

// 2^x for x <= 64 (the hardware base-2 exponential; -inf gives 0)
__device__ __forceinline__ float attn_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// one position's V segment words from shared memory
template <int BITS>
__device__ __forceinline__ void attn_seg_words(const uint8_t* src, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 4) {
    const uint4 x = *reinterpret_cast<const uint4*>(src);
    w[0] = x.x;
    w[1] = x.y;
    w[2] = x.z;
    w[3] = x.w;
  } else {
    const uint32_t* s32 = reinterpret_cast<const uint32_t*>(src);
    w[0] = s32[0];
    w[1] = s32[1];
    w[2] = s32[2];
  }
}

// ONE: a single query per CTA (then the position phases are a compile-time count
// and the value loop is unrolled with constant offsets)
template <int D, int BITS, int HG, bool ONE>
__global__ void __launch_bounds__(kAttnThreads, 2)
    attn_partial_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmKs, const __grid_constant__ CUtensorMap tmVs,
                        const AttnParams p) {
  using S = AttnShape<D, BITS>;
  using L = AttnSmem<D, BITS, HG>;
  constexpr int VB = S::kVecBytes, SEGB = 4 * BITS;
  constexpr int P = L::kPos;
  constexpr int NPAIR = L::kPairs;
  constexpr int NS = L::kStages;
  constexpr int NWARP = kAttnThreads / 32;
  static_assert(HG == 4 || HG == 8, "head groups of 4 or 8");
  extern __shared__ uint8_t attn_smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(attn_smem_raw) + 127) & ~uintptr_t{127});
  const int H = p.H;
  const int hg0 = blockIdx.y * HG;
  const int g0 = blockIdx.z * p.group;
  const int G = ONE ? 1 : min(p.group, p.M - g0);   // queries of this CTA
  const L lay(p.group);
  uint8_t* qcs = sm + lay.qc;                                     // [G][HG][D/2]
  int* qw = reinterpret_cast<int*>(sm + lay.qw);                  // [G][kQWords][HG]
  int* qoff = reinterpret_cast<int*>(sm + lay.qoff);              // [G][HG]
  float* qcoef = reinterpret_cast<float*>(sm + lay.qcoef);        // [G][HG]
  float* scores = reinterpret_cast<float*>(sm + lay.scores);      // [G][NPAIR], base-2 units
  float* wmax = reinterpret_cast<float*>(sm + lay.wmax);          // [G][NWARP][HG]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + lay.bars);    // one per stage
  float* red = reinterpret_cast<float*>(sm);                      // after the last block

  const int c = blockIdx.x;
  const int t0 = c * p.chunk;
  const int t1 = min(p.T, t0 + p.chunk);
  const int nblocks = (t1 - t0 + P - 1) / P;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&bars[i], 1);
    fence_mbarrier_init();
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmKs);
    prefetch_tmap(&tmVs);
  }
  __syncthreads();

  // block b of the chunk: four TMA tiles of P positions x the head group (rows
  // past T read as zeros; a chunk is whole blocks, so only the last one can
  // reach past its end), completing on the stage's mbarrier
  auto issue = [&](int b) {
    if (b < nblocks) {
      uint8_t* st = sm + (b % NS) * L::kStage;
      uint64_t* bar = &bars[b % NS];
      const int y = t0 + b * P;
      mbar_arrive_expect_tx(bar, static_cast<uint32_t>(L::kStage));
      tma_load_2d(&tmK, bar, st, hg0 * VB / 8, y);
      tma_load_2d(&tmV, bar, st + L::kCodes, hg0 * VB / 8, y);
      tma_load_2d(&tmKs, bar, st + 2 * L::kCodes, hg0 / 2, y);
      tma_load_2d(&tmVs, bar, st + 2 * L::kCodes + L::kScales, hg0 / 2, y);
    }
  };

  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0)
    for (int b = 0; b < NS; ++b) issue(b);
  // the queries' codes for this head group (G contiguous pieces)
  constexpr int QCH = HG * (D / 2) / 16;
  for (int i = threadIdx.x; i < G * QCH; i += kAttnThreads) {
    const int g = i / QCH, r = i - g * QCH;
    *reinterpret_cast<uint4*>(qcs + g * (HG * (D / 2)) + 16 * r) =
        ld_dep_v4(p.q + (static_cast<int64_t>(g0 + g) * H + hg0) * (D / 2) + 16 * r);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * S::kQWords * HG; i += kAttnThreads) {
    const int h = i % HG, gw = i / HG;
    const int g = gw / S::kQWords, w = gw - g * S::kQWords;
    qw[i] = static_cast<int>(attn_q_word<D, BITS>(qcs, g * HG + h, w));
  }
  // each (query, head)'s code sum: one warp per row, a word of eight codes per lane
  for (int gh = threadIdx.x >> 5; gh < G * HG; gh += NWARP) {
    const int lane = threadIdx.x & 31;
    int sum = 0;
    if (lane < D / 8) {
      const uint32_t w = reinterpret_cast<const uint32_t*>(qcs + gh * (D / 2))[lane];
#pragma unroll
      for (int e = 0; e < 8; ++e) sum += static_cast<int>((w >> (4 * e)) & 15u) - 8;
    }
    sum = __reduce_add_sync(0xFFFFFFFFu, sum);
    if (lane == 0) {
      const int g = gh / HG, h = gh - g * HG;
      qoff[gh] = S::kDotScale * S::kOffset * sum;
      qcoef[gh] = ld_dep_f32(p.qs + static_cast<int64_t>(g0 + g) * H + hg0 + h) * p.coef * (1.0f / S::kDotScale);
    }
  }
  __syncthreads();

  // score thread: pairs tid and tid + 256 (positions tl_s and tl_s + P/2, head h_s);
  // query 0's weights in registers
  const int h_s = threadIdx.x % HG, tl_s = threadIdx.x / HG;
  int qreg[S::kQWords];
#pragma unroll
  for (int i = 0; i < S::kQWords; ++i) qreg[i] = qw[i * HG + h_s];
  // value threads: one per (query, head, segment) slot, R position phases
  const int slots = G * HG * S::kSeg;
  const int R = kAttnThreads / slots;
  const int slot = threadIdx.x % slots, r = threadIdx.x / slots;
  const bool vthread = r < R;
  const int seg = slot % S::kSeg, gh_v = slot / S::kSeg;
  const int h_v = gh_v % HG, g_v = gh_v / HG;

  float2 acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = make_float2(0.f, 0.f);
  // wsum and psum carry the 2^64 factor of the weights (exp2(s - m + 64) = p * 2^64)
  float wsum = 0.f, psum = 0.f, mrun = -INFINITY;

  bool aborted = false;
  for (int b = 0; b < nblocks; ++b) {
    const int b0 = t0 + b * P;
    const int nb = min(P, t1 - b0);
    const uint8_t* st = sm + (b % NS) * L::kStage;
    const uint8_t* kst = st;
    const uint8_t* vst = st + L::kCodes;
    const float* kss = reinterpret_cast<const float*>(st + 2 * L::kCodes);
    const float* vss = kss + NPAIR;
    // each thread waits for the block itself (a wait that runs out is noted and the
    // CTA decides after the loop)
    if (!mbar_wait_bounded(&bars[b % NS], static_cast<uint32_t>((b / NS) & 1))) aborted = true;
    {
      // scores of the two pairs for every query, and each warp's maximum per head
      uint32_t kw0[S::kVecWords], kw1[S::kVecWords];
      if constexpr (S::kVecWords % 4 == 0) {
#pragma unroll
        for (int i = 0; i < S::kVecWords / 4; ++i) {
          const uint4 x0 = reinterpret_cast<const uint4*>(kst + threadIdx.x * VB)[i];
          const uint4 x1 = reinterpret_cast<const uint4*>(kst + (threadIdx.x + kAttnThreads) * VB)[i];
          kw0[4 * i] = x0.x;
          kw0[4 * i + 1] = x0.y;
          kw0[4 * i + 2] = x0.z;
          kw0[4 * i + 3] = x0.w;
          kw1[4 * i] = x1.x;
          kw1[4 * i + 1] = x1.y;
          kw1[4 * i + 2] = x1.z;
          kw1[4 * i + 3] = x1.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < S::kVecWords / 2; ++i) {
          const uint2 x0 = reinterpret_cast<const uint2*>(kst + threadIdx.x * VB)[i];
          const uint2 x1 = reinterpret_cast<const uint2*>(kst + (threadIdx.x + kAttnThreads) * VB)[i];
          kw0[2 * i] = x0.x;
          kw0[2 * i + 1] = x0.y;
          kw1[2 * i] = x1.x;
          kw1[2 * i + 1] = x1.y;
        }
      }
      const float ks0 = kss[threadIdx.x], ks1 = kss[threadIdx.x + kAttnThreads];
      const int ta = b0 + tl_s, tb = ta + P / 2;
      const bool ma = tl_s >= nb || ta == p.bos, mb_ = tl_s + P / 2 >= nb || tb == p.bos;
      for (int g = 0; g < G; ++g) {
        int d0, d1;
        if (g == 0) {
          d0 = attn_dot<D, BITS>(kw0, [&](int i) { return qreg[i]; });
          d1 = attn_dot<D, BITS>(kw1, [&](int i) { return qreg[i]; });
        } else {
          d0 = attn_dot<D, BITS>(kw0, [&](int i) { return qw[(g * S::kQWords + i) * HG + h_s]; });
          d1 = attn_dot<D, BITS>(kw1, [&](int i) { return qw[(g * S::kQWords + i) * HG + h_s]; });
        }
        const int last = p.T - p.M + g0 + g;
        const float cf = qcoef[g * HG + h_s];
        const int qo = qoff[g * HG + h_s];
        float s0 = static_cast<float>(d0 - qo) * ks0 * cf;
        float s1 = static_cast<float>(d1 - qo) * ks1 * cf;
        if (ma || ta > last) s0 = -INFINITY;
        if (mb_ || tb > last) s1 = -INFINITY;
        scores[g * NPAIR + threadIdx.x] = s0;
        scores[g * NPAIR + threadIdx.x + kAttnThreads] = s1;
        float mx = fmaxf(s0, s1);
#pragma unroll
        for (int o = HG; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        if ((threadIdx.x & 31) < HG) wmax[(g * NWARP + (threadIdx.x >> 5)) * HG + h_s] = mx;
      }
    }
    __syncthreads();
    if (vthread) {
      float bm = -INFINITY;
#pragma unroll
      for (int w = 0; w < NWARP; ++w) bm = fmaxf(bm, wmax[(g_v * NWARP + w) * HG + h_v]);
      if (bm > mrun) {   // a block with no allowed position leaves everything as it is
        const float f = exp2f(mrun - bm);
        const float2 ff = make_float2(f, f);
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[j] = __fmul2_rn(acc[j], ff);
        wsum *= f;
        psum *= f;
        mrun = bm;
      }
      if (bm != -INFINITY) {
        const float m64 = mrun - static_cast<float>(kAttnWScale);
        const float* sc = scores + g_v * NPAIR;
        if constexpr (ONE) {
          // every position phase takes P / RR positions at constant offsets; positions
          // past the block's end have score -inf (weight 0) and lie inside the stage
          constexpr int RR = kAttnThreads / (HG * S::kSeg);
          const int pv0 = r * HG + h_v;
          const uint8_t* vp = vst + pv0 * VB + seg * SEGB;
#pragma unroll
          for (int i = 0; i < P / RR; ++i) {
            constexpr int kStep = RR * HG;
            uint32_t w[BITS];
            attn_seg_words<BITS>(vp + i * kStep * VB, w);
            const float pr = attn_ex2(sc[pv0 + i * kStep] - m64);
            const float wt = pr * vss[pv0 + i * kStep];
            psum += pr;
            wsum += wt;
            attn_v_acc<BITS>(acc, w, wt, std::make_integer_sequence<int, 16>{});
          }
        } else {
#pragma unroll 2
          for (int tl = r; tl < nb; tl += R) {
            const int pv = tl * HG + h_v;
            uint32_t w[BITS];
            attn_seg_words<BITS>(vst + pv * VB + seg * SEGB, w);
            const float pr = attn_ex2(sc[pv] - m64);   // masked positions: 2^-inf = 0
            const float wt = pr * vss[pv];
            psum += pr;
            wsum += wt;
            attn_v_acc<BITS>(acc, w, wt, std::make_integer_sequence<int, 16>{});
          }
        }
      }
    }
    __syncthreads();   // the stage, the scores and the maxima are free again
    if (threadIdx.x == 0) issue(b + NS);
  }
  // one decision for the CTA: after a wait ran out, let copies still in flight land
  // before the CTA's shared memory is released, and write nothing (the status word
  // reports the timeout)
  if (__syncthreads_or(aborted ? 1 : 0)) {
    const uint64_t tw = globaltimer_ns();
    while (globaltimer_ns() - tw < 200000ull) {
    }
    return;
  }

  // sum the position phases; then sum_t w_t (u_t - offset) = acc_j * 2^(149 - 64 - off_j) - offset * S
  if (vthread && r > 0) {
    float* dst = red + ((r - 1) * slots + slot) * kAttnAcc;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      dst[2 * j] = acc[j].x;
      dst[2 * j + 1] = acc[j].y;
    }
    dst[32] = wsum;
    dst[33] = psum;
  }
  __syncthreads();
  if (vthread && r == 0) {
    for (int q = 1; q < R; ++q) {
      const float* src = red + ((q - 1) * slots + slot) * kAttnAcc;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        acc[j].x += src[2 * j];
        acc[j].y += src[2 * j + 1];
      }
      wsum += src[32];
      psum += src[33];
    }
    float sc[32];
    attn_v_scales<BITS>(sc, std::make_integer_sequence<int, 32>{});
    const float unscale = __uint_as_float(static_cast<uint32_t>(127 - kAttnWScale) << 23);
    const float base = static_cast<float>(S::kOffset) * (wsum * unscale);
    const int m = g0 + g_v;
    float* dst = p.part + ((static_cast<int64_t>(c) * p.M + m) * H + hg0 + h_v) * (D + 4);
    if (seg == 0) {
      dst[0] = mrun;
      dst[1] = psum * unscale;
      dst[2] = 0.f;
      dst[3] = 0.f;
    }
    float4* o4 = reinterpret_cast<float4*>(dst + 4 + 32 * seg);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      o4[j] = make_float4(fmaf(acc[2 * j].x, sc[4 * j], -base), fmaf(acc[2 * j].y, sc[4 * j + 1], -base),
                          fmaf(acc[2 * j + 1].x, sc[4 * j + 2], -base), fmaf(acc[2 * j + 1].y, sc[4 * j + 3], -base));
  }
}

// One CTA per (head, query, 32 channels).  Every global load is issued up front
// (one round trip): thread t reads chunk t's maximum and probability sum, and
// warp w lane l reads channel d0 + l of chunks w, w + 8, ...; the maxima are
// reduced in shared memory, each lane weights its values, and the warps' sums
// are added at the end.
template <int D, int BITS>
__global__ void __launch_bounds__(kAttnThreads) attn_combine_kernel(const AttnParams p) {
  constexpr int NWARP = kAttnThreads / 32;
  constexpr int kBatch = 16;   // values in flight per lane
  __shared__ float wts[kAttnMaxChunks];
  __shared__ float red[NWARP];
  __shared__ float osum[NWARP][32];
  const int h = blockIdx.x, m = blockIdx.y, d0 = 32 * blockIdx.z;
  const int mh = m * p.H + h;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  const int64_t stride = static_cast<int64_t>(p.M) * p.H * (D + 4);
  const float* base = p.part + static_cast<int64_t>(mh) * (D + 4);
  const float* col = base + 4 + d0 + lane;
  const int nc = p.nchunks;

  // loads first: this thread's chunk statistics and the first batch of values
  float mc[kAttnMaxChunks / kAttnThreads], lc[kAttnMaxChunks / kAttnThreads];
#pragma unroll
  for (int k = 0; k < kAttnMaxChunks / kAttnThreads; ++k) {
    const int c = threadIdx.x + k * kAttnThreads;
    mc[k] = c < nc ? base[c * stride] : -INFINITY;
    lc[k] = c < nc ? base[c * stride + 1] : 0.f;
  }
  float x[kBatch];
#pragma unroll
  for (int k = 0; k < kBatch; ++k) {
    const int c = warp + k * NWARP;
    x[k] = c < nc ? col[c * stride] : 0.f;
  }

  auto block_reduce = [&](float v, bool is_max) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float y = __shfl_xor_sync(0xFFFFFFFFu, v, o);
      v = is_max ? fmaxf(v, y) : v + y;
    }
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int i = 1; i < NWARP; ++i) r = is_max ? fmaxf(r, red[i]) : r + red[i];
    return r;
  };

  // the BOS position of a 3-bit cache, from its 4-bit codes (offset 8)
  const bool bos = p.bos >= 0 && p.bos <= p.T - p.M + m;
  float s_bos = -INFINITY;
  if (bos) {
    float prod = 0.f;
    if (threadIdx.x < D) {
      const int d = threadIdx.x;
      const int kc = static_cast<int>((p.kbos[h * (D / 2) + (d >> 1)] >> (4 * (d & 1))) & 15) - 8;
      prod = static_cast<float>(attn_q_code<D>(p.q, mh, d) * kc);
    }
    const float isum = block_reduce(prod, false);   // an exact integer
    s_bos = isum * p.ks[static_cast<int64_t>(p.bos) * p.H + h] * (p.qs[mh] * p.coef);
  }
  float mx = s_bos;
#pragma unroll
  for (int k = 0; k < kAttnMaxChunks / kAttnThreads; ++k) mx = fmaxf(mx, mc[k]);
  const float gmax = block_reduce(mx, true);
  float lsum = 0.f;
#pragma unroll
  for (int k = 0; k < kAttnMaxChunks / kAttnThreads; ++k) {
    const int c = threadIdx.x + k * kAttnThreads;
    const float w = exp2f(mc[k] - gmax);   // chunks with nothing allowed (and padding): 0
    if (c < nc) wts[c] = w;
    lsum = fmaf(w, lc[k], lsum);
  }
  float l = block_reduce(lsum, false);   // its barriers also publish wts
  float o = 0.f;
#pragma unroll
  for (int k = 0; k < kBatch; ++k) {
    const int c = warp + k * NWARP;
    if (c < nc) o = fmaf(wts[c], x[k], o);
  }
  for (int c = warp + kBatch * NWARP; c < nc; c += NWARP) o = fmaf(wts[c], col[c * stride], o);   // more than 128 chunks
  osum[warp][lane] = o;
  __syncthreads();
  if (threadIdx.x < 32) {
    const int d = d0 + threadIdx.x;
    float od = 0.f;
#pragma unroll
    for (int w = 0; w < NWARP; ++w) od += osum[w][threadIdx.x];
    if (bos) {
      const float wb = exp2f(s_bos - gmax);
      const int vc = static_cast<int>((p.vbos[h * (D / 2) + (d >> 1)] >> (4 * (d & 1))) & 15) - 8;
      od = fmaf(wb, static_cast<float>(vc) * p.vs[static_cast<int64_t>(p.bos) * p.H + h], od);
      l += wb;
    }
    p.out[static_cast<int64_t>(m) * p.ldo + h * D + d] = __bfloat16_as_ushort(__float2bfloat16_rn(__fdiv_rn(od, l)));
  }
}

}  // namespace bl
