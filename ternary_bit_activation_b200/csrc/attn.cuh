// Low-bit attention: 4-bit queries over a 3- or 4-bit key/value cache
// (BitNet a4.8, §3.4 "Low-Bit KV Cache Quantization": post-RoPE Q, K and V
// quantized by absmax to unsigned integers; Table 3's "4-bit Q, 3-bit KV" and
// "4-bit QKV" rows).  Reading: softmax attention over the dequantized codes,
//   s_t = softmax_scale * <(q - 8) q_scale, (k_t - 2^(b-1)) k_scale_t>,
//   o = sum_t softmax(s)_t (v_t - 2^(b-1)) v_scale_t,
// the BOS position of a 3-bit cache at 4 bits; the M queries are the cache's
// last M positions (query m at T - M + m, attending positions 0 .. T - M + m).
//
// Split over positions (decode reads every K and V code once, so the grid
// spreads the cache over all SMs):
//  * attn_partial_kernel: CTA (chunk, query group) takes a contiguous range of
//    positions for every head.  Per block of <= 32 positions, one thread per
//    (position, head) forms the exact integer <q, k> with dp4a straight from
//    the packed codes (3-bit fields masked in place, one field per byte lane,
//    the lane's shift folded into the query's weight bytes), then one thread
//    per (query, head, 32-value segment) keeps an online softmax and 32 fp32
//    sums of the weights times the V codes.  A V code becomes a float by
//    OR-ing it into the mantissa of 1.0 (value 1 + u/8 or 1 + u/16); the
//    constant part is removed once at the end, from the sum of the weights.
//  * attn_combine_kernel: per (query, head), the chunks' partial results are
//    merged in the log-sum-exp way, the BOS position of a 3-bit cache is added
//    from its 4-bit codes, and the output is rounded to bf16.
#pragma once

#include <utility>

#include "common.cuh"

namespace bl {

constexpr int kAttnThreads = 256;
constexpr int kAttnMaxPos = 32;       // positions per block (scores staged in shared memory)
constexpr int kAttnMaxGroup = 8;      // queries per CTA
constexpr int kAttnMaxChunks = 512;   // position chunks
constexpr int kAttnAcc = 34;          // per V thread: 32 sums, the weight sum, the probability sum
// lanes 0-3 of a word hold the 3-bit fields at bits 0-2, 9-11, 18-20, 27-29
constexpr uint32_t kAttn3Mask = 0x381C0E07u;

template <int D, int BITS>
struct AttnShape {
  static constexpr int kSeg = D / 32;                      // 32-code segments per vector
  static constexpr int kSegWords = BITS;                   // 3 or 4 words per segment
  static constexpr int kVecWords = kSeg * kSegWords;       // words per (position, head) vector
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
  int chunk;           // positions per CTA
  int nchunks;
  int blk;             // positions per block (<= kAttnMaxPos)
  float* part;         // [nchunks x M x H x (D + 4)]: max, probability sum, 0, 0, D sums
  uint16_t* out;       // [M x ldo] bf16, element h*D + d of row m
  int64_t ldo;
};

// 4-bit query code d of (m, h), as a signed value c = code - 8
template <int D>
__device__ __forceinline__ int attn_q_code(const uint8_t* q, int mh, int d) {
  const uint32_t b = q[static_cast<int64_t>(mh) * (D / 2) + (d >> 1)];
  return static_cast<int>((d & 1) ? (b >> 4) : (b & 15u)) - 8;
}

// The query's dp4a weight word `w` of a (m, h) pair.
// 3-bit: a segment's 32 codes are 96 bits; words x = (bits from base 0, 36, 72)
// shifted by 0, 3 and 6 and masked with kAttn3Mask hold codes 12W + S + 3l in
// lane l, scaled by 2^l; the weight byte q * 2^(3-l) makes every product 8 q u.
// 4-bit: even and odd nibbles of each word, weight q.
template <int D, int BITS>
__device__ __forceinline__ uint32_t attn_q_word(const uint8_t* q, int mh, int w) {
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
    if (j < 32) byte = attn_q_code<D>(q, mh, 32 * seg + j) * (1 << shift);
    word |= (static_cast<uint32_t>(byte) & 0xFFu) << (8 * l);
  }
  return word;
}

// kDotScale * <q, u> over one (position, head) vector; kw: its code words,
// qw: the query's weight words (shared memory)
template <int D, int BITS>
__device__ __forceinline__ int attn_dot(const uint32_t (&kw)[AttnShape<D, BITS>::kVecWords], const int* qw) {
  using S = AttnShape<D, BITS>;
  int acc = 0;
#pragma unroll
  for (int s = 0; s < S::kSeg; ++s) {
    const int* wq = qw + s * S::kWordsPerSeg;
    if constexpr (BITS == 3) {
      const uint32_t w0 = kw[3 * s], w1 = kw[3 * s + 1], w2 = kw[3 * s + 2];
      acc = __dp4a(static_cast<int>(w0 & kAttn3Mask), wq[0], acc);
      acc = __dp4a(static_cast<int>(__funnelshift_r(w0, w1, 3) & kAttn3Mask), wq[1], acc);
      acc = __dp4a(static_cast<int>(__funnelshift_r(w0, w1, 6) & kAttn3Mask), wq[2], acc);
      acc = __dp4a(static_cast<int>(__funnelshift_r(w1, w2, 4) & kAttn3Mask), wq[3], acc);
      acc = __dp4a(static_cast<int>(__funnelshift_r(w1, w2, 7) & kAttn3Mask), wq[4], acc);
      acc = __dp4a(static_cast<int>(__funnelshift_r(w1, w2, 10) & kAttn3Mask), wq[5], acc);
      acc = __dp4a(static_cast<int>((w2 >> 8) & kAttn3Mask), wq[6], acc);
      acc = __dp4a(static_cast<int>((w2 >> 11) & kAttn3Mask), wq[7], acc);
      acc = __dp4a(static_cast<int>((w2 >> 14) & kAttn3Mask), wq[8], acc);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t w = kw[4 * s + i];
        acc = __dp4a(static_cast<int>(w & 0x0F0F0F0Fu), wq[2 * i], acc);
        acc = __dp4a(static_cast<int>((w >> 4) & 0x0F0F0F0Fu), wq[2 * i + 1], acc);
      }
    }
  }
  return acc;
}

// the words of one (position, head) vector (16-byte loads where the vector
// size allows, else 8-byte)
template <int D, int BITS>
__device__ __forceinline__ void attn_load_vec(const uint8_t* src, uint32_t (&w)[AttnShape<D, BITS>::kVecWords]) {
  using S = AttnShape<D, BITS>;
  if constexpr (S::kVecWords % 4 == 0) {
#pragma unroll
    for (int i = 0; i < S::kVecWords / 4; ++i) {
      const uint4 x = ld_dep_v4(src + 16 * i);
      w[4 * i] = x.x;
      w[4 * i + 1] = x.y;
      w[4 * i + 2] = x.z;
      w[4 * i + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < S::kVecWords / 2; ++i) {
      uint32_t a, b;
      asm volatile("ld.global.v2.u32 {%0,%1}, [%2];" : "=r"(a), "=r"(b) : "l"(src + 8 * i));
      w[2 * i] = a;
      w[2 * i + 1] = b;
    }
  }
}

// shift a word left (SH > 0) or right (SH < 0) by a compile-time amount
template <int SH>
__device__ __forceinline__ uint32_t attn_shift(uint32_t x) {
  if constexpr (SH >= 0)
    return x << SH;
  else
    return x >> (-SH);
}

// V code J of a segment (words w) as the bit pattern of 1 + u/8 (3-bit) or
// 1 + u/16 (4-bit): the field moved to the top of the mantissa of 1.0
template <int BITS, int J>
__device__ __forceinline__ uint32_t attn_v_bits(const uint32_t* w) {
  constexpr int b = BITS * J, wi = b / 32, off = b % 32;
  constexpr int top = BITS == 3 ? 20 : 19;
  constexpr uint32_t mask = BITS == 3 ? 0x00700000u : 0x00780000u;
  if constexpr (off + BITS <= 32)
    return (attn_shift<top - off>(w[wi]) & mask) | 0x3F800000u;
  else
    return (__funnelshift_r(w[wi], w[wi + 1], off - top) & mask) | 0x3F800000u;
}

template <int BITS, int... J>
__device__ __forceinline__ void attn_v_acc(float (&acc)[32], const uint32_t* w, float p,
                                           std::integer_sequence<int, J...>) {
  ((acc[J] = fmaf(p, __uint_as_float(attn_v_bits<BITS, J>(w)), acc[J])), ...);
}

// one segment (32 codes: 3 or 4 words) of a value vector
template <int BITS>
__device__ __forceinline__ void attn_load_seg(const uint8_t* src, uint32_t (&w)[BITS]) {
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

// Shared memory of attn_partial_kernel (bytes) for `group` queries and H heads.
template <int D, int BITS>
__host__ __device__ constexpr size_t attn_smem_bytes(int group, int H) {
  return 4u * (static_cast<size_t>(group) * H * AttnShape<D, BITS>::kQWords + 2u * group * H +
               static_cast<size_t>(group) * kAttnMaxPos * H + static_cast<size_t>(kAttnThreads) * kAttnAcc);
}

// L2 prefetch of [src, src + bytes) spread over the CTA's threads, one line each
__device__ __forceinline__ void attn_prefetch_range(const uint8_t* src, int64_t bytes) {
  const uint64_t a0 = reinterpret_cast<uint64_t>(src) & ~uint64_t{127};
  const uint64_t a1 = reinterpret_cast<uint64_t>(src) + static_cast<uint64_t>(bytes);
  for (uint64_t a = a0 + 128u * threadIdx.x; a < a1; a += 128u * kAttnThreads)
    prefetch_l2(reinterpret_cast<const void*>(a));
}

template <int D, int BITS>
__global__ void __launch_bounds__(kAttnThreads) attn_partial_kernel(const AttnParams p) {
  using S = AttnShape<D, BITS>;
  constexpr int kVecBytes = 4 * S::kVecWords;
  extern __shared__ __align__(16) unsigned char attn_smem[];
  const int H = p.H;
  const int g0 = blockIdx.y * p.group;
  const int G = min(p.group, p.M - g0);   // queries of this CTA
  const int GH = G * H;
  int* qw = reinterpret_cast<int*>(attn_smem);              // [G*H][kQWords] weight words
  int* qoff = qw + p.group * H * S::kQWords;                 // [G*H] the code offset's share of the dot
  float* qcoef = reinterpret_cast<float*>(qoff + p.group * H);   // [G*H] q_scale * coef / kDotScale
  float* scores = qcoef + p.group * H;                       // [G][kAttnMaxPos][H], base-2 units
  float* red = scores + p.group * kAttnMaxPos * H;           // [kAttnThreads][kAttnAcc]

  const int c = blockIdx.x;
  const int t0 = c * p.chunk;
  const int t1 = min(p.T, t0 + p.chunk);

  // V threads: one per (query, head, segment) slot, R position phases
  const int slots = GH * S::kSeg;
  const int R = kAttnThreads / slots;
  const int slot = threadIdx.x % slots, r = threadIdx.x / slots;
  const bool vthread = r < R;
  const int seg = slot % S::kSeg, gh_v = slot / S::kSeg;
  const int h_v = gh_v % H, g_v = gh_v / H;

  pdl_wait();
  pdl_trigger();
  {
    const int nb = min(p.blk, t1 - t0);
    attn_prefetch_range(p.k + static_cast<int64_t>(t0) * H * kVecBytes, static_cast<int64_t>(nb) * H * kVecBytes);
    attn_prefetch_range(p.v + static_cast<int64_t>(t0) * H * kVecBytes, static_cast<int64_t>(nb) * H * kVecBytes);
  }
  for (int i = threadIdx.x; i < GH * S::kQWords; i += kAttnThreads) {
    const int gh = i / S::kQWords;
    qw[i] = static_cast<int>(attn_q_word<D, BITS>(p.q, g0 * H + gh, i - gh * S::kQWords));
  }
  for (int gh = threadIdx.x; gh < GH; gh += kAttnThreads) {
    int sum = 0;
    for (int d = 0; d < D; ++d) sum += attn_q_code<D>(p.q, g0 * H + gh, d);
    qoff[gh] = S::kDotScale * S::kOffset * sum;
    qcoef[gh] = ld_dep_f32(p.qs + static_cast<int64_t>(g0) * H + gh) * p.coef * (1.0f / S::kDotScale);
  }
  __syncthreads();

  float acc[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) acc[j] = 0.f;
  float wsum = 0.f, psum = 0.f, mrun = -INFINITY;

  for (int b0 = t0; b0 < t1; b0 += p.blk) {
    const int nb = min(p.blk, t1 - b0);
    if (b0 + p.blk < t1) {   // the next block's codes into L2
      const int nb2 = min(p.blk, t1 - b0 - p.blk);
      const int64_t off = static_cast<int64_t>(b0 + p.blk) * H * kVecBytes;
      attn_prefetch_range(p.k + off, static_cast<int64_t>(nb2) * H * kVecBytes);
      attn_prefetch_range(p.v + off, static_cast<int64_t>(nb2) * H * kVecBytes);
    }
    // scores: one thread per (position, head), every query of the CTA
    for (int pr = threadIdx.x; pr < nb * H; pr += kAttnThreads) {
      const int tl = pr / H, h = pr - tl * H;
      const int t = b0 + tl;
      const int64_t vec = static_cast<int64_t>(t) * H + h;
      uint32_t kw[S::kVecWords];
      attn_load_vec<D, BITS>(p.k + vec * kVecBytes, kw);
      const float kscale = ld_dep_f32(p.ks + vec);
      const bool is_bos = t == p.bos;
      for (int g = 0; g < G; ++g) {
        const int gh = g * H + h;
        const int dot = attn_dot<D, BITS>(kw, qw + gh * S::kQWords) - qoff[gh];
        float sc = static_cast<float>(dot) * kscale * qcoef[gh];
        if (t > p.T - p.M + g0 + g || is_bos) sc = -INFINITY;
        scores[(g * kAttnMaxPos + tl) * H + h] = sc;
      }
    }
    __syncthreads();
    // values: one thread per (query, head, segment) and position phase
    if (vthread) {
      const float* sc = scores + g_v * kAttnMaxPos * H + h_v;
      float bm = -INFINITY;
      for (int tl = 0; tl < nb; ++tl) bm = fmaxf(bm, sc[tl * H]);
      if (bm > mrun) {   // a block with no allowed position leaves everything as it is
        const float f = exp2f(mrun - bm);
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] *= f;
        wsum *= f;
        psum *= f;
        mrun = bm;
      }
      if (bm != -INFINITY) {
        const uint8_t* vb = p.v + (static_cast<int64_t>(b0) * H + h_v) * kVecBytes + seg * (4 * BITS);
        const float* vsb = p.vs + static_cast<int64_t>(b0) * H + h_v;
        const int64_t step = static_cast<int64_t>(H) * kVecBytes;
        int tl = r;
        uint32_t nw[BITS];
        float nvs = 0.f;
        if (tl < nb) {
          attn_load_seg<BITS>(vb + tl * step, nw);
          nvs = vsb[static_cast<int64_t>(tl) * H];
        }
        for (; tl < nb; tl += R) {
          uint32_t w[BITS];
#pragma unroll
          for (int i = 0; i < BITS; ++i) w[i] = nw[i];
          const float vsc = nvs;
          if (tl + R < nb) {   // the next position's words are in flight while this one is summed
            attn_load_seg<BITS>(vb + (tl + R) * step, nw);
            nvs = vsb[static_cast<int64_t>(tl + R) * H];
          }
          const float pr = exp2f(sc[tl * H] - mrun);   // masked positions: exp2(-inf) = 0
          const float wt = pr * vsc;
          psum += pr;
          wsum += wt;
          attn_v_acc<BITS>(acc, w, wt, std::make_integer_sequence<int, 32>{});
        }
      }
    }
    __syncthreads();   // the next block's scores overwrite these
  }

  // sum the position phases, then o = kF * acc - kC * wsum (kF (1 + u/kF) - kC = u - offset)
  if (vthread && r > 0) {
    float* dst = red + ((r - 1) * slots + slot) * kAttnAcc;
#pragma unroll
    for (int j = 0; j < 32; ++j) dst[j] = acc[j];
    dst[32] = wsum;
    dst[33] = psum;
  }
  __syncthreads();
  if (vthread && r == 0) {
    for (int q = 1; q < R; ++q) {
      const float* src = red + ((q - 1) * slots + slot) * kAttnAcc;
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] += src[j];
      wsum += src[32];
      psum += src[33];
    }
    constexpr float kF = BITS == 3 ? 8.f : 16.f;
    constexpr float kC = BITS == 3 ? 12.f : 24.f;
    const int m = g0 + g_v;
    float* dst = p.part + ((static_cast<int64_t>(c) * p.M + m) * H + h_v) * (D + 4);
    if (seg == 0) {
      dst[0] = mrun;
      dst[1] = psum;
      dst[2] = 0.f;
      dst[3] = 0.f;
    }
    const float base = kC * wsum;
    float4* o4 = reinterpret_cast<float4*>(dst + 4 + 32 * seg);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      o4[j] = make_float4(fmaf(kF, acc[4 * j], -base), fmaf(kF, acc[4 * j + 1], -base),
                          fmaf(kF, acc[4 * j + 2], -base), fmaf(kF, acc[4 * j + 3], -base));
  }
}

template <int NW>
__device__ __forceinline__ float attn_block_max(float v, float* red) {
  v = warp_max(v);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < NW; ++i) r = fmaxf(r, red[i]);
  return r;
}

template <int NW>
__device__ __forceinline__ float attn_block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < NW; ++i) r += red[i];
  return r;
}

// One CTA per (head, query), one thread per channel d.
template <int D, int BITS>
__global__ void __launch_bounds__(D) attn_combine_kernel(const AttnParams p) {
  constexpr int NW = D / 32;
  __shared__ float wts[kAttnMaxChunks];
  __shared__ float red[NW];
  const int h = blockIdx.x, m = blockIdx.y, d = threadIdx.x;
  const int mh = m * p.H + h;
  pdl_wait();
  pdl_trigger();
  const int64_t stride = static_cast<int64_t>(p.M) * p.H * (D + 4);
  const float* base = p.part + static_cast<int64_t>(mh) * (D + 4);

  // the BOS position of a 3-bit cache, from its 4-bit codes (offset 8)
  const bool bos = p.bos >= 0 && p.bos <= p.T - p.M + m;
  float s_bos = -INFINITY, v_bos = 0.f;
  if (bos) {
    const int kc = static_cast<int>((p.kbos[h * (D / 2) + (d >> 1)] >> (4 * (d & 1))) & 15) - 8;
    const float isum = attn_block_sum<NW>(static_cast<float>(attn_q_code<D>(p.q, mh, d) * kc), red);
    const int64_t bv = static_cast<int64_t>(p.bos) * p.H + h;
    s_bos = isum * p.ks[bv] * (p.qs[mh] * p.coef);
    const int vc = static_cast<int>((p.vbos[h * (D / 2) + (d >> 1)] >> (4 * (d & 1))) & 15) - 8;
    v_bos = static_cast<float>(vc) * p.vs[bv];
  }
  float mx = s_bos;
  for (int c = d; c < p.nchunks; c += D) mx = fmaxf(mx, base[c * stride]);
  const float gmax = attn_block_max<NW>(mx, red);
  float l = 0.f;
  for (int c = d; c < p.nchunks; c += D) {
    const float w = exp2f(base[c * stride] - gmax);   // chunks with nothing allowed: 0
    wts[c] = w;
    l = fmaf(w, base[c * stride + 1], l);
  }
  l = attn_block_sum<NW>(l, red);   // its barriers also publish wts
  float o = 0.f;
  for (int c = 0; c < p.nchunks; ++c) o = fmaf(wts[c], base[c * stride + 4 + d], o);
  if (bos) {
    const float wb = exp2f(s_bos - gmax);
    o = fmaf(wb, v_bos, o);
    l += wb;
  }
  p.out[static_cast<int64_t>(m) * p.ldo + h * D + d] = __bfloat16_as_ushort(__float2bfloat16_rn(__fdiv_rn(o, l)));
}

}  // namespace bl
