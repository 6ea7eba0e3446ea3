// BitLinear product (BitNet a4.8, §3.4: Y = Q_x(X) . Q_w(W)^T with integer
// accumulation, then the per-token x per-tensor dequant):
//   acc[m,n] = sum_k a[m,k] * t[n,k],   y[m,n] = bf16(acc * a_scale[m] * alpha[n / group])
//
// gemm_tc_kernel   -- int8 x int8 on the 5th-generation tensor cores
//                     (tcgen05.mma kind::i8, s32 accumulators in TMEM), operands
//                     streamed by TMA into a 128B-swizzled shared-memory ring,
//                     persistent over output tiles with a double-buffered
//                     accumulator so the epilogue overlaps the next tile.
// gemm_tc2_kernel  -- the same on CTA pairs (cta_group::2), 256 x 256 tiles.
// gemm_t2tc_kernel -- 2-bit ternary weights x int8 activations for 8..256
//                     tokens (decode): weights widened to int8 in registers
//                     and stored into tensor memory as the MMA's A operand.
// gemv_t2_kernel   -- 1 to 8 tokens x 2-bit weights: offset codes c + 1
//                     isolated per byte field, dp4a against transposed
//                     activations in shared memory (long rows).
// gemv_mma_t2_kernel -- the same offset codes fed to warp-level integer MMA
//                     (16 weight rows x 8 or 16 token slots per instruction).
// gemv_stream_t2_kernel -- 1-2 tokens, the CTA's contiguous weight range
//                     streamed through shared memory by 1-D bulk copies.
// gemv_gated_t2_kernel -- the conditional Up projection (Gate rows first, Up
//                     rows only for channels with a positive gate), 1-2 tokens.
// gemm_simt_kernel -- CUDA-core kernel that reads packed operands directly
//                     (2-bit ternary weights, INT4 / E2M1 nibbles); decode of
//                     3 to 7 tokens and the packed activation formats.
#pragma once

#include "common.cuh"
#include "quant.cuh"

namespace bl {

// ---------------------------------------------------------------------------
// tcgen05 kernel
// ---------------------------------------------------------------------------
constexpr int kTcBM = 128;      // tile rows (TMEM lanes)
constexpr int kTcBN = 256;      // tile columns (TMEM columns per accumulator)
constexpr int kTcBK = 128;      // K bytes per stage = one 128-byte swizzle atom row
constexpr int kTcStages = 4;
constexpr int kTcThreads = 192; // warp 0: TMA producer, warp 1: MMA issuer, warps 2-5: epilogue
constexpr uint32_t kTcStageA = kTcBM * kTcBK;
constexpr uint32_t kTcStageB = kTcBN * kTcBK;
constexpr uint32_t kTcTmemCols = 2 * kTcBN;
constexpr int kTcGroupM = 16;   // m-blocks per rasterisation group (L2 reuse of B)
constexpr size_t kTcSmemBytes = 1024 /*align slack*/ + kTcStages * (kTcStageA + kTcStageB) + 256;

struct TcParams {
  const float* a_scale;
  const float* alpha;
  int64_t alpha_group;
  int M, N, K;
  uint16_t* y;
  int64_t ldy;
  int32_t* acc;
  int num_m_blocks, num_n_blocks, num_tiles, num_kb;
};

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4)    // start address, 16-byte units
         | (static_cast<uint64_t>(1) << 16)                 // leading offset (unused for this layout)
         | (static_cast<uint64_t>(1024 >> 4) << 32)         // stride offset between 8-row groups
         | (static_cast<uint64_t>(1) << 46)                 // descriptor version for sm_100
         | (static_cast<uint64_t>(2) << 61);                // 128-byte swizzle
}

// Instruction descriptor: s32 accumulate, signed int8 A and B, both K-major,
// N = 256, M = 128.
constexpr uint32_t kTcIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(kTcBN) >> 3) << 17) |
                              ((static_cast<uint32_t>(kTcBM) >> 4) << 24);

__device__ __forceinline__ void tc_tile_coords(int tile, int nmb, int nnb, int& mb, int& nb) {
  const int group = tile / (kTcGroupM * nnb);
  const int first_m = group * kTcGroupM;
  const int gsize = min(nmb - first_m, kTcGroupM);
  const int in = tile - group * kTcGroupM * nnb;
  mb = first_m + in % gsize;
  nb = in / gsize;
}

// Lane 0 waits (bounded) and the result is shared with the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  const int lane = threadIdx.x & 31;
  uint32_t ok = 1;
  if (lane == 0) ok = mbar_wait_bounded(bar, parity) ? 1u : 0u;
  ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
  return ok != 0;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(kTcThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kTcStages * kTcStageA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kTcStages * kTcStageB);
  uint64_t* full = bars;
  uint64_t* empty = bars + kTcStages;
  uint64_t* tfull = bars + 2 * kTcStages;
  uint64_t* tempty = bars + 2 * kTcStages + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kTcStages + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The next kernel may start once every CTA holds its tensor memory (a later
  // allocation on this SM then waits for this CTA, never the reverse) and has
  // passed its own wait (so at most one kernel runs ahead of its inputs).
  pdl_wait();
  pdl_trigger();
  bool aborted = false;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles && !aborted; tile += gridDim.x) {
        int mb, nb;
        tc_tile_coords(tile, p.num_m_blocks, p.num_n_blocks, mb, nb);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u)) {
            aborted = true;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kTcStageA + kTcStageB);
          tma_load_2d(&tmA, &full[s], sA + s * kTcStageA, kb * kTcBK, mb * kTcBM);
          tma_load_2d(&tmB, &full[s], sB + s * kTcStageB, kb * kTcBK, nb * kTcBN);
          if (++s == kTcStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (one thread) ----------------
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int local = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles && !aborted; tile += gridDim.x, ++local) {
        const int buf = local & 1;
        const uint32_t tph = (local >> 1) & 1;
        if (!mbar_wait_bounded(&tempty[buf], tph ^ 1u)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kTcBN);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(&full[s], ph)) {
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kTcStageA);
          const uint32_t b0 = smem_u32(sB + s * kTcStageB);
#pragma unroll
          for (int kk = 0; kk < kTcBK / 32; ++kk) {
            mma_i8(d_tmem, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), kTcIdesc,
                   (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit(&empty[s]);  // frees the stage once these MMAs have read it
          if (++s == kTcStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (aborted) break;
        mma_commit(&tfull[buf]);  // accumulator ready for the epilogue
      }
    }
  } else {
    // ---------------- epilogue (warps 2-5) ----------------
    const int quad = warp & 3;  // TMEM lanes [32*quad, 32*quad + 32) belong to this warp
    int local = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++local) {
      const int buf = local & 1;
      const uint32_t tph = (local >> 1) & 1;
      if (!warp_wait(&tfull[buf], tph)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      int mb, nb;
      tc_tile_coords(tile, p.num_m_blocks, p.num_n_blocks, mb, nb);
      const int row = mb * kTcBM + quad * 32 + lane;
      const bool row_ok = row < p.M;
      const float rs = row_ok ? ld_dep_f32(p.a_scale + row) : 0.f;
#pragma unroll 1
      for (int c = 0; c < kTcBN / 32; ++c) {
        uint32_t r[32];
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                               static_cast<uint32_t>(buf * kTcBN + c * 32);
        tmem_ld_32x32b_x32(taddr, r);
        tmem_wait_ld();
        const int n0 = nb * kTcBN + c * 32;
        if (!row_ok || n0 >= p.N) continue;
        const int64_t ga = n0 / p.alpha_group;
        const bool one_alpha = ((n0 + 31) / p.alpha_group) == ga;
        const float cs_uniform = __fmul_rn(rs, ld_dep_f32(p.alpha + (one_alpha ? ga : 0)));
        float yv[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float cs = one_alpha ? cs_uniform
                                     : __fmul_rn(rs, ld_dep_f32(p.alpha + min(static_cast<int64_t>(n0 + j), static_cast<int64_t>(p.N - 1)) / p.alpha_group));
          yv[j] = __fmul_rn(__int2float_rn(static_cast<int>(r[j])), cs);
        }
        const bool full_chunk = n0 + 32 <= p.N;
        if (p.y != nullptr) {
          uint16_t* yr = p.y + static_cast<int64_t>(row) * p.ldy + n0;
          if (full_chunk) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 o;
              o.x = pack_bf16x2(yv[8 * q + 0], yv[8 * q + 1]);
              o.y = pack_bf16x2(yv[8 * q + 2], yv[8 * q + 3]);
              o.z = pack_bf16x2(yv[8 * q + 4], yv[8 * q + 5]);
              o.w = pack_bf16x2(yv[8 * q + 6], yv[8 * q + 7]);
              reinterpret_cast<uint4*>(yr)[q] = o;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (n0 + j < p.N) {
                const __nv_bfloat16 b = __float2bfloat16_rn(yv[j]);
                yr[j] = *reinterpret_cast<const uint16_t*>(&b);
              }
            }
          }
        }
        if (p.acc != nullptr) {
          int32_t* ar = p.acc + static_cast<int64_t>(row) * p.N + n0;
          if (full_chunk && (p.N & 3) == 0) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              reinterpret_cast<uint4*>(ar)[q] = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n0 + j < p.N) ar[j] = static_cast<int32_t>(r[j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
    }
  }

  // One decision for the whole CTA: if any thread gave up on a wait, every
  // thread waits out the drain together, so the warp-wide dealloc below runs
  // converged and only after copies or MMAs still in flight have landed.
  if (__syncthreads_or(aborted ? 1 : 0)) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) {
    }
  }
  __syncwarp();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTcTmemCols);
  }
}

// ---------------------------------------------------------------------------
// tcgen05 kernel on CTA pairs (cluster of 2, cta_group::2): a 256 x 256 tile
// per pair, each CTA holding 128 rows of A and 128 rows (half the columns) of
// B per stage, so every CTA streams half the B bytes of the 1-CTA kernel and
// the 6-stage ring prefetches deeper in the same shared memory.  The leader
// CTA (rank 0) issues the MMAs for both; both CTAs' TMA loads complete on the
// leader's full barrier; every commit is sent to each CTA's barrier by its
// cluster address; each CTA's epilogue reads its own 128 TMEM lanes and
// releases the accumulator on the leader's barrier.
// ---------------------------------------------------------------------------
constexpr int kT2BM = 256;       // pair tile rows (128 per CTA)
constexpr int kT2BN = 256;       // pair tile columns (128 B rows per CTA)
constexpr int kT2Stages = 6;
constexpr uint32_t kT2StageA = 128 * kTcBK;
constexpr uint32_t kT2StageB = 128 * kTcBK;
constexpr int kT2GroupM = 16;    // pair m-blocks per rasterisation group (4096 rows of A share each B tile)
constexpr size_t kT2SmemBytes = 1024 + kT2Stages * (kT2StageA + kT2StageB) + 256;
constexpr uint32_t kT2Idesc = (2u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(kT2BN) >> 3) << 17) |
                              ((static_cast<uint32_t>(kT2BM) >> 4) << 24);

// FP4 variant (E2M1 activations x E2M1-coded ternary weights, kind::mxf4): a
// 128-byte stage row holds 256 values, an MMA takes K = 64 (32 bytes), so the
// same ring moves twice the K of the int8 kernel.  The fp32 accumulator holds
// the exact sum (every partial sum is a multiple of 1/2 far below 2^24).  Tiles
// are 256 x 224 so that two accumulators (2 x 224 TMEM columns) and the block
// scales (64 columns, every byte 2^0 in UE8M0) fit in the 512 columns.
constexpr int kF4BN = 224;
constexpr uint32_t kF4StageB = (kF4BN / 2) * kTcBK;
constexpr size_t kF4SmemBytes = 1024 + kT2Stages * (kT2StageA + kF4StageB) + 256;
constexpr uint32_t kF4SfCol = 2 * kF4BN;    // scale-factor columns 448..511
constexpr uint32_t kF4Idesc = (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(kF4BN) >> 3) << 17) | (1u << 23) |
                              ((static_cast<uint32_t>(kT2BM) >> 4) << 24);   // E2M1 x E2M1, UE8M0 scales, K = 64

template <bool FP4>
struct PairCfg {
  static constexpr int BN = FP4 ? kF4BN : kT2BN;
  static constexpr uint32_t StageB = FP4 ? kF4StageB : kT2StageB;
};

__device__ __forceinline__ void t2_tile_coords(int tile, int nmb, int nnb, int& mb, int& nb) {
  const int group = tile / (kT2GroupM * nnb);
  const int first_m = group * kT2GroupM;
  const int gsize = min(nmb - first_m, kT2GroupM);
  const int in = tile - group * kT2GroupM * nnb;
  mb = first_m + in % gsize;
  nb = in / gsize;
}

// One row's 32 consecutive accumulators -> y (bf16, scaled) and/or acc (int32).
// FP4: the accumulators are fp32 sums of E2M1 values (multiples of 1/2); acc
// receives twice the sum.
template <bool FP4 = false>
__device__ __forceinline__ void epilogue_chunk(const TcParams& p, int row, int n0, float rs, const uint32_t (&r)[32]) {
  const int group = static_cast<int>(p.alpha_group);   // host keeps alpha_group < 2^31
  const int ga = n0 / group;
  const bool one_alpha = (n0 + 31) / group == ga;
  const float cs_uniform = __fmul_rn(rs, ld_dep_f32(p.alpha + ga));
  float yv[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float cs = one_alpha ? cs_uniform : __fmul_rn(rs, ld_dep_f32(p.alpha + min(n0 + j, p.N - 1) / group));
    yv[j] = __fmul_rn(FP4 ? __uint_as_float(r[j]) : __int2float_rn(static_cast<int>(r[j])), cs);
  }
  const bool full_chunk = n0 + 32 <= p.N;
  if (p.y != nullptr) {
    uint16_t* yr = p.y + static_cast<int64_t>(row) * p.ldy + n0;
    if (full_chunk) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 o;
        o.x = pack_bf16x2(yv[8 * q + 0], yv[8 * q + 1]);
        o.y = pack_bf16x2(yv[8 * q + 2], yv[8 * q + 3]);
        o.z = pack_bf16x2(yv[8 * q + 4], yv[8 * q + 5]);
        o.w = pack_bf16x2(yv[8 * q + 6], yv[8 * q + 7]);
        st_global_stream_v4(reinterpret_cast<uint4*>(yr) + q, o);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (n0 + j < p.N) {
          const __nv_bfloat16 b = __float2bfloat16_rn(yv[j]);
          yr[j] = *reinterpret_cast<const uint16_t*>(&b);
        }
      }
    }
  }
  if (p.acc != nullptr) {
    uint32_t iv[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
      iv[j] = FP4 ? static_cast<uint32_t>(__float2int_rn(__fmul_rn(__uint_as_float(r[j]), 2.f))) : r[j];
    int32_t* ar = p.acc + static_cast<int64_t>(row) * p.N + n0;
    if (full_chunk && (p.N & 3) == 0) {
#pragma unroll
      for (int q = 0; q < 8; ++q)
        reinterpret_cast<uint4*>(ar)[q] = make_uint4(iv[4 * q], iv[4 * q + 1], iv[4 * q + 2], iv[4 * q + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (n0 + j < p.N) ar[j] = static_cast<int32_t>(iv[j]);
    }
  }
}

constexpr int kT2Threads = 320;  // warp 0: TMA, warp 1: MMA (leader), warps 2-9: epilogue

template <bool FP4>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kT2Threads, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TcParams p) {
  constexpr int BN = PairCfg<FP4>::BN;
  constexpr uint32_t SB = PairCfg<FP4>::StageB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kT2Stages * kT2StageA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kT2Stages * SB);
  uint64_t* full = bars;
  uint64_t* empty = bars + kT2Stages;
  uint64_t* tfull = bars + 2 * kT2Stages;
  uint64_t* tempty = bars + 2 * kT2Stages + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kT2Stages + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kT2Stages; ++s) {
      mbar_init(&full[s], 1);    // the leader's arrive.expect_tx; both CTAs' bytes
      mbar_init(&empty[s], 1);   // one commit from the leader's MMA thread
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 16);  // 8 epilogue warps in each CTA
    }
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTcTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();   // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if constexpr (FP4) {
    // block scales: every byte 0x7F (2^0 in UE8M0) in columns 448..511 of all 128 lanes
    if (warp >= 2 && warp < 6) {
      uint32_t ones[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) ones[j] = 0x7F7F7F7Fu;
      const uint32_t lanes = static_cast<uint32_t>((warp & 3) * 32) << 16;
      tmem_st_32x32b_x32(tmem_base + lanes + kF4SfCol, ones);
      tmem_st_32x32b_x32(tmem_base + lanes + kF4SfCol + 32, ones);
      tmem_wait_st();
    }
    tc_fence_before();
    cluster_sync_all();   // scales in place in both CTAs before the first MMA
    tc_fence_after();
  }
  pdl_wait();
  pdl_trigger();   // after the tensor-memory allocation and the wait, as in gemm_tc_kernel
  bool aborted = false;

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      for (int tile = pair; tile < p.num_tiles && !aborted; tile += npairs) {
        int mb, nb;
        t2_tile_coords(tile, p.num_m_blocks, p.num_n_blocks, mb, nb);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u)) {
            aborted = true;
            break;
          }
          const uint32_t leader_full = mapa_shared(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * (kT2StageA + SB));
          tma_load_2d_pair(&tmA, leader_full, sA + s * kT2StageA, kb * kTcBK, mb * kT2BM + rank * 128);
          tma_load_2d_pair(&tmB, leader_full, sB + s * SB, kb * kTcBK, nb * BN + rank * (BN / 2));
          if (++s == kT2Stages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader CTA, one thread) ----------------
    if (leader && lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int local = 0;
      for (int tile = pair; tile < p.num_tiles && !aborted; tile += npairs, ++local) {
        const int buf = local & 1;
        const uint32_t tph = (local >> 1) & 1;
        if (!mbar_wait_bounded(&tempty[buf], tph ^ 1u)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(&full[s], ph)) {
            aborted = true;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kT2StageA);
          const uint32_t b0 = smem_u32(sB + s * SB);
#pragma unroll
          for (int kk = 0; kk < kTcBK / 32; ++kk) {
            if constexpr (FP4) {
              mma_mxf4_pair(d_tmem, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), kF4Idesc,
                            tmem_base + kF4SfCol, tmem_base + kF4SfCol + 32, (kb | kk) != 0 ? 1u : 0u);
            } else {
              mma_i8_pair(d_tmem, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), kT2Idesc,
                          (kb | kk) != 0 ? 1u : 0u);
            }
          }
          // free stage s in both CTAs once these MMAs have read it
          mma_commit_pair(mapa_shared(smem_u32(&empty[s]), 0));
          mma_commit_pair(mapa_shared(smem_u32(&empty[s]), 1));
          if (++s == kT2Stages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (aborted) break;
        mma_commit_pair(mapa_shared(smem_u32(&tfull[buf]), 0));   // accumulator ready in both CTAs
        mma_commit_pair(mapa_shared(smem_u32(&tfull[buf]), 1));
      }
    }
  } else {
    // ---------------- epilogue (warps 2-9 of both CTAs) ----------------
    // Two warps per TMEM lane quadrant, up to 4 chunks of 32 columns each; the
    // TMEM load of the next chunk is in flight while the current one is stored.
    const int quad = warp & 3;
    constexpr int kChunks = BN / 32;
    const int c_begin = ((warp - 2) >> 2) * 4;
    const int c_end = min(c_begin + 4, kChunks);
    int local = 0;
    for (int tile = pair; tile < p.num_tiles; tile += npairs, ++local) {
      const int buf = local & 1;
      const uint32_t tph = (local >> 1) & 1;
      if (!warp_wait(&tfull[buf], tph)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      int mb, nb;
      t2_tile_coords(tile, p.num_m_blocks, p.num_n_blocks, mb, nb);
      const int row = mb * kT2BM + static_cast<int>(rank) * 128 + quad * 32 + lane;
      const bool row_ok = row < p.M;
      const float rs = row_ok ? ld_dep_f32(p.a_scale + row) : 0.f;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf * BN);
      uint32_t ra[32], rb[32];
      if (c_begin < c_end) {
        tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>(c_begin * 32), ra);
        tmem_wait_ld();
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = c_begin + i;
        if (c >= c_end) break;
        uint32_t(&r)[32] = (i & 1) ? rb : ra;
        if (c + 1 < c_end) tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>((c + 1) * 32), (i & 1) ? ra : rb);
        const int n0 = nb * BN + c * 32;
        if (row_ok && n0 < p.N) epilogue_chunk<FP4>(p, row, n0, rs, r);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[buf]), 0));
    }
  }

  // CTA-wide abort decision (see gemm_tc_kernel): the drain is taken by every
  // thread or by none, before the aligned cluster barrier and the dealloc.
  if (__syncthreads_or(aborted ? 1 : 0)) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) {
    }
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();   // no CTA leaves while its peer may still signal its barriers
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTcTmemCols);
}

// ---------------------------------------------------------------------------
// gemm_t2tc_kernel -- 2-bit ternary weights x int8 activations on the tensor
// cores, for few tokens (decode).  The product is taken transposed,
//   D[n, m] = sum_k t[n, k] * a[m, k],
// so 128 weight rows form the MMA's M side and the tokens its N side (8, or a
// multiple of 16 up to 256).  The weights stay 2-bit in HBM and shared memory:
// widen warps turn each 16-code word into int8 in registers (5 bit operations
// and 8 byte permutes) and store the rows into tensor memory, which the MMA
// reads as its A operand; the activations reach shared memory by TMA in the
// 128-byte-swizzled layout of the B operand.
//   warp 0: TMA producer    warp 1: MMA issuer (one thread)
//   warps 2-9: widen (warp w owns TMEM lanes 32*(w%4).. and half of every
//              64-byte piece of its rows), then the epilogue of each tile
// A TMA stage carries SUB sub-stages of 256 codes (SUB*64 bytes of each of the
// tile's 128 weight rows): the TMA engine moves a box row at a time, so longer
// rows move more bytes per SM.  Each sub-stage is widened into one of several
// TMEM A buffers, so the widen warps run ahead of the MMA.  Consecutive MMAs go
// to up to four accumulators in turn (summed in the epilogue).  A work unit is
// one 128-row weight tile against one block of tokens, over all of K; the grid
// is persistent over units.
// ---------------------------------------------------------------------------
constexpr int kTsBN = 128;                 // weight rows per tile (MMA M)
constexpr int kTsSubK = 256;               // codes per sub-stage: 64 bytes of 2-bit weights per row
constexpr int kTsWidenWarps = 8;
constexpr int kTsThreads = 32 * (2 + kTsWidenWarps);
constexpr uint32_t kTsACols = kTsSubK / 4; // TMEM columns of one widened sub-stage (4 codes per column)
constexpr int kTsMaxStages = 16;
constexpr int kTsMaxABufs = 6;             // widened sub-stages held in TMEM
// Below this many tokens the CUDA-core kernel is faster: every tcgen05.mma
// (M = 128, K = 32) costs about a hundred cycles of issue whatever N is, while
// the CUDA-core kernel's work grows with the token count.
constexpr int kTsMinTokens = 8;

struct TsParams {
  const float* a_scale;
  const float* alpha;
  int64_t alpha_group;
  int M, N, K;
  uint16_t* y;
  int64_t ldy;
  int32_t* acc;
  int nt;                 // tokens per MMA (N side)
  int num_n_tiles, num_units, num_kb, stages;
  uint32_t stage_x;       // activation bytes per stage (nt * 256 * SUB)
  uint32_t abufs;         // TMEM A buffers (2..kTsMaxABufs)
  uint32_t dslots;        // accumulators (1, 2 or 4)
};

// int8 of a 2-bit code {00 -> 0, 01 -> 1, 11 -> -1}, as byte permute table.
constexpr uint32_t kT2Lut = 0xFF000100u;

// 16 codes (element e in bits 2e..2e+1) -> 4 words of int8, element order kept.
__device__ __forceinline__ void widen_t2_word(uint32_t x, uint32_t* out) {
  const uint32_t m1 = x & 0x33333333u;           // nibble i: code 2i
  const uint32_t m2 = (x >> 2) & 0x33333333u;    // nibble i: code 2i+1
  const uint32_t e0 = __byte_perm(kT2Lut, kT2Lut, m1);          // codes 0, 2, 4, 6
  const uint32_t e1 = __byte_perm(kT2Lut, kT2Lut, m2);          // codes 1, 3, 5, 7
  const uint32_t e2 = __byte_perm(kT2Lut, kT2Lut, m1 >> 16);    // codes 8, 10, 12, 14
  const uint32_t e3 = __byte_perm(kT2Lut, kT2Lut, m2 >> 16);    // codes 9, 11, 13, 15
  out[0] = __byte_perm(e0, e1, 0x5140);
  out[1] = __byte_perm(e0, e1, 0x7362);
  out[2] = __byte_perm(e2, e3, 0x5140);
  out[3] = __byte_perm(e2, e3, 0x7362);
}

template <int SUB>
__global__ void __launch_bounds__(kTsThreads, 1)
    gemm_t2tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, TsParams p) {
  constexpr uint32_t kStageW = kTsBN * SUB * (kTsSubK / 4);   // weight bytes per stage
  constexpr int kRowBytes = SUB * (kTsSubK / 4);              // bytes of one weight row per stage
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem;
  uint8_t* sW = smem + static_cast<size_t>(p.stages) * p.stage_x;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sW + static_cast<size_t>(p.stages) * kStageW);
  uint64_t* full = bars;
  uint64_t* empty = bars + kTsMaxStages;
  uint64_t* afull = bars + 2 * kTsMaxStages;
  uint64_t* aempty = afull + kTsMaxABufs;
  uint64_t* dfull = aempty + kTsMaxABufs;
  uint64_t* dempty = dfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dempty + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kTsWidenWarps);   // MMA commit (activations read) + widen warps (weights read)
    }
    for (int b = 0; b < static_cast<int>(p.abufs); ++b) {
      mbar_init(&afull[b], kTsWidenWarps);
      mbar_init(&aempty[b], 1);
    }
    mbar_init(dfull, 1);
    mbar_init(dempty, kTsWidenWarps);
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t d_col = p.abufs * kTsACols;  // accumulators follow the A buffers
  if (warp == 0 && lane == 0 && blockIdx.x < p.num_units) {
    // pull the first unit's weight tiles into L2 while the previous kernel finishes
    const int nb = blockIdx.x % p.num_n_tiles;
    for (int kb = 0; kb < p.num_kb; ++kb) tma_prefetch_2d(&tmW, kb * (kRowBytes / 8), nb * kTsBN);
  }
  pdl_wait();
  pdl_trigger();   // after the tensor-memory allocation and the wait, as in gemm_tc_kernel
  bool aborted = false;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      for (int unit = blockIdx.x; unit < p.num_units && !aborted; unit += gridDim.x) {
        const int nb = unit % p.num_n_tiles, mb = unit / p.num_n_tiles;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u)) {
            aborted = true;
            break;
          }
          uint8_t* xs = sX + static_cast<size_t>(s) * p.stage_x;
          mbar_arrive_expect_tx(&full[s], p.stage_x + kStageW);
          tma_load_2d(&tmW, &full[s], sW + static_cast<size_t>(s) * kStageW, kb * (kRowBytes / 8), nb * kTsBN);
#pragma unroll
          for (int q = 0; q < 2 * SUB; ++q)
            tma_load_2d(&tmX, &full[s], xs + q * p.nt * 128, kb * SUB * kTsSubK + 128 * q, mb * p.nt);
          if (++s == p.stages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (one thread) ----------------
    if (lane == 0) {
      const uint32_t idesc = (2u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(p.nt) >> 3) << 17) |
                             ((static_cast<uint32_t>(kTsBN) >> 4) << 24);
      int s = 0;
      uint32_t ph = 0, abuf = 0, aph = 0;
      int local = 0;
      for (int unit = blockIdx.x; unit < p.num_units && !aborted; unit += gridDim.x, ++local) {
        if (!mbar_wait_bounded(dempty, (static_cast<uint32_t>(local) & 1u) ^ 1u)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < p.num_kb && !aborted; ++kb) {
          if (!mbar_wait_bounded(&full[s], ph)) {
            aborted = true;
            break;
          }
          const uint32_t xs = smem_u32(sX + static_cast<size_t>(s) * p.stage_x);
          for (int j = 0; j < SUB; ++j) {
            if (!mbar_wait_bounded(&afull[abuf], aph)) {
              aborted = true;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kTsSubK / 32; ++kk) {
              const uint32_t slot = static_cast<uint32_t>(kk) & (p.dslots - 1u);
              const uint32_t a_tmem = tmem_base + abuf * kTsACols + static_cast<uint32_t>(kk * 8);
              const uint32_t b_addr = xs + static_cast<uint32_t>((2 * j + (kk >> 2)) * p.nt * 128 + (kk & 3) * 32);
              mma_i8_ts(tmem_base + d_col + slot * static_cast<uint32_t>(p.nt), a_tmem, sw128_kmajor_desc(b_addr),
                        idesc, (kb != 0 || j != 0 || static_cast<uint32_t>(kk) >= p.dslots) ? 1u : 0u);
            }
            mma_commit(&aempty[abuf]);    // widened weights of this sub-stage read
            if (++abuf == p.abufs) {
              abuf = 0;
              aph ^= 1u;
            }
          }
          if (aborted) break;
          mma_commit(&empty[s]);          // activations of this stage read
          if (++s == p.stages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (aborted) break;
        mma_commit(dfull);                // accumulators ready
      }
    }
  } else if (warp < 2 + kTsWidenWarps) {
    // ---------------- widen + epilogue (warps 2-9) ----------------
    const int wi = warp - 2;
    const int quad = warp & 3;
    const int half = wi >> 2;
    const int trow = quad * 32 + lane;                    // weight row within the tile = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    int s = 0;
    uint32_t ph = 0, abuf = 0, aph = 0;
    int local = 0;
    for (int unit = blockIdx.x; unit < p.num_units && !aborted; unit += gridDim.x, ++local) {
      const int nb = unit % p.num_n_tiles, mb = unit / p.num_n_tiles;
      for (int kb = 0; kb < p.num_kb && !aborted; ++kb) {
        if (!warp_wait(&full[s], ph)) {
          aborted = true;
          break;
        }
        // this thread's bytes of the stage: SUB pieces of 64 bytes, it widens 32 of each
        const uint8_t* row = sW + static_cast<size_t>(s) * kStageW + trow * kRowBytes + half * 32;
        uint4 w[SUB][2];
#pragma unroll
        for (int j = 0; j < SUB; ++j) {
          w[j][0] = reinterpret_cast<const uint4*>(row + j * 64)[0];
          w[j][1] = reinterpret_cast<const uint4*>(row + j * 64)[1];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);            // this warp is done with the stage's weights
#pragma unroll
        for (int j = 0; j < SUB; ++j) {
          if (!warp_wait(&aempty[abuf], aph ^ 1u)) {
            aborted = true;
            break;
          }
          const uint32_t x[8] = {w[j][0].x, w[j][0].y, w[j][0].z, w[j][0].w,
                                 w[j][1].x, w[j][1].y, w[j][1].z, w[j][1].w};
          uint32_t a[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) widen_t2_word(x[i], a + 4 * i);
          tc_fence_after();
          tmem_st_32x32b_x32(tmem_base + lane_addr + abuf * kTsACols + static_cast<uint32_t>(half * 32), a);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&afull[abuf]);
          if (++abuf == p.abufs) {
            abuf = 0;
            aph ^= 1u;
          }
        }
        if (++s == p.stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (aborted) break;
      // epilogue: lane = weight row n, columns = tokens; the two warps of a
      // quadrant take alternate 8-column chunks
      if (!warp_wait(dfull, static_cast<uint32_t>(local) & 1u)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      const int n = nb * kTsBN + trow;
      const bool n_ok = n < p.N;
      const float al = n_ok ? ld_dep_f32(p.alpha + n / p.alpha_group) : 0.f;
      for (int c = half; c < p.nt / 8; c += 2) {
        uint32_t r[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (uint32_t slot = 0; slot < p.dslots; ++slot) {
          uint32_t t[8];
          tmem_ld_32x32b_x8(tmem_base + lane_addr + d_col + slot * static_cast<uint32_t>(p.nt) +
                                static_cast<uint32_t>(c * 8),
                            t);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j) r[j] += t[j];
        }
        if (!n_ok) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int m = mb * p.nt + c * 8 + j;
          if (m >= p.M) break;
          const int v = static_cast<int>(r[j]);
          if (p.acc != nullptr) p.acc[static_cast<int64_t>(m) * p.N + n] = v;
          if (p.y != nullptr) {
            const float cs = __fmul_rn(ld_dep_f32(p.a_scale + m), al);
            const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn(__int2float_rn(v), cs));
            p.y[static_cast<int64_t>(m) * p.ldy + n] = *reinterpret_cast<const uint16_t*>(&b);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dempty);
    }
  }

  // CTA-wide abort decision (see gemm_tc_kernel)
  if (__syncthreads_or(aborted ? 1 : 0)) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) {
    }
  }
  __syncwarp();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------------------
// CUDA-core kernel for packed operands.  One warp per output column n (a row
// of W); lanes split K in units of 64 codes; MT rows of A per pass share the
// expanded weight unit.  dp4a on int8x4 words.
// ---------------------------------------------------------------------------
enum : int { kSimtA_I8 = 0, kSimtA_I4 = 1, kSimtA_E2M1 = 2 };
// GEMV activation sources that are bf16 rows quantized in the kernel's prologue
// (INT4 absmean, FP4 E2M1 MinMax as twice the value), bit-identical to quant_a4
enum : int { kGvX_Int4 = 3, kGvX_Fp4 = 4 };

// four 2-bit ternary codes (one byte) -> four int8 {-1,0,1} (two's-complement sign extension)
__device__ __forceinline__ uint32_t expand_t2_byte(uint32_t b) {
  const uint32_t spread = (b & 0x3u) | ((b & 0xCu) << 6) | ((b & 0x30u) << 12) | ((b & 0xC0u) << 18);
  return __vsub4(spread ^ 0x02020202u, 0x02020202u);
}

template <int AF>
__device__ __forceinline__ void load_a_unit(const uint8_t* a_row, int u, uint32_t (&out)[16]) {
  if constexpr (AF == kSimtA_I8) {
    const uint4* p = reinterpret_cast<const uint4*>(a_row + static_cast<int64_t>(u) * 64);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = ld_dep_v4(p + i);
      out[4 * i] = v.x; out[4 * i + 1] = v.y; out[4 * i + 2] = v.z; out[4 * i + 3] = v.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(a_row + static_cast<int64_t>(u) * 32);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 v = ld_dep_v4(p + i);
      const uint32_t pk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t w0, w1;
        split_nibbles(pk[j], w0, w1);
        if constexpr (AF == kSimtA_I4) {
          out[8 * i + 2 * j] = sext_nibble_bytes(w0);
          out[8 * i + 2 * j + 1] = sext_nibble_bytes(w1);
        } else {
          out[8 * i + 2 * j] = e2m1_bytes_to_twice(w0);
          out[8 * i + 2 * j + 1] = e2m1_bytes_to_twice(w1);
        }
      }
    }
  }
}

template <bool WT2>
__device__ __forceinline__ void load_w_unit(const uint8_t* w_row, int u, uint32_t (&out)[16]) {
  if constexpr (WT2) {
    const uint4 v = ld_global_nc_v4(w_row + static_cast<int64_t>(u) * 16);
    const uint32_t pk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int b = 0; b < 4; ++b) out[4 * j + b] = expand_t2_byte((pk[j] >> (8 * b)) & 0xFFu);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = ld_global_nc_v4(w_row + static_cast<int64_t>(u) * 64 + 16 * i);
      out[4 * i] = v.x; out[4 * i + 1] = v.y; out[4 * i + 2] = v.z; out[4 * i + 3] = v.w;
    }
  }
}

// A tile in shared memory: MT rows of K codes widened to int8, stored as words
// so that, for a fixed word i of a unit, the 32 lanes of a warp (units
// u = 32*uh + lane) read 32 consecutive words:  word(m, u, i) at
// ((m * units_hi + u / 32) * 16 + i) * 32 + u % 32.
__device__ __forceinline__ int simt_a_word(int m, int u, int i, int units_hi) {
  return ((m * units_hi + (u >> 5)) * 16 + i) * 32 + (u & 31);
}

// Rows per warp for a round of UPL units per lane: 2-bit weight units are 16 B,
// so a lane keeps UPL * R = 8 of them in flight; int8 units are 64 B (one row).
template <bool WT2, int UPL>
struct SimtShape {
  static constexpr int R = WT2 ? (UPL >= 8 ? 1 : 8 / UPL) : 1;
  static constexpr int Q = WT2 ? 1 : 4;  // 16-byte words per weight unit
};

template <int AF, bool WT2, int MT, int UPL>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const uint8_t* __restrict__ a, const float* __restrict__ a_scale,
                                                        const uint8_t* __restrict__ w, const float* __restrict__ alpha,
                                                        int64_t alpha_group, int M, int N, int K,
                                                        uint16_t* __restrict__ y, int64_t ldy,
                                                        int32_t* __restrict__ acc_out) {
  constexpr int R = SimtShape<WT2, UPL>::R;
  constexpr int Q = SimtShape<WT2, UPL>::Q;
  extern __shared__ uint32_t sa[];
  // byte of four 2-bit codes -> four int8 {-1,0,1}: one table read instead of bit arithmetic
  __shared__ uint32_t t2_table[256];
  if (WT2) t2_table[threadIdx.x & 255] = expand_t2_byte(threadIdx.x & 255);
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int units = K >> 6;                 // 64 codes per unit
  const int units_hi = (units + 31) >> 5;
  const int64_t a_row_bytes = (AF == kSimtA_I8) ? K : (K >> 1);
  const int64_t w_row_bytes = WT2 ? (K >> 2) : K;
  const float unit_scale = (AF == kSimtA_E2M1 || AF == kGvX_Fp4) ? 0.5f : 1.0f;
  pdl_wait();
  pdl_trigger();

  for (int m0 = 0; m0 < M; m0 += MT) {
    __syncthreads();  // the previous tile's readers are done with sa
    for (int i = threadIdx.x; i < MT * units_hi * 32; i += blockDim.x) {
      const int m = i / (units_hi * 32);
      const int u = i - m * units_hi * 32;
      uint32_t wv[16];
      if (m0 + m < M && u < units) {
        load_a_unit<AF>(a + static_cast<int64_t>(m0 + m) * a_row_bytes, u, wv);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) wv[j] = 0;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) sa[simt_a_word(m, u, j, units_hi)] = wv[j];
    }
    __syncthreads();

    for (int64_t n0 = (static_cast<int64_t>(blockIdx.x) * 8 + warp) * R; n0 < N;
         n0 += static_cast<int64_t>(gridDim.x) * 8 * R) {
      int acc[R][MT];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0;
      for (int u0 = 0; u0 < units; u0 += 32 * UPL) {
        // every weight load of the round first, so they are in flight together
        uint4 raw[UPL][R][Q];
#pragma unroll
        for (int j = 0; j < UPL; ++j) {
          const int u = u0 + j * 32 + lane;
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const bool ok = u < units && n0 + r < N;
            const uint8_t* wr = w + (n0 + r < N ? n0 + r : n0) * w_row_bytes + static_cast<int64_t>(u) * (WT2 ? 16 : 64);
#pragma unroll
            for (int q = 0; q < Q; ++q) raw[j][r][q] = ok ? ld_global_nc_v4(wr + 16 * q) : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int j = 0; j < UPL; ++j) {
          const int u = u0 + j * 32 + lane;
          if (u >= units) continue;
#pragma unroll
          for (int r = 0; r < R; ++r) {
            uint32_t wx[16];
            if constexpr (WT2) {
              const uint32_t pk[4] = {raw[j][r][0].x, raw[j][r][0].y, raw[j][r][0].z, raw[j][r][0].w};
#pragma unroll
              for (int jj = 0; jj < 4; ++jj)
#pragma unroll
                for (int b = 0; b < 4; ++b) wx[4 * jj + b] = t2_table[(pk[jj] >> (8 * b)) & 0xFFu];
            } else {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                wx[4 * q] = raw[j][r][q].x; wx[4 * q + 1] = raw[j][r][q].y;
                wx[4 * q + 2] = raw[j][r][q].z; wx[4 * q + 3] = raw[j][r][q].w;
              }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
              for (int i = 0; i < 16; ++i)
                acc[r][m] = __dp4a(static_cast<int>(sa[simt_a_word(m, u, i, units_hi)]), static_cast<int>(wx[i]), acc[r][m]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc[r][m] += __shfl_xor_sync(0xFFFFFFFFu, acc[r][m], o);
      // every lane holds every reduced sum; output (r, m) is written by lane (r * MT + m) % 32
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (lane == ((r * MT + m) & 31)) {
            const int64_t n = n0 + r;
            const int mm = m0 + m;
            if (n < N && mm < M) {
              const int v = acc[r][m];
              if (acc_out != nullptr) acc_out[static_cast<int64_t>(mm) * N + n] = v;
              if (y != nullptr) {
                const float cs = __fmul_rn(__fmul_rn(ld_dep_f32(a_scale + mm), unit_scale), ld_dep_f32(alpha + n / alpha_group));
                const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn(__int2float_rn(v), cs));
                y[static_cast<int64_t>(mm) * ldy + n] = *reinterpret_cast<const uint16_t*>(&b);
              }
            }
          }
        }
    }
  }
}

// ---------------------------------------------------------------------------
// gemv_t2_kernel -- 1 to 8 tokens against 2-bit ternary weights (decode).
//
// A 16-code weight word x (code e in bits 2e..2e+1: 00 -> 0, 01 -> +1,
// 11 -> -1) becomes offset codes c + 1 in {0, 1, 2} with one shift and one
// three-input logic op,
//     u = ~x & (0x55555555 | (x << 1))
// (a field's low bit is set for code 0 only, its high bit for +1 only).  Field
// j of every byte (code 4b + j of the word) is dotted with the activation
// bytes a[4b + j] by dp4a (unsigned x signed).  For one token the field is
// isolated in place by one AND, u & (0x03030303 << 2j) = 4^j (c + 1), into one
// of four accumulators, each an exact multiple of 4^j:
//     sum_k (c_k + 1) a_k  =  s_0 + s_1/4 + s_2/16 + s_3/64   (exact shifts);
// for several tokens the fields are shifted down once per word and every token
// keeps a single accumulator.  The token's sum_k a_k is subtracted at the end.
//
// The activations (INT8, INT4 or E2M1 codes; E2M1 as twice their value) are
// staged once per CTA in shared memory as int8, the 16 bytes of each word
// transposed field-major so that the four dp4a operands of a word are one
// 16-byte load.  CTAs are persistent: G row groups of R rows per pass, warp w
// taking group w / S and 4096-code round w % S of it; the S partial sums of a
// row meet in shared memory.  Before its wait each warp issues L2 prefetches
// for every weight byte it will read, so HBM streams the whole matrix while
// the CTAs stage activations and compute.
// ---------------------------------------------------------------------------
// 16 activation codes -> the field-major word f (field j = bytes j of v[0..3])
// and the sum of the codes
__device__ __forceinline__ uint4 gv_transpose(const uint32_t (&v)[4], int& sum) {
  const uint32_t t0 = __byte_perm(v[0], v[1], 0x5140), t1 = __byte_perm(v[0], v[1], 0x7362);
  const uint32_t t2 = __byte_perm(v[2], v[3], 0x5140), t3 = __byte_perm(v[2], v[3], 0x7362);
  const uint4 f = make_uint4(__byte_perm(t0, t2, 0x5410), __byte_perm(t0, t2, 0x7632),
                             __byte_perm(t1, t3, 0x5410), __byte_perm(t1, t3, 0x7632));
  int sv = __dp4a(static_cast<int>(f.x), 0x01010101, 0);
  sv = __dp4a(static_cast<int>(f.y), 0x01010101, sv);
  sv = __dp4a(static_cast<int>(f.z), 0x01010101, sv);
  sum += __dp4a(static_cast<int>(f.w), 0x01010101, sv);
  return f;
}

template <int MT>
struct GvShape {
  static constexpr int R = 4;   // weight rows per warp
};
constexpr int kGvMaxThreads = 512;

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// 16 activation codes of word q of row m as int8, element order (w[i] holds 4i..4i+3)
template <int AF>
__device__ __forceinline__ void gv_load_word(const uint8_t* a, int K, int m, int q, uint32_t (&w)[4]) {
  if constexpr (AF == kSimtA_I8) {
    const uint4 v = ld_dep_v4(a + static_cast<int64_t>(m) * K + static_cast<int64_t>(q) * 16);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else {
    const uint8_t* src = a + static_cast<int64_t>(m) * (K >> 1) + static_cast<int64_t>(q) * 8;
    uint32_t p0, p1;
    asm volatile("ld.global.v2.u32 {%0,%1}, [%2];" : "=r"(p0), "=r"(p1) : "l"(src));
    uint32_t n[4];
    split_nibbles(p0, n[0], n[1]);
    split_nibbles(p1, n[2], n[3]);
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = AF == kSimtA_I4 ? sext_nibble_bytes(n[i]) : e2m1_bytes_to_twice(n[i]);
  }
}
// Stage the activations of M tokens into shared memory as field-major int8
// words (gv_transpose) at act[slot(q, m)], zeros for the token slots M..TOK-1,
// and add each token's code sum to asum[m].  A thread's loads for all tokens of
// a word are in flight together.  For the bf16 sources (kGvX_*) the tokens are
// quantized here as quant_a4 does it: a first pass over the rows reduces each
// token's statistic (the exact fp64 sum of |x|, or max |x|) over the CTA
// through red[warp][token], the second quantizes; s_scale[m] receives the
// token's dequant scale.
template <int AF>
constexpr bool gv_fused() { return AF == kGvX_Int4 || AF == kGvX_Fp4; }

constexpr int kGvMaxWarps = kGvMaxThreads / 32;

// bf16 x 8 -> eight int8 codes in two words (INT4: the code; FP4: twice the value)
template <int AF>
__device__ __forceinline__ void gv_quant8(const uint4& h, float mult, int p, uint32_t& lo, uint32_t& hi) {
  float f[8];
  unpack_bf16x8(h, f);
  uint32_t q[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    if constexpr (AF == kGvX_Int4) {
      q[e] = q4_code_bits(f[e], mult);   // low byte: the code, two's complement
    } else {
      const float sv = mul_pow2(f[e], -p);
      const int i = e2m1_index(fabsf(sv));
      const int tv = (i <= 4) ? i : (i == 5 ? 6 : (i == 6 ? 8 : 12));
      q[e] = static_cast<uint32_t>((sv < 0.f && i != 0) ? -tv : tv);
    }
  }
  lo = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
  hi = __byte_perm(__byte_perm(q[4], q[5], 0x0040), __byte_perm(q[6], q[7], 0x0040), 0x5410);
}

template <int AF, int TOK, typename Slot>
__device__ __forceinline__ void gv_stage(const uint8_t* a, int64_t ldx, float eps, int M, int K, uint4* act,
                                         Slot slot, int* asum, double (*red)[TOK], float* s_scale) {
  const int kw16 = K >> 4;
  float mult[TOK];
  int pexp[TOK];
#pragma unroll
  for (int m = 0; m < TOK; ++m) {
    mult[m] = 0.f;
    pexp[m] = 0;
  }
  if constexpr (gv_fused<AF>()) {
    const uint16_t* x = reinterpret_cast<const uint16_t*>(a);
    double ps[TOK];
    uint32_t pm[TOK];
#pragma unroll
    for (int m = 0; m < TOK; ++m) {
      ps[m] = 0.0;
      pm[m] = 0u;
    }
    for (int q = threadIdx.x; q < kw16; q += blockDim.x) {
#pragma unroll
      for (int m = 0; m < TOK; ++m) {
        if (m >= M) continue;
        const uint16_t* src = x + static_cast<int64_t>(m) * ldx + static_cast<int64_t>(q) * 16;
        const uint4 h[2] = {ld_dep_v4(src), ld_dep_v4(src + 8)};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          if constexpr (AF == kGvX_Int4) {
            float f[8];
            unpack_bf16x8(h[hh], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) ps[m] += static_cast<double>(fabsf(f[e]));
          } else {
            uint32_t k[8];
            bf16x8_mag_keys(h[hh], k);
#pragma unroll
            for (int e = 0; e < 8; ++e) pm[m] = max(pm[m], k[e]);
          }
        }
      }
    }
    const int warp = threadIdx.x >> 5;
#pragma unroll
    for (int m = 0; m < TOK; ++m) {
      if constexpr (AF == kGvX_Int4) {
        double v = ps[m];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        if ((threadIdx.x & 31) == 0) red[warp][m] = v;
      } else {
        const uint32_t v = __reduce_max_sync(0xFFFFFFFFu, pm[m]);
        if ((threadIdx.x & 31) == 0) red[warp][m] = static_cast<double>(v);
      }
    }
    __syncthreads();
    const int nw = static_cast<int>(blockDim.x >> 5);
#pragma unroll
    for (int m = 0; m < TOK; ++m) {
      float sc;
      if constexpr (AF == kGvX_Int4) {
        // the sum of bf16 magnitudes in fp64 is exact, so the order of the
        // partial sums does not change it (the same value as quant_a4's)
        double S = 0.0;
        for (int i = 0; i < nw; ++i) S += red[i][m];
        const float beta = __double2float_rn(S / static_cast<double>(K));
        mult[m] = __fdiv_rn(sqrt7_f32(), __fadd_rn(beta, eps));
        sc = __fdiv_rn(beta, sqrt7_f32());
      } else {
        uint32_t mk = 0u;
        for (int i = 0; i < nw; ++i) mk = max(mk, static_cast<uint32_t>(red[i][m]));
        pexp[m] = fp4_scale_exponent(mk << 16);
        sc = exact_pow2(pexp[m]);
      }
      if (threadIdx.x == m && m < M) s_scale[m] = sc;
    }
  }
  int tsum[TOK];
#pragma unroll
  for (int m = 0; m < TOK; ++m) tsum[m] = 0;
  for (int q = threadIdx.x; q < kw16; q += blockDim.x) {
    uint32_t v[TOK][4];
#pragma unroll
    for (int m = 0; m < TOK; ++m) {
      v[m][0] = v[m][1] = v[m][2] = v[m][3] = 0u;
      if (m >= M) continue;
      if constexpr (gv_fused<AF>()) {
        const uint16_t* src =
            reinterpret_cast<const uint16_t*>(a) + static_cast<int64_t>(m) * ldx + static_cast<int64_t>(q) * 16;
        const uint4 h0 = ld_dep_v4(src), h1 = ld_dep_v4(src + 8);
        gv_quant8<AF>(h0, mult[m], pexp[m], v[m][0], v[m][1]);
        gv_quant8<AF>(h1, mult[m], pexp[m], v[m][2], v[m][3]);
      } else {
        gv_load_word<AF>(a, K, m, q, v[m]);
      }
    }
#pragma unroll
    for (int m = 0; m < TOK; ++m) act[slot(q, m)] = gv_transpose(v[m], tsum[m]);
  }
#pragma unroll
  for (int m = 0; m < TOK; ++m) {
    const int v = __reduce_add_sync(0xFFFFFFFFu, tsum[m]);
    if ((threadIdx.x & 31) == 0 && v != 0) atomicAdd(&asum[m], v);
  }
}

template <int AF, int MT>
__global__ void __launch_bounds__(kGvMaxThreads) gemv_t2_kernel(const uint8_t* __restrict__ a,
                                                                const float* __restrict__ a_scale,
                                                                const uint8_t* __restrict__ w,
                                                                const float* __restrict__ alpha, int64_t alpha_group,
                                                                int M, int N, int K, int S, int G,
                                                                uint16_t* __restrict__ y, int64_t ldy,
                                                                int32_t* __restrict__ acc_out, int64_t ldx,
                                                                float eps) {
  constexpr int R = GvShape<MT>::R;
  extern __shared__ uint4 gv_smem[];
  __shared__ int asum[MT];
  __shared__ float s_scale[MT];
  __shared__ double red[kGvMaxWarps][MT];
  const int kw16 = K >> 4;                              // 16-code words per row
  const int kq = kw16 >> 2;                             // words per lane slot (kw16 % 4 == 0)
  uint4* act = gv_smem;                                 // [MT][4][kw16 / 4], field-major bytes
  int* part = reinterpret_cast<int*>(act + MT * kw16);  // [2][G][S][R][MT] partial sums
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = warp / S;
  const int rd = warp - g * S;
  const int64_t wrow_bytes = K >> 2;
  const int64_t groups = (static_cast<int64_t>(N) + R - 1) / R;
  const int64_t group_step = static_cast<int64_t>(gridDim.x) * G;

  // every weight line this warp will read (R rows x its 1 KiB round per pass)
  // into L2 while the previous kernel finishes
  if (lane < 8 * R) {
    const int r = lane >> 3;
    const int64_t b = static_cast<int64_t>(rd) * 1024 + (lane & 7) * 128;
    if (b < wrow_bytes)
      for (int64_t gi = static_cast<int64_t>(blockIdx.x) * G + g; gi < groups; gi += group_step) {
        const int64_t n = gi * R + r;
        if (n < N) prefetch_l2(w + n * wrow_bytes + b);
      }
  }
  if (threadIdx.x < MT) asum[threadIdx.x] = 0;
  __syncthreads();
  pdl_wait();
  pdl_trigger();

  // weights of a pass: lane l holds words 4l..4l+3 and 128+4l..128+4l+3 of the
  // round; the first pass's loads go out before the activations are staged
  uint4 wv[R][2];
  auto load_weights = [&](int64_t gb) {
    const int64_t n0 = (gb + g) * R;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int wq = rd * 256 + h * 128 + 4 * lane;
      const bool ok = gb < groups && n0 < N && wq < kw16;   // kw16 is a multiple of 4
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int64_t n = n0 + r < N ? n0 + r : n0;
        wv[r][h] = ok ? ld_global_nc_v4(w + n * wrow_bytes + static_cast<int64_t>(wq) * 4) : make_uint4(0, 0, 0, 0);
      }
    }
  };
  load_weights(static_cast<int64_t>(blockIdx.x) * G);

  // stage the activations (zeros for token slots past M) and their sums
  // word 4p + j of token m at [m][j][p]: the lanes of a warp read consecutive slots
  gv_stage<AF, MT>(a, ldx, eps, M, K, act, [kq](int q, int m) { return (m * 4 + (q & 3)) * kq + (q >> 2); }, asum,
                   red, s_scale);
  __syncthreads();
  const float unit_scale = (AF == kSimtA_E2M1 || AF == kGvX_Fp4) ? 0.5f : 1.0f;

  int par = 0;
  for (int64_t gb = static_cast<int64_t>(blockIdx.x) * G; gb < groups; gb += group_step, par ^= 1) {
    const int64_t n0 = (gb + g) * R;
    const bool rows_ok = n0 < N;
    int tot[R][MT];
    if constexpr (MT == 1) {
      int acc[R][4];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[r][j] = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int wq = rd * 256 + h * 128 + 4 * lane;
        if (!rows_ok || wq >= kw16) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 av = act[j * kq + (wq >> 2)];
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const uint32_t x = j == 0 ? wv[r][h].x : (j == 1 ? wv[r][h].y : (j == 2 ? wv[r][h].z : wv[r][h].w));
            const uint32_t u = ~x & (0x55555555u | (x << 1));
            acc[r][0] = dp4a_us(u & 0x03030303u, av.x, acc[r][0]);
            acc[r][1] = dp4a_us(u & 0x0C0C0C0Cu, av.y, acc[r][1]);
            acc[r][2] = dp4a_us(u & 0x30303030u, av.z, acc[r][2]);
            acc[r][3] = dp4a_us(u & 0xC0C0C0C0u, av.w, acc[r][3]);
          }
        }
      }
      load_weights(gb + group_step);   // the next pass's loads overlap the reductions
#pragma unroll
      for (int r = 0; r < R; ++r)
        tot[r][0] = __reduce_add_sync(0xFFFFFFFFu, acc[r][0] + (acc[r][1] >> 2) + (acc[r][2] >> 4) + (acc[r][3] >> 6));
    } else {
      int acc[R][MT];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int wq = rd * 256 + h * 128 + 4 * lane;
        if (!rows_ok || wq >= kw16) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t f[R][4];
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const uint32_t x = j == 0 ? wv[r][h].x : (j == 1 ? wv[r][h].y : (j == 2 ? wv[r][h].z : wv[r][h].w));
            const uint32_t u = ~x & (0x55555555u | (x << 1));
            f[r][0] = u & 0x03030303u;
            f[r][1] = (u >> 2) & 0x03030303u;
            f[r][2] = (u >> 4) & 0x03030303u;
            f[r][3] = (u >> 6) & 0x03030303u;
          }
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const uint4 av = act[(m * 4 + j) * kq + (wq >> 2)];
#pragma unroll
            for (int r = 0; r < R; ++r) {
              int t = dp4a_us(f[r][0], av.x, acc[r][m]);
              t = dp4a_us(f[r][1], av.y, t);
              t = dp4a_us(f[r][2], av.z, t);
              acc[r][m] = dp4a_us(f[r][3], av.w, t);
            }
          }
        }
      }
      load_weights(gb + group_step);
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) tot[r][m] = __reduce_add_sync(0xFFFFFFFFu, acc[r][m]);
    }
    if (S > 1) {
      // rounds of a row group meet in shared memory (two buffers: the readers
      // of one pass are done before the pass after next writes it again)
      int* pp = part + par * (G * S * R * MT);
      if (lane == 0) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int m = 0; m < MT; ++m) pp[((g * S + rd) * R + r) * MT + m] = tot[r][m];
      }
      __syncthreads();
      if (rd != 0) continue;
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m)
          for (int q = 1; q < S; ++q) tot[r][m] += pp[((g * S + q) * R + r) * MT + m];
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int64_t n = n0 + r;
        if (lane == r * MT + m && n < N && m < M) {
          const int v = tot[r][m] - asum[m];
          if (acc_out != nullptr) acc_out[static_cast<int64_t>(m) * N + n] = v;
          if (y != nullptr) {
            const float cs =
                __fmul_rn(__fmul_rn(gv_fused<AF>() ? s_scale[m] : ld_dep_f32(a_scale + m), unit_scale),
                        ld_dep_f32(alpha + n / alpha_group));
            const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn(__int2float_rn(v), cs));
            y[static_cast<int64_t>(m) * ldy + n] = *reinterpret_cast<const uint16_t*>(&b);
          }
        }
      }
  }
}

// ---------------------------------------------------------------------------
// gemv_mma_t2_kernel -- up to 8 tokens against 2-bit ternary weights (decode)
// on warp-level integer MMA (m16n8k32, u8 x s8 -> s32): weight rows are the
// MMA's 16 rows, the 8 token slots its 8 columns.  The MMA adds up 32 codes per
// row and token whatever order they come in, so each lane feeds it the offset
// codes c + 1 of the weight words it loaded itself (field j of a word, isolated
// with a shift and an AND as in gemv_t2_kernel) and the B fragment holds the
// activations of the same codes: the field-major activation words staged in
// shared memory are exactly that.  Lane (g, t) of a warp (g = lane / 4,
// t = lane % 4) loads 16 bytes (4 words, 64 codes) of rows g and g + 8 of the
// warp's 16-row tile per 256-code step, word 4t + c of the step; per word pair
// it issues two MMAs (fields 0, 1 and fields 2, 3).  The sums are of c + 1;
// each token's sum_k a_k is subtracted at the end.  CTAs are persistent and
// stage the activations once; K is split into 1024-code batches over S warps
// per tile whose partial sums meet in shared memory; every weight line a warp
// will read is prefetched into L2 before its wait.  With 16 token slots (NT)
// every weight fragment feeds two MMAs, one per 8 tokens.
// ---------------------------------------------------------------------------
constexpr int kGmTokens = 8;          // MMA columns: token slots of one MMA
constexpr int kGmBatchWords = 64;     // 16-code words per row and batch (4 steps of 16)

__device__ __forceinline__ void mma_u8s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int AF, int NT>
__global__ void __launch_bounds__(kGvMaxThreads) gemv_mma_t2_kernel(const uint8_t* __restrict__ a,
                                                                    const float* __restrict__ a_scale,
                                                                    const uint8_t* __restrict__ w,
                                                                    const float* __restrict__ alpha,
                                                                    int64_t alpha_group, int M, int N, int K, int S,
                                                                    int G, uint16_t* __restrict__ y, int64_t ldy,
                                                                    int32_t* __restrict__ acc_out, int64_t ldx,
                                                                    float eps) {
  extern __shared__ uint4 gm_smem[];
  static_assert(NT == 8 || NT == 16, "token slots");
  constexpr int kH = NT / kGmTokens;   // MMAs per weight fragment
  __shared__ int asum[NT];
  __shared__ float s_scale[NT];
  __shared__ double red[kGvMaxWarps][NT];
  const int kw16 = K >> 4;      // 16-code words per row (a multiple of 4)
  const int kq = kw16 >> 2;
  // activation word 4p + c of token m at (p * 4 + c) * 8 + m: the 32 lanes of
  // a B-fragment load hit 8 consecutive slots 4 times (no bank conflict)
  uint4* act = gm_smem;
  int4* part = reinterpret_cast<int4*>(act + static_cast<size_t>(kq) * 4 * NT);   // [2][G][S][kH][32]
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = warp / S;
  const int rd = warp - g * S;
  const int grp = lane >> 2;
  const int tig = lane & 3;
  const int64_t wrow_bytes = K >> 2;
  const int64_t tiles = (static_cast<int64_t>(N) + 15) >> 4;
  const int64_t tile_step = static_cast<int64_t>(gridDim.x) * G;
  const int batches = (kw16 + kGmBatchWords - 1) / kGmBatchWords;

  // every weight line this warp will read into L2 while the previous kernel
  // finishes: per tile and batch 16 rows x 256 bytes, one 128-byte line a lane
  for (int64_t tile = static_cast<int64_t>(blockIdx.x) * G + g; tile < tiles; tile += tile_step)
    for (int b = rd; b < batches; b += S) {
      const int64_t n = tile * 16 + (lane & 15);
      const int64_t off = static_cast<int64_t>(b) * (kGmBatchWords * 4) + (lane >> 4) * 128;
      if (n < N && off < wrow_bytes) prefetch_l2(w + n * wrow_bytes + off);
    }
  if (threadIdx.x < NT) asum[threadIdx.x] = 0;
  __syncthreads();
  pdl_wait();
  pdl_trigger();

  // stage the activations (zeros for token slots past M) and their sums
  gv_stage<AF, NT>(a, ldx, eps, M, K, act, [](int q, int m) { return ((q >> 2) * 4 + (q & 3)) * NT + m; }, asum,
                   red, s_scale);
  __syncthreads();
  const float unit_scale = (AF == kSimtA_E2M1 || AF == kGvX_Fp4) ? 0.5f : 1.0f;

  int par = 0;
  for (int64_t tb = static_cast<int64_t>(blockIdx.x) * G; tb < tiles; tb += tile_step, par ^= 1) {
    const int64_t tile = tb + g;
    const int64_t r0 = tile * 16 + grp;
    const int64_t r1 = r0 + 8;
    const bool ok0 = tile < tiles && r0 < N;
    const bool ok1 = tile < tiles && r1 < N;
    int c[kH][4] = {};
    for (int b = rd; b < batches; b += S) {
      // words 4 tig .. 4 tig + 3 of rows r0 and r1 in each of the batch's 4 steps
      uint4 w0[4], w1[4];
#pragma unroll
      for (int st = 0; st < 4; ++st) {
        const int q = b * kGmBatchWords + st * 16 + 4 * tig;
        const bool okq = q < kw16;
        w0[st] = ok0 && okq ? ld_global_nc_v4(w + r0 * wrow_bytes + static_cast<int64_t>(q) * 4) : make_uint4(0, 0, 0, 0);
        w1[st] = ok1 && okq ? ld_global_nc_v4(w + r1 * wrow_bytes + static_cast<int64_t>(q) * 4) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int st = 0; st < 4; ++st) {
        const uint32_t x0[4] = {w0[st].x, w0[st].y, w0[st].z, w0[st].w};
        const uint32_t x1[4] = {w1[st].x, w1[st].y, w1[st].z, w1[st].w};
        const int q = b * kGmBatchWords + st * 16 + 4 * tig;
        const bool okq = q < kw16;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const uint32_t p0 = ~x0[cc] & (0x55555555u | (x0[cc] << 1));
          const uint32_t p1 = ~x1[cc] & (0x55555555u | (x1[cc] << 1));
          const uint32_t f0 = p0 & 0x03030303u, f1 = p1 & 0x03030303u;
          const uint32_t f2 = (p0 >> 2) & 0x03030303u, f3 = (p1 >> 2) & 0x03030303u;
          const uint32_t f4 = (p0 >> 4) & 0x03030303u, f5 = (p1 >> 4) & 0x03030303u;
          const uint32_t f6 = (p0 >> 6) & 0x03030303u, f7 = (p1 >> 6) & 0x03030303u;
#pragma unroll
          for (int hh = 0; hh < kH; ++hh) {
            // words past K: zero activations (the weight side is then irrelevant)
            const uint4 bv = okq ? act[((q >> 2) * 4 + cc) * NT + hh * kGmTokens + grp] : make_uint4(0, 0, 0, 0);
            mma_u8s8_16832(c[hh], f0, f1, f2, f3, bv.x, bv.y);
            mma_u8s8_16832(c[hh], f4, f5, f6, f7, bv.z, bv.w);
          }
        }
      }
    }
    if (S > 1) {
      // batches of a tile meet in shared memory (two buffers, as in gemv_t2_kernel)
      int4* pp = part + static_cast<size_t>(par) * (G * S * kH * 32);
#pragma unroll
      for (int hh = 0; hh < kH; ++hh)
        pp[((g * S + rd) * kH + hh) * 32 + lane] = make_int4(c[hh][0], c[hh][1], c[hh][2], c[hh][3]);
      __syncthreads();
      if (rd != 0) continue;
      for (int q = 1; q < S; ++q)
#pragma unroll
        for (int hh = 0; hh < kH; ++hh) {
          const int4 o = pp[((g * S + q) * kH + hh) * 32 + lane];
          c[hh][0] += o.x;
          c[hh][1] += o.y;
          c[hh][2] += o.z;
          c[hh][3] += o.w;
        }
    }
    // lane (grp, tig) holds rows r0 (c0, c1) and r1 (c2, c3), tokens 8 hh + 2 tig and 8 hh + 2 tig + 1
#pragma unroll
    for (int e = 0; e < 4 * kH; ++e) {
      const int64_t n = (e & 3) < 2 ? r0 : r1;
      const int m = (e >> 2) * kGmTokens + 2 * tig + (e & 1);
      if (((e & 3) < 2 ? ok0 : ok1) && m < M) {
        const int v = c[e >> 2][e & 3] - asum[m];
        if (acc_out != nullptr) acc_out[static_cast<int64_t>(m) * N + n] = v;
        if (y != nullptr) {
          const float cs =
              __fmul_rn(__fmul_rn(gv_fused<AF>() ? s_scale[m] : ld_dep_f32(a_scale + m), unit_scale),
                        ld_dep_f32(alpha + n / alpha_group));
          const __nv_bfloat16 bb = __float2bfloat16_rn(__fmul_rn(__int2float_rn(v), cs));
          y[static_cast<int64_t>(m) * ldy + n] = *reinterpret_cast<const uint16_t*>(&bb);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// gemv_stream_t2_kernel -- 1 or 2 tokens against 2-bit ternary weights, the
// weights streamed.  One CTA per SM owns a contiguous run of whole 4-row
// groups, i.e. one contiguous byte range of the packed matrix.  Before its wait
// the CTA asks L2 for the whole range; after it, one thread moves the range
// through a ring of shared-memory stages (32 rows each) with 1-D bulk copies
// that complete on mbarriers, so the copy engine keeps the CTA's bytes in
// flight with no registers tied up.  Eight consumer warps take 4 rows of each
// stage and compute as gemv_t2_kernel does (offset codes, dp4a against the
// field-major activations staged once per CTA), reading the weights from
// shared memory.  Every wait is bounded.
// ---------------------------------------------------------------------------
constexpr int kGsConsumers = 8;                            // consumer warps; the last warp copies
constexpr int kGsThreads = (kGsConsumers + 1) * 32;
constexpr int kGsStageRows = kGsConsumers * 4;             // 32 rows per stage
constexpr int kGsMaxStages = 4;

template <int AF, int MT>
__global__ void __launch_bounds__(kGsThreads, 1) gemv_stream_t2_kernel(const uint8_t* __restrict__ a,
                                                                      const float* __restrict__ a_scale,
                                                                      const uint8_t* __restrict__ w,
                                                                      const float* __restrict__ alpha,
                                                                      int64_t alpha_group, int M, int N, int K,
                                                                      int stages, uint16_t* __restrict__ y,
                                                                      int64_t ldy, int32_t* __restrict__ acc_out) {
  constexpr int R = 4;
  extern __shared__ __align__(128) uint8_t gs_smem[];
  __shared__ __align__(8) uint64_t full[kGsMaxStages];
  __shared__ __align__(8) uint64_t empty[kGsMaxStages];
  __shared__ int asum[MT];
  __shared__ float s_scale[MT];
  __shared__ double red[kGvMaxWarps][MT];
  __shared__ int s_abort;
  const int kw16 = K >> 4;
  const int kq = kw16 >> 2;
  const uint32_t rowbytes = static_cast<uint32_t>(K >> 2);
  const uint32_t stage_bytes = kGsStageRows * rowbytes;
  uint8_t* ring = gs_smem;
  uint4* act = reinterpret_cast<uint4*>(gs_smem + static_cast<size_t>(stages) * stage_bytes);   // [MT][4][kq]
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const bool producer = warp == kGsConsumers;

  // this CTA's 4-row groups [g0, g1): rows [4 g0, min(4 g1, N)), contiguous bytes
  const int64_t groups = (static_cast<int64_t>(N) + 3) / 4;
  const int64_t g0 = groups * blockIdx.x / gridDim.x;
  const int64_t g1 = groups * (blockIdx.x + 1) / gridDim.x;
  const int64_t row0 = 4 * g0;
  const int64_t row_end = min(4 * g1, static_cast<int64_t>(N));
  const int nstage = static_cast<int>((g1 - g0 + kGsConsumers - 1) / kGsConsumers);
  auto stage_rows = [&](int i) {
    const int64_t r = row0 + static_cast<int64_t>(i) * kGsStageRows;
    return static_cast<uint32_t>(min(static_cast<int64_t>(kGsStageRows), row_end - r));
  };

  if (threadIdx.x == 0) {
    for (int st = 0; st < stages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kGsConsumers);
    }
    fence_mbarrier_init();
    s_abort = 0;
  }
  if (threadIdx.x < MT) asum[threadIdx.x] = 0;
  if (producer && lane == 0 && row_end > row0)
    bulk_prefetch_l2(w + row0 * rowbytes, static_cast<uint32_t>(row_end - row0) * rowbytes);
  __syncthreads();
  pdl_wait();
  pdl_trigger();

  // the first stages go out before the activations are staged
  if (producer && lane == 0) {
    for (int i = 0; i < nstage && i < stages; ++i) {
      const uint32_t bytes = stage_rows(i) * rowbytes;
      mbar_arrive_expect_tx(&full[i], bytes);
      bulk_load_1d(ring + static_cast<size_t>(i) * stage_bytes, w + (row0 + static_cast<int64_t>(i) * kGsStageRows) * rowbytes,
                   bytes, &full[i]);
    }
  }
  gv_stage<AF, MT>(a, 0, 0.f, M, K, act, [kq](int q, int m) { return (m * 4 + (q & 3)) * kq + (q >> 2); }, asum,
                   red, s_scale);
  __syncthreads();

  if (producer) {
    if (lane == 0) {
      for (int i = stages; i < nstage; ++i) {
        const int st = i % stages;
        if (!mbar_wait_bounded(&empty[st], static_cast<uint32_t>((i / stages - 1) & 1))) {
          s_abort = 1;
          break;
        }
        const uint32_t bytes = stage_rows(i) * rowbytes;
        mbar_arrive_expect_tx(&full[st], bytes);
        bulk_load_1d(ring + static_cast<size_t>(st) * stage_bytes, w + (row0 + static_cast<int64_t>(i) * kGsStageRows) * rowbytes,
                     bytes, &full[st]);
      }
    }
  } else {
    const float unit_scale = (AF == kSimtA_E2M1) ? 0.5f : 1.0f;
    const int rounds = (kw16 + 255) >> 8;
    for (int i = 0; i < nstage; ++i) {
      const int st = i % stages;
      if (!mbar_wait_bounded(&full[st], static_cast<uint32_t>((i / stages) & 1))) {
        s_abort = 1;
        break;
      }
      const int64_t n0 = row0 + static_cast<int64_t>(i) * kGsStageRows + warp * R;
      const bool rows_ok = n0 < row_end;
      const uint8_t* sw = ring + static_cast<size_t>(st) * stage_bytes + static_cast<size_t>(warp * R) * rowbytes;
      int tot[R][MT];
      if constexpr (MT == 1) {
        int acc[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[r][j] = 0;
        for (int rd = 0; rd < rounds; ++rd) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int wq = rd * 256 + h * 128 + 4 * lane;
            if (!rows_ok || wq >= kw16) continue;
            uint4 wv[R];
#pragma unroll
            for (int r = 0; r < R; ++r)
              wv[r] = n0 + r < row_end ? *reinterpret_cast<const uint4*>(sw + r * rowbytes + wq * 4)
                                       : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint4 av = act[j * kq + (wq >> 2)];
#pragma unroll
              for (int r = 0; r < R; ++r) {
                const uint32_t x = j == 0 ? wv[r].x : (j == 1 ? wv[r].y : (j == 2 ? wv[r].z : wv[r].w));
                const uint32_t u = ~x & (0x55555555u | (x << 1));
                acc[r][0] = dp4a_us(u & 0x03030303u, av.x, acc[r][0]);
                acc[r][1] = dp4a_us(u & 0x0C0C0C0Cu, av.y, acc[r][1]);
                acc[r][2] = dp4a_us(u & 0x30303030u, av.z, acc[r][2]);
                acc[r][3] = dp4a_us(u & 0xC0C0C0C0u, av.w, acc[r][3]);
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);   // this warp is done with the stage
#pragma unroll
        for (int r = 0; r < R; ++r)
          tot[r][0] =
              __reduce_add_sync(0xFFFFFFFFu, acc[r][0] + (acc[r][1] >> 2) + (acc[r][2] >> 4) + (acc[r][3] >> 6));
      } else {
        int acc[R][MT];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int m = 0; m < MT; ++m) acc[r][m] = 0;
        for (int rd = 0; rd < rounds; ++rd) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int wq = rd * 256 + h * 128 + 4 * lane;
            if (!rows_ok || wq >= kw16) continue;
            uint4 wv[R];
#pragma unroll
            for (int r = 0; r < R; ++r)
              wv[r] = n0 + r < row_end ? *reinterpret_cast<const uint4*>(sw + r * rowbytes + wq * 4)
                                       : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t f[R][4];
#pragma unroll
              for (int r = 0; r < R; ++r) {
                const uint32_t x = j == 0 ? wv[r].x : (j == 1 ? wv[r].y : (j == 2 ? wv[r].z : wv[r].w));
                const uint32_t u = ~x & (0x55555555u | (x << 1));
                f[r][0] = u & 0x03030303u;
                f[r][1] = (u >> 2) & 0x03030303u;
                f[r][2] = (u >> 4) & 0x03030303u;
                f[r][3] = (u >> 6) & 0x03030303u;
              }
#pragma unroll
              for (int m = 0; m < MT; ++m) {
                const uint4 av = act[(m * 4 + j) * kq + (wq >> 2)];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                  int t = dp4a_us(f[r][0], av.x, acc[r][m]);
                  t = dp4a_us(f[r][1], av.y, t);
                  t = dp4a_us(f[r][2], av.z, t);
                  acc[r][m] = dp4a_us(f[r][3], av.w, t);
                }
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int m = 0; m < MT; ++m) tot[r][m] = __reduce_add_sync(0xFFFFFFFFu, acc[r][m]);
      }
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int64_t n = n0 + r;
          if (lane == r * MT + m && n < row_end && m < M) {
            const int v = tot[r][m] - asum[m];
            if (acc_out != nullptr) acc_out[static_cast<int64_t>(m) * N + n] = v;
            if (y != nullptr) {
              const float cs =
                  __fmul_rn(__fmul_rn(ld_dep_f32(a_scale + m), unit_scale), ld_dep_f32(alpha + n / alpha_group));
              const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn(__int2float_rn(v), cs));
              y[static_cast<int64_t>(m) * ldy + n] = *reinterpret_cast<const uint16_t*>(&b);
            }
          }
        }
    }
  }
  __syncthreads();
  if (s_abort) {
    // let any copies still in flight land before the CTA's memory goes away
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) {
    }
  }
}

// ---------------------------------------------------------------------------
// gemv_gated_t2_kernel -- the conditional Up projection for 1 or 2 tokens
// (the FFN's Gate first, Up only where it matters).  W holds [W_up; W_gate]
// (F rows each, 2-bit).  A warp takes 4 channels n: it computes their Gate rows
// (F + n) exactly as gemv_t2_kernel does and writes y[:, F + n]; a channel is
// active when some token's bf16 gate output is > 0, and only then are its Up
// row's bytes loaded and y[:, n] computed -- elsewhere y[:, n] = +0 (and acc 0):
// ReLU^2 makes h = up * max(0, gate)^2 a zero there whatever up is, so the
// ReLU^2-GLU quantizer gives the same codes, mask and scale.  Rows of up to
// 4096 codes (one round per warp); persistent CTAs stage the activations once.
// ---------------------------------------------------------------------------
template <int AF, int MT>
__global__ void __launch_bounds__(256) gemv_gated_t2_kernel(const uint8_t* __restrict__ a,
                                                            const float* __restrict__ a_scale,
                                                            const uint8_t* __restrict__ w,
                                                            const float* __restrict__ alpha, int M, int F, int K,
                                                            uint16_t* __restrict__ y, int64_t ldy,
                                                            int32_t* __restrict__ acc_out) {
  constexpr int R = 4;
  extern __shared__ uint4 gg_smem[];
  __shared__ int asum[MT];
  __shared__ float s_scale[MT];
  __shared__ double red[kGvMaxWarps][MT];
  const int kw16 = K >> 4;                 // <= 256: one 4096-code round
  const int kq = kw16 >> 2;
  uint4* act = gg_smem;                    // [MT][4][kq]
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t wrow_bytes = K >> 2;
  const int64_t groups = (static_cast<int64_t>(F) + R - 1) / R;
  const int64_t group_step = static_cast<int64_t>(gridDim.x) * 8;
  const int64_t N2 = 2 * static_cast<int64_t>(F);

  // the Gate rows this warp will read go to L2 before the wait (the Up rows
  // are read only where the gate says so)
  if (lane < 8 * R) {
    const int r = lane >> 3;
    const int64_t b = (lane & 7) * 128;
    if (b < wrow_bytes)
      for (int64_t gi = static_cast<int64_t>(blockIdx.x) * 8 + warp; gi < groups; gi += group_step) {
        const int64_t n = gi * R + r;
        if (n < F) prefetch_l2(w + (F + n) * wrow_bytes + b);
      }
  }
  if (threadIdx.x < MT) asum[threadIdx.x] = 0;
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  gv_stage<AF, MT>(a, 0, 0.f, M, K, act, [kq](int q, int m) { return (m * 4 + (q & 3)) * kq + (q >> 2); }, asum,
                   red, s_scale);
  __syncthreads();
  const float unit_scale = (AF == kSimtA_E2M1) ? 0.5f : 1.0f;
  float sc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) sc[m] = m < M ? __fmul_rn(ld_dep_f32(a_scale + m), unit_scale) : 0.f;
  const float al_up = ld_dep_f32(alpha), al_gate = ld_dep_f32(alpha + 1);

  // one matrix row block: R rows starting at `row` (skipping rows whose bit in
  // `use` is clear), sums of (c + 1) a over this lane's codes, reduced over the warp
  auto row_sums = [&](int64_t row, int64_t nrows, uint32_t use, int (&tot)[R][MT]) {
    uint4 wv[R][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int wq = h * 128 + 4 * lane;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const bool ok = wq < kw16 && r < nrows && ((use >> r) & 1u);
        wv[r][h] = ok ? ld_global_nc_v4(w + (row + r) * wrow_bytes + static_cast<int64_t>(wq) * 4)
                      : make_uint4(0, 0, 0, 0);
      }
    }
    int acc[R][MT][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[r][m][j] = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int wq = h * 128 + 4 * lane;
      if (wq >= kw16) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint4 av[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) av[m] = act[(m * 4 + j) * kq + (wq >> 2)];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if (!((use >> r) & 1u)) continue;
          const uint32_t x = j == 0 ? wv[r][h].x : (j == 1 ? wv[r][h].y : (j == 2 ? wv[r][h].z : wv[r][h].w));
          const uint32_t u = ~x & (0x55555555u | (x << 1));
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            acc[r][m][0] = dp4a_us(u & 0x03030303u, av[m].x, acc[r][m][0]);
            acc[r][m][1] = dp4a_us(u & 0x0C0C0C0Cu, av[m].y, acc[r][m][1]);
            acc[r][m][2] = dp4a_us(u & 0x30303030u, av[m].z, acc[r][m][2]);
            acc[r][m][3] = dp4a_us(u & 0xC0C0C0C0u, av[m].w, acc[r][m][3]);
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m)
        tot[r][m] = __reduce_add_sync(0xFFFFFFFFu, acc[r][m][0] + (acc[r][m][1] >> 2) + (acc[r][m][2] >> 4) +
                                                       (acc[r][m][3] >> 6));
  };

  for (int64_t gb = static_cast<int64_t>(blockIdx.x) * 8; gb < groups; gb += group_step) {
    const int64_t n0 = (gb + warp) * R;
    if (n0 >= F) continue;   // warp-uniform; no barrier follows
    const int64_t nrows = min(static_cast<int64_t>(R), static_cast<int64_t>(F) - n0);
    // ---- Gate rows ----
    int tg[R][MT];
    row_sums(F + n0, nrows, 0xFu, tg);
    uint32_t pos = 0;   // lane r * MT + m: the gate output is > 0
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (lane == r * MT + m && r < nrows && m < M) {
          const int64_t n = F + n0 + r;
          const int v = tg[r][m] - asum[m];
          if (acc_out != nullptr) acc_out[static_cast<int64_t>(m) * N2 + n] = v;
          const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn(__int2float_rn(v), __fmul_rn(sc[m], al_gate)));
          const uint16_t bits = *reinterpret_cast<const uint16_t*>(&b);
          y[static_cast<int64_t>(m) * ldy + n] = bits;
          pos = (bits & 0x8000u) == 0u && bits != 0u;
        }
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, pos != 0u);
    uint32_t use = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) use |= (((bal >> (r * MT)) & ((1u << MT) - 1u)) != 0u ? 1u : 0u) << r;
    // ---- Up rows of the active channels ----
    int tu[R][MT];
    row_sums(n0, nrows, use, tu);
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (lane == r * MT + m && r < nrows && m < M) {
          const int64_t n = n0 + r;
          const bool on = (use >> r) & 1u;
          const int v = on ? tu[r][m] - asum[m] : 0;
          if (acc_out != nullptr) acc_out[static_cast<int64_t>(m) * N2 + n] = v;
          const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn(__int2float_rn(v), __fmul_rn(sc[m], al_up)));
          y[static_cast<int64_t>(m) * ldy + n] = on ? *reinterpret_cast<const uint16_t*>(&b) : uint16_t(0);
        }
  }
}

}  // namespace bl
