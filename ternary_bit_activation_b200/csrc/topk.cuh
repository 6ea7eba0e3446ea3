// Top-K + INT8 absmax quantization of token rows (BitNet a4.8, arXiv 2411.04965,
// §3.4, Eq. 1 with Q_INT8), for the raw bf16 inputs (sparsify_a8) and for the
// ReLU^2-GLU output h = up * max(0, gate)^2 in fp32 (Eq. 5, relu2_glu).
//
// One group of G warps handles one row; a 256-thread CTA holds 8/G groups that
// share nothing but the CTA.  The row is copied once from HBM into the group's
// shared memory (bf16 for sparsify, the fp32 h for relu2), so the selection
// passes read shared memory, registers stay few and many rows are in flight per
// SM.  Groups synchronize with their own named barrier (or a warp barrier).
//
// Selection: exactly `keep` survivors ranked by magnitude, ties to the lower
// index.  If at most `keep` magnitudes are nonzero the threshold is 0 (every
// nonzero survives, zeros fill the rest in index order).  Otherwise an MSD
// radix select over the nonzero keys finds the keep-th largest key; with fp32
// keys the candidates left after the first digit are compacted into a short
// list that the remaining passes read.
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kRowThreads = 256;          // threads per CTA
constexpr int kRowListCap = 1024;         // compacted candidates (fp32 keys)

template <bool F32>
struct RowTraits {
  static constexpr int kElemBytes = F32 ? 4 : 2;
  static constexpr int kPasses = F32 ? 4 : 2;
};

// Per-group shared state, followed in memory by the row values.
struct GroupSmem {
  uint32_t hist[256];
  uint32_t red[8];          // per-warp partials (max key / nonzero count / tie totals)
  uint32_t red2[8];
  uint32_t sel_digit, sel_above, sel_count, list_n;
  int32_t tie_tot[64];      // ties per (warp in group, chunk slot): [warp * slots + slot]; G * slots <= 64
};

template <int G>
__device__ __forceinline__ void group_sync(int gid) {
  if constexpr (G == 1) {
    __syncwarp();
  } else {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + gid), "r"(G * 32) : "memory");
  }
}

template <bool F32>
__device__ __forceinline__ void chunk_keys(const uint4* vals, uint32_t (&k)[8]) {
  if constexpr (F32) {
    const uint4 a = vals[0], b = vals[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) k[e] = w[e] & 0x7FFFFFFFu;
  } else {
    bf16x8_mag_keys(vals[0], k);
  }
}

template <bool F32>
__device__ __forceinline__ void chunk_values(const uint4* vals, float (&f)[8]) {
  if constexpr (F32) {
    const uint4 a = vals[0], b = vals[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(w[e]);
  } else {
    unpack_bf16x8(vals[0], f);
  }
}

// Within one warp: digit d with above(d) < r <= above(d) + hist[d], counting
// from the top (above(d) = candidates with a larger digit); zeroes the
// histogram.  Lane l owns bins l, l+32, ... (conflict-free).
__device__ __forceinline__ void warp_select_digit(uint32_t* hist, int nbins, uint32_t r, GroupSmem& gs) {
  const int lane = threadIdx.x & 31;
  const int slots = nbins / 32;
  uint32_t h[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = 0;
    if (i < slots) {
      h[i] = hist[32 * i + lane];
      hist[32 * i + lane] = 0;
    }
  }
  uint32_t above_slots = 0;
#pragma unroll
  for (int i = 7; i >= 0; --i) {
    if (i >= slots) continue;
    uint32_t inc = h[i];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t other = __shfl_down_sync(0xFFFFFFFFu, inc, o);
      if (lane + o < 32) inc += other;
    }
    const uint32_t above = above_slots + inc - h[i];
    if (above < r && r <= above + h[i]) {
      gs.sel_digit = static_cast<uint32_t>(32 * i + lane);
      gs.sel_above = above;
      gs.sel_count = h[i];
    }
    above_slots += __shfl_sync(0xFFFFFFFFu, inc, 0);
  }
}

// G warps per row.  RELU2: values are h computed from gate/up; otherwise the
// bf16 input row.  Chunk q (8 consecutive values) of a row belongs to thread
// q % (32G); the row lives in shared memory as chunk-major 16-byte words.
template <int G, bool RELU2>
__global__ void __launch_bounds__(kRowThreads) topk_rows_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ up, int64_t M, int K, int64_t ldx, int keep,
    float eps, int8_t* __restrict__ codes, float* __restrict__ scale, uint32_t* __restrict__ mask,
    int row_words /* 16-byte words of one row's values in shared memory */) {
  constexpr bool F32 = RELU2;
  constexpr int GT = G * 32;
  constexpr int kWpc = F32 ? 2 : 1;                    // 16-byte words per chunk
  constexpr int kGroups = kRowThreads / GT;
  extern __shared__ uint4 dyn[];
  const int gid = threadIdx.x / GT;
  const int tid = threadIdx.x % GT;
  const int lane = threadIdx.x & 31;
  const int wig = tid >> 5;                            // warp in group
  GroupSmem* gsm = reinterpret_cast<GroupSmem*>(dyn);
  GroupSmem& gs = gsm[gid];
  uint4* vals = reinterpret_cast<uint4*>(gsm + kGroups) + static_cast<int64_t>(gid) * row_words;
  uint32_t* list = reinterpret_cast<uint32_t*>(reinterpret_cast<uint4*>(gsm + kGroups) +
                                               static_cast<int64_t>(kGroups) * row_words) +
                   gid * kRowListCap;

  const int nchunk = K >> 3;
  const int my_chunks = (nchunk - tid + GT - 1) / GT;   // chunks q = tid + c*GT, c < my_chunks

  for (int i = tid; i < 256; i += GT) gs.hist[i] = 0;

  for (int64_t row = static_cast<int64_t>(blockIdx.x) * kGroups + gid; row < M;
       row += static_cast<int64_t>(gridDim.x) * kGroups) {
    // ---- copy the row into shared memory; max key and nonzero count ----
    uint32_t mk = 0, nz = 0;
    {
      const uint16_t* xr = x + row * ldx;
      const uint16_t* ur = RELU2 ? up + row * ldx : nullptr;
#pragma unroll 4
      for (int c = 0; c < my_chunks; ++c) {
        const int q = tid + c * GT;
        if constexpr (RELU2) {
          const uint4 gv = ld_global_nc_v4(xr + static_cast<int64_t>(q) * 8);
          const uint4 uv = ld_global_nc_v4(ur + static_cast<int64_t>(q) * 8);
          float g[8], u[8];
          unpack_bf16x8(gv, g);
          unpack_bf16x8(uv, u);
          uint32_t hb[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float rg = g[e] > 0.f ? g[e] : 0.f;
            hb[e] = __float_as_uint(__fmul_rn(u[e], __fmul_rn(rg, rg)));
            const uint32_t key = hb[e] & 0x7FFFFFFFu;
            mk = max(mk, key);
            nz += key != 0u;
          }
          vals[q * 2] = make_uint4(hb[0], hb[1], hb[2], hb[3]);
          vals[q * 2 + 1] = make_uint4(hb[4], hb[5], hb[6], hb[7]);
        } else {
          const uint4 v = ld_global_nc_v4(xr + static_cast<int64_t>(q) * 8);
          uint32_t k[8];
          bf16x8_mag_keys(v, k);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            mk = max(mk, k[e]);
            nz += k[e] != 0u;
          }
          vals[q] = v;
        }
      }
    }
    mk = __reduce_max_sync(0xFFFFFFFFu, mk);
    nz = __reduce_add_sync(0xFFFFFFFFu, nz);
    if (lane == 0) {
      gs.red[wig] = mk;
      gs.red2[wig] = nz;
    }
    if (tid == 0) gs.list_n = 0;
    group_sync<G>(gid);
    uint32_t gk = 0, nnz = 0;
#pragma unroll
    for (int w = 0; w < G; ++w) {
      gk = max(gk, gs.red[w]);
      nnz += gs.red2[w];
    }

    // ---- threshold key `thr`; `take` elements equal to it survive ----
    uint32_t thr, take, tie_total;
    if (nnz <= static_cast<uint32_t>(keep)) {
      thr = 0;
      take = static_cast<uint32_t>(keep) - nnz;
      tie_total = static_cast<uint32_t>(K) - nnz;
    } else {
      uint32_t prefix = 0, fixed = 0, r = static_cast<uint32_t>(keep);
      bool listed = false;
      tie_total = 0;
#pragma unroll 1
      for (int pass = 0; pass < RowTraits<F32>::kPasses; ++pass) {
        const int shift = F32 ? max(23 - 8 * pass, 0) : 7 - 7 * pass;
        const int width = shift == 0 ? 7 : 8;
        const uint32_t dmask = (1u << width) - 1u;
        if (listed) {
          const int n = static_cast<int>(gs.list_n);
          for (int i = tid; i < n; i += GT) {
            const uint32_t key = list[i];
            if ((key & fixed) == prefix) atomicAdd(&gs.hist[(key >> shift) & dmask], 1u);
          }
        } else {
#pragma unroll 2
          for (int c = 0; c < my_chunks; ++c) {
            uint32_t k[8];
            chunk_keys<F32>(vals + (tid + c * GT) * kWpc, k);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if (k[e] != 0u && (k[e] & fixed) == prefix) atomicAdd(&gs.hist[(k[e] >> shift) & dmask], 1u);
          }
        }
        group_sync<G>(gid);
        if (wig == 0) warp_select_digit(gs.hist, 1 << width, r, gs);
        group_sync<G>(gid);
        r -= gs.sel_above;
        tie_total = gs.sel_count;
        prefix |= gs.sel_digit << shift;
        fixed |= dmask << shift;
        if (F32 && pass == 0 && tie_total <= static_cast<uint32_t>(kRowListCap)) {
          // candidates left after the top digit -> list (read by the remaining passes)
#pragma unroll 2
          for (int c = 0; c < my_chunks; ++c) {
            uint32_t k[8];
            chunk_keys<F32>(vals + (tid + c * GT) * kWpc, k);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if (k[e] != 0u && (k[e] & fixed) == prefix) list[atomicAdd(&gs.list_n, 1u)] = k[e];
          }
          group_sync<G>(gid);
          listed = true;
        }
      }
      thr = prefix;
      take = r;
    }
    // Ranks among the ties are needed only when some are dropped -- and not when
    // the tied key is 0 without a mask: a kept zero and a dropped one both get code 0.
    const bool partial = take < tie_total && (thr != 0u || mask != nullptr);

    // ---- codes and mask; ties at the threshold ranked in index order ----
    // chunk q = tid + c*GT, so index order is slot c first, then thread.  When
    // some ties are dropped, pass A publishes each warp's tie count per slot;
    // pass B re-scans its lanes to rank them.
    const float gamma = F32 ? __uint_as_float(gk) : __uint_as_float(gk << 16);
    const float mult = __fdiv_rn(127.f, __fadd_rn(gamma, eps));
    if (tid == 0) scale[row] = __fdiv_rn(gamma, 127.f);
    const int slots = (nchunk + GT - 1) / GT;
    const int mwords = (K + 31) >> 5;
    if (partial) {
#pragma unroll 1
      for (int c = 0; c < slots; ++c) {
        int cnt = 0;
        if (c < my_chunks) {
          uint32_t k[8];
          chunk_keys<F32>(vals + (tid + c * GT) * kWpc, k);
#pragma unroll
          for (int e = 0; e < 8; ++e) cnt += k[e] == thr;
        }
        cnt = __reduce_add_sync(0xFFFFFFFFu, cnt);
        if (lane == 0) gs.tie_tot[wig * slots + c] = cnt;
      }
      group_sync<G>(gid);
    }
    int slot_base = 0;   // ties in earlier slots, all threads of the group
#pragma unroll 1
    for (int c = 0; c < slots; ++c) {
      const int q = tid + c * GT;
      const bool ok = c < my_chunks;
      uint32_t k[8];
      float f[8];
      if (ok) {
        chunk_keys<F32>(vals + q * kWpc, k);
        chunk_values<F32>(vals + q * kWpc, f);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          k[e] = 0;
          f[e] = 0.f;
        }
      }
      int rank = 0;
      if (partial) {
        int cnt = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) cnt += ok && k[e] == thr;
        int inc = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int other = __shfl_up_sync(0xFFFFFFFFu, inc, o);
          if (lane >= o) inc += other;
        }
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < G; ++w) {
          const int tw = gs.tie_tot[w * slots + c];
          before += w < wig ? tw : 0;
          total += tw;
        }
        rank = slot_base + before + inc - cnt;
        slot_base += total;
      }
      uint32_t bits = 0;
      uint2 w2 = make_uint2(0, 0);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        bool keepit = k[e] > thr;
        if (k[e] == thr) {
          keepit = !partial || rank < static_cast<int>(take);
          ++rank;
        }
        keepit = keepit && ok;
        const int code = keepit ? round_clip(__fmul_rn(f[e], mult), -128.f, 127.f) : 0;
        bits |= (keepit ? 1u : 0u) << e;
        const uint32_t b = static_cast<uint32_t>(code) & 0xFFu;
        if (e < 4) w2.x |= b << (8 * e); else w2.y |= b << (8 * (e - 4));
      }
      if (ok) reinterpret_cast<uint2*>(codes + row * static_cast<int64_t>(K))[q] = w2;
      if (mask != nullptr) {
        // chunks q..q+3 (lanes 4i..4i+3 of one slot) form one 32-bit mask word
        const uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, bits, 1);
        const uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, bits, 2);
        const uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, bits, 3);
        if (ok && (lane & 3) == 0) mask[row * mwords + (q >> 2)] = bits | (b1 << 8) | (b2 << 16) | (b3 << 24);
      }
    }
    group_sync<G>(gid);   // the row buffer and group state are reused by the next row
  }
}

}  // namespace bl
