// libbitlinear: C ABI over the sm_100a kernels of the BitNet a4.8 BitLinear
// forward path (arXiv 2411.04965, §3.4).  One translation unit: the kernels
// live in the headers included below; this file validates arguments, encodes
// TMA descriptors and launches.  The declarations and their contracts are in
// include/bitlinear.h.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>
#ifndef BITLINEAR_NO_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

#include "bitlinear.h"
#include "attn.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "kv.cuh"
#include "pack.cuh"
#include "quant.cuh"
#include "topk.cuh"

namespace {

static_assert(int{BL_QUANT_INT4} == bl::kQInt4 && int{BL_QUANT_FP4_E2M1} == bl::kQFp4 &&
                  int{BL_QUANT_INT4_ABSMAX} == bl::kQInt4Absmax &&
                  int{BL_QUANT_INT4_ABSMEAN2} == bl::kQInt4Absmean2 && int{BL_QUANT_FP4_E1M2} == bl::kQFp4E1M2,
              "bl_quant values are the quantizer kernel's variant ids");

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An NVTX range named after the entry point around every call that enqueues
// work, so that a profiler groups each call's kernels under its name.  Without a
// tool attached the push and pop are no-ops; -DBITLINEAR_NO_NVTX compiles them out.
class NvtxRange {
 public:
  explicit NvtxRange(const char* name) {
#ifndef BITLINEAR_NO_NVTX
    nvtxRangePushA(name);
#else
    (void)name;
#endif
  }
  ~NvtxRange() {
#ifndef BITLINEAR_NO_NVTX
    nvtxRangePop();
#endif
  }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// The last CUDA runtime error that made an entry point of this thread return
// BL_ERR_CUDA (bitlinear_last_cuda_error reports its name).
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

// true on success; a failure is recorded for bitlinear_last_cuda_error
bool cuda_ok(cudaError_t e) {
  if (e == cudaSuccess) return true;
  t_last_cuda_error = e;
  return false;
}

// The error of the last launch_pdl call of this thread that failed and has not
// yet been reported by launch_status.
thread_local cudaError_t t_launch_error = cudaSuccess;

bl_status launch_status() {
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = t_launch_error;
  t_launch_error = cudaSuccess;
  return cuda_ok(e) ? BL_OK : BL_ERR_CUDA;
}

// Launch with programmatic stream serialization (see pdl_wait / pdl_trigger):
// the kernel may start while the previous kernel of the stream finishes.
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  if (e != cudaSuccess) t_launch_error = e;
}

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}

int sm_count() {
  static int cached[kMaxDevices] = {0};
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 148;
  if (cached[d] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
    cached[d] = n;
  }
  return cached[d];
}

// ---------------------------------------------------------------------------
// TMA descriptors through the driver entry point (no link-time libcuda).
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2-D int8 tensor [rows x cols] (cols contiguous), box of box_cols x box_rows, 128B swizzle.
bool make_i8_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                 uint32_t box_cols) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Unswizzled map over a row-major byte matrix viewed in 8-byte elements
// (cols_bytes % 16 == 0); a box row carries box_bytes of one matrix row.
bool make_u64_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols_bytes, uint32_t box_rows,
                  uint32_t box_bytes) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols_bytes / 8, rows};
  const cuuint64_t strides[1] = {cols_bytes};
  const cuuint32_t box[2] = {box_bytes / 8, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tc_kernel_ready() {
  static bool done[kMaxDevices] = {false};
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return false;
  if (!done[d]) {
    if (!cuda_ok(cudaFuncSetAttribute(bl::gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(bl::kTcSmemBytes))))
      return false;
    if (!cuda_ok(cudaFuncSetAttribute(bl::gemm_tc2_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(bl::kT2SmemBytes))) ||
        !cuda_ok(cudaFuncSetAttribute(bl::gemm_tc2_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(bl::kF4SmemBytes))))
      return false;
    if (!cuda_ok(cudaFuncSetAttribute(bl::gemm_t2tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      227 * 1024)) ||
        !cuda_ok(cudaFuncSetAttribute(bl::gemm_t2tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      227 * 1024)) ||
        !cuda_ok(cudaFuncSetAttribute(bl::gemm_t2tc_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      227 * 1024)))
      return false;
    done[d] = true;
  }
  return true;
}

// ---------------------------------------------------------------------------
// launch helpers
// ---------------------------------------------------------------------------
// The optional parts of a quantizer launch: the RMSNorm prologue (gnorm may be
// NULL for a unit weight) and the tensor-wide beta of kQInt4Tensor.
struct QuantExtra {
  bool norm = false;
  const float* gnorm = nullptr;
  float eps_n = 0.f;
  const float* beta = nullptr;
};

template <int C, int VAR>
void launch_quant_a4_cv(const uint16_t* x, int64_t M, int K, int64_t ldx, bool packed, float eps, uint8_t* codes,
                        float* scale, cudaStream_t s, dim3 grid, const QuantExtra& q) {
  auto go = [&](auto kern) { launch_pdl(kern, grid, 256, 0, s, x, M, K, ldx, eps, codes, scale, q.gnorm, q.eps_n, q.beta); };
  if (q.norm) {
    if (packed) go(bl::quant_a4_kernel<C, VAR, true, true>);
    else go(bl::quant_a4_kernel<C, VAR, false, true>);
  } else {
    if (packed) go(bl::quant_a4_kernel<C, VAR, true, false>);
    else go(bl::quant_a4_kernel<C, VAR, false, false>);
  }
}

template <int C>
void launch_quant_a4_c(const uint16_t* x, int64_t M, int K, int64_t ldx, int var, bool packed, float eps,
                       uint8_t* codes, float* scale, cudaStream_t s, const QuantExtra& q) {
  // persistent: two rows per CTA and iteration, eight CTAs per SM
  const int64_t need = (M + 1) / 2;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const dim3 grid(static_cast<unsigned>(need < cap ? need : cap));
  switch (var) {
    case bl::kQInt4: launch_quant_a4_cv<C, bl::kQInt4>(x, M, K, ldx, packed, eps, codes, scale, s, grid, q); break;
    case bl::kQFp4: launch_quant_a4_cv<C, bl::kQFp4>(x, M, K, ldx, packed, eps, codes, scale, s, grid, q); break;
    case bl::kQInt4Absmax:
      launch_quant_a4_cv<C, bl::kQInt4Absmax>(x, M, K, ldx, packed, eps, codes, scale, s, grid, q);
      break;
    case bl::kQInt4Absmean2:
      launch_quant_a4_cv<C, bl::kQInt4Absmean2>(x, M, K, ldx, packed, eps, codes, scale, s, grid, q);
      break;
    case bl::kQInt4Tensor:
      launch_quant_a4_cv<C, bl::kQInt4Tensor>(x, M, K, ldx, packed, eps, codes, scale, s, grid, q);
      break;
    default: launch_quant_a4_cv<C, bl::kQFp4E1M2>(x, M, K, ldx, packed, eps, codes, scale, s, grid, q); break;
  }
}

// The quantizer launch for rows of K values (chunks of 8 per thread and row).
void launch_quant_a4(const uint16_t* x, int64_t M, int K, int64_t ldx, int var, bool packed, float eps,
                     uint8_t* codes, float* scale, cudaStream_t s, const QuantExtra& q) {
  const int64_t c = (K / 8 + bl::kQ4ThreadsPerRow - 1) / bl::kQ4ThreadsPerRow;
  if (c <= 1) launch_quant_a4_c<1>(x, M, K, ldx, var, packed, eps, codes, scale, s, q);
  else if (c <= 2) launch_quant_a4_c<2>(x, M, K, ldx, var, packed, eps, codes, scale, s, q);
  else if (c <= 4) launch_quant_a4_c<4>(x, M, K, ldx, var, packed, eps, codes, scale, s, q);
  else if (c <= 8) launch_quant_a4_c<8>(x, M, K, ldx, var, packed, eps, codes, scale, s, q);
  else launch_quant_a4_c<16>(x, M, K, ldx, var, packed, eps, codes, scale, s, q);
}

// Top-K rows: one 256-thread CTA per row, persistent grid sized by the occupancy
// that the shared-memory row stages allow.
template <bool RELU2>
bl_status launch_topk_rows(const uint16_t* x, const uint16_t* up, int64_t M, int K, int64_t ldx, int keep,
                           float eps, int8_t* codes, float* scale, uint32_t* mask, cudaStream_t s) {
  const size_t smem = bl::tk_smem_bytes<RELU2>(K);
  if (smem > 227 * 1024) return BL_ERR_SHAPE;
  auto kern = bl::topk_rows_kernel<RELU2>;
  static size_t attr_set[kMaxDevices] = {};
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return BL_ERR_CUDA;
  if (smem > attr_set[d]) {
    if (!cuda_ok(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))))
      return BL_ERR_CUDA;
    attr_set[d] = smem;
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, bl::kTkThreads, smem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm;
  const unsigned grid = static_cast<unsigned>(M < cap ? M : cap);
  launch_pdl(kern, grid, bl::kTkThreads, smem, s, x, up, M, K, ldx, keep, eps, codes, scale, mask);
  return launch_status();
}

// Top-K rows of up to 4096 bf16 values: one warp per row (persistent, four warps
// per CTA, as many CTAs as are resident); C = 16-byte chunks per lane.
template <int C>
bl_status launch_topk_warp_c(const uint16_t* x, int64_t M, int K, int64_t ldx, int keep, float eps, int8_t* codes,
                             float* scale, uint32_t* mask, cudaStream_t s) {
  auto kern = bl::topk_warp_kernel<C>;
  constexpr size_t smem = bl::tw_smem_bytes<C>();
  static int per_sm[kMaxDevices] = {};
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return BL_ERR_CUDA;
  if (per_sm[d] == 0) {
    if (!cuda_ok(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))))
      return BL_ERR_CUDA;
    int n = 0;
    if (!cuda_ok(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 32 * bl::kTwWarps, smem))) return BL_ERR_CUDA;
    per_sm[d] = n < 1 ? 1 : n;
  }
  const int64_t need = (M + bl::kTwWarps - 1) / bl::kTwWarps;
  const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm[d];
  const unsigned grid = static_cast<unsigned>(need < cap ? need : cap);
  launch_pdl(kern, grid, 32 * bl::kTwWarps, smem, s, x, M, K, ldx, keep, eps, codes, scale, mask);
  return launch_status();
}

bl_status launch_topk_warp(const uint16_t* x, int64_t M, int K, int64_t ldx, int keep, float eps, int8_t* codes,
                           float* scale, uint32_t* mask, cudaStream_t s) {
  const int per_lane = (K / 8 + 31) / 32;
  if (per_lane <= 1) return launch_topk_warp_c<1>(x, M, K, ldx, keep, eps, codes, scale, mask, s);
  if (per_lane <= 2) return launch_topk_warp_c<2>(x, M, K, ldx, keep, eps, codes, scale, mask, s);
  if (per_lane <= 4) return launch_topk_warp_c<4>(x, M, K, ldx, keep, eps, codes, scale, mask, s);
  if (per_lane <= 8) return launch_topk_warp_c<8>(x, M, K, ldx, keep, eps, codes, scale, mask, s);
  return launch_topk_warp_c<16>(x, M, K, ldx, keep, eps, codes, scale, mask, s);
}

template <int AF, bool WT2, int MT, int UPL>
bool launch_simt_mu(const uint8_t* a, const float* sc, const uint8_t* w, const float* al, int64_t g, int M, int N,
                    int K, uint16_t* y, int64_t ldy, int32_t* acc, cudaStream_t s) {
  constexpr int R = bl::SimtShape<WT2, UPL>::R;
  const int units_hi = ((K >> 6) + 31) >> 5;
  const size_t smem = static_cast<size_t>(MT) * units_hi * 32 * 16 * sizeof(uint32_t);
  auto kern = bl::gemm_simt_kernel<AF, WT2, MT, UPL>;
  // Raise the kernel's dynamic shared-memory limit to what this tile needs (once
  // per size and device).  The default limit counts static shared memory too, and
  // the kernel holds a 1 KiB static table, so a 48 KiB tile already needs it.
  static size_t attr_set[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return false;
  if (smem > attr_set[dev]) {
    if (!cuda_ok(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))))
      return false;
    attr_set[dev] = smem;
  }
  const int64_t warps_needed = (static_cast<int64_t>(N) + R - 1) / R;
  const int64_t blocks_needed = (warps_needed + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const unsigned grid = static_cast<unsigned>(blocks_needed < cap ? blocks_needed : cap);
  launch_pdl(kern, grid, 256, smem, s, a, sc, w, al, g, M, N, K, y, ldy, acc);
  return true;
}

// Units per lane per round (UPL, a power of two up to 8 for 2-bit weights and
// up to 2 for int8 weights): enough to cover K in one round where possible.
template <int AF, bool WT2, int MT>
bool launch_simt_m(const uint8_t* a, const float* sc, const uint8_t* w, const float* al, int64_t g, int M, int N,
                   int K, uint16_t* y, int64_t ldy, int32_t* acc, cudaStream_t s) {
  const int per_lane = ((K >> 6) + 31) >> 5;
  if (per_lane <= 1) return launch_simt_mu<AF, WT2, MT, 1>(a, sc, w, al, g, M, N, K, y, ldy, acc, s);
  if (per_lane <= 2 || !WT2) return launch_simt_mu<AF, WT2, MT, 2>(a, sc, w, al, g, M, N, K, y, ldy, acc, s);
  if (per_lane <= 4) return launch_simt_mu<AF, WT2, MT, 4>(a, sc, w, al, g, M, N, K, y, ldy, acc, s);
  return launch_simt_mu<AF, WT2, MT, 8>(a, sc, w, al, g, M, N, K, y, ldy, acc, s);
}

// Rows of A per staged tile (MT): up to 8 tokens share each streamed weight
// unit, fewer where MT rows of K codes would not fit in shared memory (the
// kernel walks the rows of A in tiles of MT).
constexpr size_t kSimtMaxSmem = 192 * 1024;
constexpr int64_t kSimtMaxK = 196608;   // one row of A per tile still fits

template <int AF, bool WT2>
bool launch_simt(const uint8_t* a, const float* sc, const uint8_t* w, const float* al, int64_t g, int M, int N,
                 int K, uint16_t* y, int64_t ldy, int32_t* acc, cudaStream_t s) {
  const size_t row_bytes = static_cast<size_t>(((K >> 6) + 31) >> 5) * 32 * 16 * sizeof(uint32_t);
  int mt = M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : 8));
  while (mt > 1 && static_cast<size_t>(mt) * row_bytes > kSimtMaxSmem) mt >>= 1;
  if (mt == 1) return launch_simt_m<AF, WT2, 1>(a, sc, w, al, g, M, N, K, y, ldy, acc, s);
  if (mt == 2) return launch_simt_m<AF, WT2, 2>(a, sc, w, al, g, M, N, K, y, ldy, acc, s);
  if (mt == 4) return launch_simt_m<AF, WT2, 4>(a, sc, w, al, g, M, N, K, y, ldy, acc, s);
  return launch_simt_m<AF, WT2, 8>(a, sc, w, al, g, M, N, K, y, ldy, acc, s);
}

// CTAs of the exact-sum kernel resident per SM: its grid is one wave, so every
// CTA streams to the end and flushes its bins once.
int bins_ctas_per_sm() {
  static int per_sm[kMaxDevices] = {};
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 4;
  if (per_sm[d] == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, bl::ternary_bins_kernel<false>, bl::kBinThreads, 0) != cudaSuccess ||
        n < 1)
      n = 1;
    per_sm[d] = n;
  }
  return per_sm[d];
}

// Scratch of pack_ternary_noalloc: the exponent bins of the exact |W| sum, one
// array per device that loads the library.  Host code only ever uses the device
// address looked up below, never the symbol itself.
static __device__ __align__(256) unsigned long long g_noalloc_bins[bl::kBins];
constexpr int64_t kNoallocMaxElems = bl::kMaxPackElems;  // keeps every 64-bit bin below overflow

// Device address of g_noalloc_bins on the current device, looked up once per
// device (with that device current) and cached.  The cache outlives the
// device's primary context: after a cudaDeviceReset the address is stale (the
// header says so).
unsigned long long* noalloc_bins_ptr() {
  static unsigned long long* cached[kMaxDevices] = {nullptr};
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return nullptr;
  if (cached[d] == nullptr) {
    void* p = nullptr;
    if (!cuda_ok(cudaGetSymbolAddress(&p, g_noalloc_bins))) return nullptr;
    cached[d] = static_cast<unsigned long long*>(p);
  }
  return cached[d];
}

// GEMV for up to kGvMaxTokens tokens against 2-bit weights: token slots per
// launch, and the limits that keep the staged activations in shared memory.
constexpr int kGvMaxTokens = 8;
constexpr int64_t kGvMaxK = 65536;                  // 16 rounds of 4096 codes: 512 threads
constexpr int64_t kGvMaxActBytes = 144 * 1024;      // token slots x K int8 activations
constexpr int kGvSmemLimit = 144 * 1024 + 8192;     // + round partial sums (two buffers)

int64_t gv_tokens(int m) { return m <= 1 ? 1 : (m <= 2 ? 2 : (m <= 4 ? 4 : 8)); }

template <int AF, int MT>
bl_status launch_gemv_mt(const uint8_t* A, const float* a_scale, const uint8_t* W, const float* alpha,
                         int64_t alpha_group, int m, int n, int k, uint16_t* Y, int64_t ldy, int32_t* acc_out,
                         cudaStream_t s, int64_t ldx, float eps) {
  static bool attr_done[kMaxDevices] = {};
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return BL_ERR_CUDA;
  if (!attr_done[d]) {
    if (!cuda_ok(cudaFuncSetAttribute(bl::gemv_t2_kernel<AF, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kGvSmemLimit)))
      return BL_ERR_CUDA;
    attr_done[d] = true;
  }
  constexpr int R = bl::GvShape<MT>::R;
  const int S = (k / 16 + 255) / 256;   // 4096-code rounds of a row, one warp each
  const int G = S >= 8 ? 1 : 8 / S;     // row groups per CTA and pass
  const int threads = 32 * G * S;
  const int64_t groups = (static_cast<int64_t>(n) + R - 1) / R;
  const size_t smem =
      static_cast<size_t>(MT) * static_cast<size_t>(k) + 2 * static_cast<size_t>(G * S * R * MT) * sizeof(int);
  // persistent CTAs: as many as are resident at once, at most one pass each
  int per_sm = 0;
  if (!cuda_ok(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, bl::gemv_t2_kernel<AF, MT>, threads, smem)))
    return BL_ERR_CUDA;
  if (per_sm < 1) per_sm = 1;
  const int64_t passes = (groups + G - 1) / G;
  const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm;
  const unsigned grid = static_cast<unsigned>(passes < cap ? passes : cap);
  launch_pdl(bl::gemv_t2_kernel<AF, MT>, grid, threads, smem, s, A, a_scale, W, alpha, alpha_group, m, n, k, S, G,
             Y, ldy, acc_out, ldx, eps);
  return launch_status();
}

// Warp-MMA GEMV: 8 or 16 token slots (NT) staged, so NT x K activation bytes.
// One or two tokens run faster on the dp4a GEMV (the MMA's 8 columns mostly
// idle); beyond 16 tokens the tcgen05 decode kernel takes over.
constexpr int64_t kGmMinTokens = 3;
constexpr int64_t kGmMaxTokens = 16;
constexpr int64_t kGmActBytes = 176 * 1024;
constexpr int kGmSmemLimit = 176 * 1024 + 32768;    // + batch partial sums (two buffers)

int64_t gm_slots(int64_t m) { return m <= 8 ? 8 : 16; }
bool gm_applies(int64_t M, int64_t K) {
  return M >= kGmMinTokens && M <= kGmMaxTokens && gm_slots(M) * K <= kGmActBytes;
}

template <int AF, int NT>
bl_status launch_gemv_mma(const uint8_t* A, const float* a_scale, const uint8_t* W, const float* alpha,
                          int64_t alpha_group, int m, int n, int k, uint16_t* Y, int64_t ldy, int32_t* acc_out,
                          cudaStream_t s, int64_t ldx = 0, float eps = 0.f) {
  static bool attr_done[kMaxDevices] = {};
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return BL_ERR_CUDA;
  if (!attr_done[d]) {
    if (!cuda_ok(cudaFuncSetAttribute(bl::gemv_mma_t2_kernel<AF, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kGmSmemLimit)))
      return BL_ERR_CUDA;
    attr_done[d] = true;
  }
  const int batches = (k / 16 + bl::kGmBatchWords - 1) / bl::kGmBatchWords;   // 1024-code batches of a row
  const int S = batches < 16 ? batches : 16;                                  // warps per 16-row tile
  const int G = S >= 8 ? 1 : 8 / S;                                           // tiles per CTA and pass
  const int threads = 32 * G * S;
  const int64_t tiles = (static_cast<int64_t>(n) + 15) / 16;
  const size_t smem = static_cast<size_t>(NT) * static_cast<size_t>(k) +
                      2 * static_cast<size_t>(G * S * (NT / 8) * 32) * sizeof(int4);
  int per_sm = 0;
  if (!cuda_ok(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, bl::gemv_mma_t2_kernel<AF, NT>, threads, smem)))
    return BL_ERR_CUDA;
  if (per_sm < 1) per_sm = 1;
  const int64_t passes = (tiles + G - 1) / G;
  const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm;
  const unsigned grid = static_cast<unsigned>(passes < cap ? passes : cap);
  launch_pdl(bl::gemv_mma_t2_kernel<AF, NT>, grid, threads, smem, s, A, a_scale, W, alpha, alpha_group, m, n, k, S, G,
             Y, ldy, acc_out, ldx, eps);
  return launch_status();
}

template <int AF>
bl_status launch_gemv(const uint8_t* A, const float* a_scale, const uint8_t* W, const float* alpha,
                      int64_t alpha_group, int m, int n, int k, uint16_t* Y, int64_t ldy, int32_t* acc_out,
                      cudaStream_t s, int64_t ldx = 0, float eps = 0.f) {
  switch (gv_tokens(m)) {
    case 1: return launch_gemv_mt<AF, 1>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s, ldx, eps);
    case 2: return launch_gemv_mt<AF, 2>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s, ldx, eps);
    case 4: return launch_gemv_mt<AF, 4>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s, ldx, eps);
    default: return launch_gemv_mt<AF, 8>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s, ldx, eps);
  }
}

// Streaming GEMV (1-2 tokens): one CTA per SM, at least two 32-row stages of
// K / 4 bytes per row in its shared-memory ring next to the staged activations.
constexpr size_t kGsSmemBudget = 200 * 1024;

int gs_stages(int64_t M, int64_t K) {
  const int64_t stage = 32 * (K / 4);
  const int64_t st = (static_cast<int64_t>(kGsSmemBudget) - M * K) / stage;
  return static_cast<int>(st > bl::kGsMaxStages ? bl::kGsMaxStages : st);
}
// Measured: it beats the dp4a GEMV when every CTA's rows fit one stage (the
// 7B O and Down shapes); with several stages per CTA the dp4a GEMV's 24 warps
// per SM win, so it is used only then.
bool gs_applies(int64_t M, int64_t N, int64_t K) {
  const int64_t groups_per_cta = ((N + 3) / 4 + sm_count() - 1) / sm_count();
  return M >= 1 && M <= 2 && gs_stages(M, K) >= 2 && groups_per_cta <= bl::kGsConsumers;
}

template <int AF, int MT>
bl_status launch_gemv_stream(const uint8_t* A, const float* a_scale, const uint8_t* W, const float* alpha,
                             int64_t alpha_group, int m, int n, int k, uint16_t* Y, int64_t ldy, int32_t* acc_out,
                             cudaStream_t s) {
  static size_t attr_set[kMaxDevices] = {};
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return BL_ERR_CUDA;
  const int stages = gs_stages(MT, k);
  const size_t smem = static_cast<size_t>(stages) * 32 * static_cast<size_t>(k / 4) + static_cast<size_t>(MT) * k;
  if (smem > attr_set[d]) {
    if (!cuda_ok(cudaFuncSetAttribute(bl::gemv_stream_t2_kernel<AF, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(smem))))
      return BL_ERR_CUDA;
    attr_set[d] = smem;
  }
  const int64_t groups = (static_cast<int64_t>(n) + 3) / 4;
  const int64_t sms = sm_count();
  const unsigned grid = static_cast<unsigned>(groups < sms ? groups : sms);
  launch_pdl(bl::gemv_stream_t2_kernel<AF, MT>, grid, bl::kGsThreads, smem, s, A, a_scale, W, alpha, alpha_group, m, n,
             k, stages, Y, ldy, acc_out);
  return launch_status();
}

// The decode GEMVs apply to 2-bit weights and up to max_tokens tokens (16; 8
// when they quantize bf16 rows themselves): the warp-MMA kernel from 3 tokens,
// the dp4a kernel otherwise (and for rows too long to stage 8 or 16 slots).
bool gemv_applies(int64_t M, int64_t K, int64_t max_tokens) {
  if (M < 1 || M > max_tokens) return false;
  if (gm_applies(M, K)) return true;
  return M <= kGvMaxTokens && K <= kGvMaxK && gv_tokens(static_cast<int>(M)) * K <= kGvMaxActBytes;
}

template <int AF>
bl_status launch_gemv_any(const uint8_t* A, const float* a_scale, const uint8_t* W, const float* alpha,
                          int64_t alpha_group, int m, int n, int k, uint16_t* Y, int64_t ldy, int32_t* acc_out,
                          cudaStream_t s, int64_t ldx = 0, float eps = 0.f) {
  if constexpr (!bl::gv_fused<AF>()) {
    if (gs_applies(m, n, k)) {
      if (m == 1) return launch_gemv_stream<AF, 1>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s);
      return launch_gemv_stream<AF, 2>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s);
    }
  }
  if (gm_applies(m, k)) {
    if (m <= 8) return launch_gemv_mma<AF, 8>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s, ldx, eps);
    if constexpr (!bl::gv_fused<AF>())
      return launch_gemv_mma<AF, 16>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s, ldx, eps);
  }
  return launch_gemv<AF>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s, ldx, eps);
}

// bitlinear_quant_gemm quantizes inside the decode GEMV for at most this many
// tokens.  Measured on 7B decode shapes: the fused layer is ~1 us faster at 1-2
// tokens, but 15-21 us slower at 4-8 (every CTA repeats the quantization, while
// the separate quantizer already overlaps the GEMV's weight prefetch), so from 3
// tokens the call runs the quantizer and the GEMM separately.
constexpr int64_t kQgFusedMaxTokens = 2;

// Workspace of bitlinear_quant_gemm when it runs as two kernels: M x K int8
// codes, then M fp32 scales, each 16-byte aligned.
int64_t qg_codes_bytes(int64_t M, int64_t K) { return (M * K + 15) / 16 * 16; }
int64_t qg_workspace_bytes(int64_t M, int64_t K) { return qg_codes_bytes(M, K) + (4 * M + 15) / 16 * 16; }

// ---------------------------------------------------------------------------
// Low-bit attention: position chunks spread over one resident wave of CTAs
// ---------------------------------------------------------------------------
size_t attn_workspace_bytes(int64_t M, int64_t H, int64_t D) {
  return static_cast<size_t>(bl::kAttnMaxChunks) * static_cast<size_t>(M) * static_cast<size_t>(H) *
         static_cast<size_t>(D + 4) * sizeof(float);
}

template <int D, int BITS, int HG, bool ONE>
bl_status launch_attention_hg(bl::AttnParams a, int group, cudaStream_t s) {
  auto kern = bl::attn_partial_kernel<D, BITS, HG, ONE>;
  const int ngroups = (a.M + group - 1) / group;
  const int nheadgroups = a.H / HG;
  const size_t smem = bl::AttnSmem<D, BITS, HG>(group).total;
  // per device: the largest shared-memory size set so far, and the occupancy of the last size asked for
  static int smem_set[kMaxDevices] = {};
  static size_t occ_smem[kMaxDevices] = {};
  static int occ_val[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return BL_ERR_CUDA;
  if (static_cast<int>(smem) > smem_set[dev]) {
    if (!cuda_ok(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))))
      return BL_ERR_CUDA;
    smem_set[dev] = static_cast<int>(smem);
  }
  if (occ_smem[dev] != smem || occ_val[dev] == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, bl::kAttnThreads, smem) != cudaSuccess || n < 1) n = 1;
    occ_smem[dev] = smem;
    occ_val[dev] = n;
  }
  // one resident wave of CTAs over (chunks, head groups, query groups); chunks are whole blocks
  constexpr int kPos = bl::AttnSmem<D, BITS, HG>::kPos;
  constexpr int kVB = bl::AttnShape<D, BITS>::kVecBytes;
  CUtensorMap tk, tv, tks, tvs;
  const uint64_t rows = static_cast<uint64_t>(a.T);
  if (!make_u64_map(&tk, a.k, rows, static_cast<uint64_t>(a.H) * kVB, kPos, HG * kVB) ||
      !make_u64_map(&tv, a.v, rows, static_cast<uint64_t>(a.H) * kVB, kPos, HG * kVB) ||
      !make_u64_map(&tks, a.ks, rows, static_cast<uint64_t>(a.H) * 4, kPos, HG * 4) ||
      !make_u64_map(&tvs, a.vs, rows, static_cast<uint64_t>(a.H) * 4, kPos, HG * 4))
    return BL_ERR_CUDA;
  int64_t target = static_cast<int64_t>(sm_count()) * occ_val[dev] / (static_cast<int64_t>(ngroups) * nheadgroups);
  if (target < 1) target = 1;
  if (target > bl::kAttnMaxChunks) target = bl::kAttnMaxChunks;
  int64_t chunk = (a.T + target - 1) / target;
  chunk = (chunk + kPos - 1) / kPos * kPos;
  a.group = group;
  a.chunk = static_cast<int>(chunk);
  a.nchunks = static_cast<int>((a.T + chunk - 1) / chunk);
  launch_pdl(kern, dim3(static_cast<unsigned>(a.nchunks), static_cast<unsigned>(nheadgroups),
                        static_cast<unsigned>(ngroups)),
             bl::kAttnThreads, smem, s, tk, tv, tks, tvs, a);
  if (launch_status() != BL_OK) return BL_ERR_CUDA;
  launch_pdl(bl::attn_combine_kernel<D, BITS>,
             dim3(static_cast<unsigned>(a.H), static_cast<unsigned>(a.M), static_cast<unsigned>(D / 32)),
             bl::kAttnThreads, 0, s, a);
  return launch_status();
}

template <int D, int BITS, int HG>
bl_status launch_attention_g(const bl::AttnParams& a, cudaStream_t s) {
  int group = bl::kAttnThreads / (HG * (D / 32));
  if (group > bl::kAttnMaxGroup) group = bl::kAttnMaxGroup;
  if (group > a.M) group = a.M;
  return group == 1 ? launch_attention_hg<D, BITS, HG, true>(a, 1, s)
                    : launch_attention_hg<D, BITS, HG, false>(a, group, s);
}

template <int D, int BITS>
bl_status launch_attention(const bl::AttnParams& a, cudaStream_t s) {
  return (a.H % 8 == 0) ? launch_attention_g<D, BITS, 8>(a, s) : launch_attention_g<D, BITS, 4>(a, s);
}

}  // namespace

extern "C" {

bl_status pack_ternary_noalloc(const float* w, int64_t N, int64_t K, int64_t ldw, float eps, int alpha_given,
                               float* alpha, bl_wfmt wfmt, void* w_out, void* stream) {
  NvtxRange nvtx_range("pack_ternary_noalloc");
  if (wfmt != BL_W_T2 && wfmt != BL_W_I8 && wfmt != BL_W_E2M1) return BL_ERR_ARG;
  if (N < 0 || K < 16 || (K & 15) || ldw < K || (ldw & 3) || K > 0x7FFFFFFF) return BL_ERR_SHAPE;
  // N * K >= limit, tested without forming the product (which can overflow)
  if (N > 0 && N >= (kNoallocMaxElems + K - 1) / K) return BL_ERR_SHAPE;
  if (!(eps >= 0.f)) return BL_ERR_ARG;
  if (N == 0) return BL_OK;
  if (w == nullptr || alpha == nullptr || w_out == nullptr) return BL_ERR_NULL;
  if (!aligned16(w) || !aligned16(w_out) || (reinterpret_cast<uintptr_t>(alpha) & 3u)) return BL_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  const int k = static_cast<int>(K);
  if (!alpha_given) {
    unsigned long long* bins = noalloc_bins_ptr();
    if (bins == nullptr) return BL_ERR_CUDA;
    if (!cuda_ok(cudaMemsetAsync(bins, 0, sizeof(g_noalloc_bins), s))) return BL_ERR_CUDA;
    const int64_t total = N * (K / 4);
    int64_t blocks = (total + bl::kBinThreads - 1) / bl::kBinThreads;
    const int64_t cap = static_cast<int64_t>(sm_count()) * bins_ctas_per_sm();   // one resident wave
    if (blocks > cap) blocks = cap;
    launch_pdl(bl::ternary_bins_kernel<false>, static_cast<unsigned>(blocks), bl::kBinThreads, 0, s,
               static_cast<const void*>(w), N, k, ldw, bins, alpha);
    if (launch_status() != BL_OK) return BL_ERR_CUDA;
  }
  const int64_t total16 = N * (K / 16);
  int64_t blocks = (total16 + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  if (blocks > cap) blocks = cap;
  uint8_t* out = static_cast<uint8_t*>(w_out);
  if (wfmt == BL_W_T2)
    launch_pdl(bl::ternary_pack_kernel<BL_W_T2>, static_cast<unsigned>(blocks), 256, 0, s, w, N, k, ldw, alpha, eps, out);
  else if (wfmt == BL_W_E2M1)
    launch_pdl(bl::ternary_pack_kernel<BL_W_E2M1>, static_cast<unsigned>(blocks), 256, 0, s, w, N, k, ldw, alpha, eps, out);
  else
    launch_pdl(bl::ternary_pack_kernel<BL_W_I8>, static_cast<unsigned>(blocks), 256, 0, s, w, N, k, ldw, alpha, eps, out);
  return launch_status();
}

const char* bitlinear_last_cuda_error(void) { return cudaGetErrorName(t_last_cuda_error); }

const char* bitlinear_version(void) { return "libbitlinear 0.1 (sm_100a)"; }

const char* bitlinear_status_string(bl_status st) {
  switch (st) {
    case BL_OK: return "BL_OK";
    case BL_ERR_NULL: return "BL_ERR_NULL";
    case BL_ERR_ALIGN: return "BL_ERR_ALIGN";
    case BL_ERR_SHAPE: return "BL_ERR_SHAPE";
    case BL_ERR_ARG: return "BL_ERR_ARG";
    case BL_ERR_UNSUPPORTED: return "BL_ERR_UNSUPPORTED";
    case BL_ERR_CUDA: return "BL_ERR_CUDA";
    case BL_ERR_TIMEOUT: return "BL_ERR_TIMEOUT";
    case BL_ERR_WORKSPACE: return "BL_ERR_WORKSPACE";
  }
  return "BL_UNKNOWN";
}

size_t bitlinear_workspace_size(const char* op, int64_t M, int64_t N, int64_t K) {
  if (op != nullptr && (strcmp(op, "pack_ternary") == 0 || strcmp(op, "quant_a4_per_tensor") == 0))
    return bl::kBins * sizeof(unsigned long long);
  if (op != nullptr && strcmp(op, "quant_gemm") == 0 && M > 0 && K > 0)
    return static_cast<size_t>(qg_workspace_bytes(M, K));
  if (op != nullptr && strcmp(op, "attention_lowbit") == 0 && M > 0 && N > 0 && K > 0)
    return attn_workspace_bytes(M, N, K);
  return 0;
}

bl_status bitlinear_sync_status(void* stream) {
  if (!cuda_ok(cudaStreamSynchronize(as_stream(stream)))) return BL_ERR_CUDA;
  int v = 0;
  if (!cuda_ok(cudaMemcpyFromSymbol(&v, bl::g_status, sizeof(int)))) return BL_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (!cuda_ok(cudaMemcpyToSymbol(bl::g_status, &zero, sizeof(int)))) return BL_ERR_CUDA;
    return static_cast<bl_status>(v);
  }
  return BL_OK;
}

bl_status bitlinear_selftest_timeout(void* stream) {
  bl::bounded_wait_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>();
  return launch_status();
}

bl_status bitlinear_quant_a4(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, bl_quant quant, bl_store store,
                             float eps, void* codes, float* scale, void* stream) {
  NvtxRange nvtx_range("bitlinear_quant_a4");
  if (quant != BL_QUANT_INT4 && quant != BL_QUANT_FP4_E2M1 && quant != BL_QUANT_INT4_ABSMAX &&
      quant != BL_QUANT_INT4_ABSMEAN2 && quant != BL_QUANT_FP4_E1M2)
    return BL_ERR_ARG;
  if (store != BL_STORE_PACKED && store != BL_STORE_BYTES) return BL_ERR_ARG;
  if (M < 0 || K < 8 || K > 16384 || (K & 7) || ldx < K || (ldx & 7) || M > 0x7FFFFFFELL) return BL_ERR_SHAPE;
  if (M == 0) return BL_OK;
  if (x_bf16 == nullptr || codes == nullptr || scale == nullptr) return BL_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scale)) return BL_ERR_ALIGN;
  if (!(eps >= 0.f)) return BL_ERR_ARG;
  const int var = static_cast<int>(quant);   // bl_quant values are the kernel's variant ids
  launch_quant_a4(static_cast<const uint16_t*>(x_bf16), M, static_cast<int>(K), ldx, var, store == BL_STORE_PACKED,
                  eps, static_cast<uint8_t*>(codes), scale, as_stream(stream), QuantExtra());
  return launch_status();
}

bl_status bitlinear_rmsnorm_quant_a4(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, const float* gamma,
                                     float eps_norm, bl_quant quant, bl_store store, float eps, void* codes,
                                     float* scale, void* stream) {
  NvtxRange nvtx_range("bitlinear_rmsnorm_quant_a4");
  if (quant != BL_QUANT_INT4 && quant != BL_QUANT_FP4_E2M1 && quant != BL_QUANT_INT4_ABSMAX &&
      quant != BL_QUANT_INT4_ABSMEAN2 && quant != BL_QUANT_FP4_E1M2)
    return BL_ERR_ARG;
  if (store != BL_STORE_PACKED && store != BL_STORE_BYTES) return BL_ERR_ARG;
  if (M < 0 || K < 8 || K > 16384 || (K & 7) || ldx < K || (ldx & 7) || M > 0x7FFFFFFELL) return BL_ERR_SHAPE;
  if (!(eps >= 0.f) || !(eps_norm > 0.f) || !(eps_norm < 3.4e38f)) return BL_ERR_ARG;
  if (M == 0) return BL_OK;
  if (x_bf16 == nullptr || codes == nullptr || scale == nullptr) return BL_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scale) || (gamma && !aligned16(gamma)))
    return BL_ERR_ALIGN;
  QuantExtra q;
  q.norm = true;
  q.gnorm = gamma;
  q.eps_n = eps_norm;
  launch_quant_a4(static_cast<const uint16_t*>(x_bf16), M, static_cast<int>(K), ldx, static_cast<int>(quant),
                  store == BL_STORE_PACKED, eps, static_cast<uint8_t*>(codes), scale, as_stream(stream), q);
  return launch_status();
}

bl_status bitlinear_quant_a4_per_tensor(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, bl_store store,
                                        float eps, void* codes, float* scale, float* beta, void* workspace,
                                        size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("bitlinear_quant_a4_per_tensor");
  if (store != BL_STORE_PACKED && store != BL_STORE_BYTES) return BL_ERR_ARG;
  if (M < 0 || K < 8 || K > 16384 || (K & 7) || ldx < K || (ldx & 7)) return BL_ERR_SHAPE;
  // M * K >= limit, tested without forming the product
  if (M > 0 && M >= (bl::kMaxPackElems + K - 1) / K) return BL_ERR_SHAPE;
  if (!(eps >= 0.f)) return BL_ERR_ARG;
  if (M == 0) return BL_OK;
  if (x_bf16 == nullptr || codes == nullptr || scale == nullptr || beta == nullptr || workspace == nullptr)
    return BL_ERR_NULL;
  if (ws_bytes < bl::kBins * sizeof(unsigned long long)) return BL_ERR_WORKSPACE;
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scale) || (reinterpret_cast<uintptr_t>(beta) & 3u) ||
      (reinterpret_cast<uintptr_t>(workspace) & 7u))
    return BL_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  unsigned long long* bins = static_cast<unsigned long long*>(workspace);
  if (!cuda_ok(cudaMemsetAsync(bins, 0, bl::kBins * sizeof(unsigned long long), s))) return BL_ERR_CUDA;
  // the exact mean of |x| over the tensor (the bins kernel of pack_ternary on bf16 values)
  const int64_t total = M * (K / 8);
  int64_t blocks = (total + bl::kBinThreads - 1) / bl::kBinThreads;
  const int64_t cap = static_cast<int64_t>(sm_count()) * bins_ctas_per_sm();
  if (blocks > cap) blocks = cap;
  launch_pdl(bl::ternary_bins_kernel<true>, static_cast<unsigned>(blocks), bl::kBinThreads, 0, s, x_bf16, M,
             static_cast<int>(K), ldx, bins, beta);
  if (launch_status() != BL_OK) return BL_ERR_CUDA;
  QuantExtra q;
  q.beta = beta;
  launch_quant_a4(static_cast<const uint16_t*>(x_bf16), M, static_cast<int>(K), ldx, bl::kQInt4Tensor,
                  store == BL_STORE_PACKED, eps, static_cast<uint8_t*>(codes), scale, s, q);
  return launch_status();
}

bl_status bitlinear_sparsify_a8(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, int64_t k_keep, float eps,
                                int8_t* codes, float* scale, uint32_t* mask, void* stream) {
  NvtxRange nvtx_range("bitlinear_sparsify_a8");
  if (M < 0 || K < 8 || K > 16384 || (K & 7) || ldx < K || (ldx & 7) || M > 0x7FFFFFFFLL) return BL_ERR_SHAPE;
  if (k_keep < 1 || k_keep > K) return BL_ERR_ARG;
  if (!(eps >= 0.f)) return BL_ERR_ARG;
  if (M == 0) return BL_OK;
  if (x_bf16 == nullptr || codes == nullptr || scale == nullptr) return BL_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scale) || (mask && !aligned16(mask))) return BL_ERR_ALIGN;
  if (K <= bl::kTwMaxK)
    return launch_topk_warp(static_cast<const uint16_t*>(x_bf16), M, static_cast<int>(K), ldx, static_cast<int>(k_keep),
                            eps, codes, scale, mask, as_stream(stream));
  return launch_topk_rows<false>(static_cast<const uint16_t*>(x_bf16), nullptr, M, static_cast<int>(K), ldx,
                                 static_cast<int>(k_keep), eps, codes, scale, mask, as_stream(stream));
}

bl_status relu2_glu(const void* gate_bf16, const void* up_bf16, int64_t M, int64_t F, int64_t ld, int64_t k_keep,
                    float eps, int8_t* codes, float* scale, uint32_t* mask, void* stream) {
  NvtxRange nvtx_range("relu2_glu");
  if (M < 0 || F < 8 || F > 16384 || (F & 7) || ld < F || (ld & 7) || M > 0x7FFFFFFFLL) return BL_ERR_SHAPE;
  if (k_keep < 1 || k_keep > F) return BL_ERR_ARG;
  if (!(eps >= 0.f)) return BL_ERR_ARG;
  if (M == 0) return BL_OK;
  if (gate_bf16 == nullptr || up_bf16 == nullptr || codes == nullptr || scale == nullptr) return BL_ERR_NULL;
  if (!aligned16(gate_bf16) || !aligned16(up_bf16) || !aligned16(codes) || !aligned16(scale) ||
      (mask && !aligned16(mask)))
    return BL_ERR_ALIGN;
  // gate and up share the row stride ld; the kernel reads gate through x
  return launch_topk_rows<true>(static_cast<const uint16_t*>(gate_bf16), static_cast<const uint16_t*>(up_bf16), M,
                                static_cast<int>(F), ld, static_cast<int>(k_keep), eps, codes, scale, mask,
                                as_stream(stream));
}

bl_status pack_ternary(const float* w, int64_t N, int64_t K, int64_t ldw, float eps, int alpha_given, float* alpha,
                       bl_wfmt wfmt, void* w_out, void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("pack_ternary");
  if (wfmt != BL_W_T2 && wfmt != BL_W_I8 && wfmt != BL_W_E2M1) return BL_ERR_ARG;
  if (N < 0 || K < 16 || (K & 15) || ldw < K || (ldw & 3) || K > 0x7FFFFFFF) return BL_ERR_SHAPE;
  // N * K >= limit, tested without forming the product (which can overflow)
  if (N > 0 && N >= (bl::kMaxPackElems + K - 1) / K) return BL_ERR_SHAPE;
  if (!(eps >= 0.f)) return BL_ERR_ARG;
  if (N == 0) return BL_OK;
  if (w == nullptr || alpha == nullptr || w_out == nullptr) return BL_ERR_NULL;
  if (!aligned16(w) || !aligned16(w_out) || (reinterpret_cast<uintptr_t>(alpha) & 3u)) return BL_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  const int k = static_cast<int>(K);
  if (!alpha_given) {
    if (workspace == nullptr) return BL_ERR_NULL;
    if (ws_bytes < bl::kBins * sizeof(unsigned long long)) return BL_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 7u) return BL_ERR_ALIGN;
    unsigned long long* bins = static_cast<unsigned long long*>(workspace);
    if (!cuda_ok(cudaMemsetAsync(bins, 0, bl::kBins * sizeof(unsigned long long), s))) return BL_ERR_CUDA;
    const int64_t total = N * (K / 4);
    int64_t blocks = (total + bl::kBinThreads - 1) / bl::kBinThreads;
    const int64_t cap = static_cast<int64_t>(sm_count()) * bins_ctas_per_sm();   // one resident wave
    if (blocks > cap) blocks = cap;
    launch_pdl(bl::ternary_bins_kernel<false>, static_cast<unsigned>(blocks), bl::kBinThreads, 0, s,
               static_cast<const void*>(w), N, k, ldw, bins, alpha);
    if (launch_status() != BL_OK) return BL_ERR_CUDA;
  }
  const int64_t total16 = N * (K / 16);
  int64_t blocks = (total16 + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  if (blocks > cap) blocks = cap;
  uint8_t* out = static_cast<uint8_t*>(w_out);
  if (wfmt == BL_W_T2)
    launch_pdl(bl::ternary_pack_kernel<BL_W_T2>, static_cast<unsigned>(blocks), 256, 0, s, w, N, k, ldw, alpha, eps, out);
  else if (wfmt == BL_W_E2M1)
    launch_pdl(bl::ternary_pack_kernel<BL_W_E2M1>, static_cast<unsigned>(blocks), 256, 0, s, w, N, k, ldw, alpha, eps, out);
  else
    launch_pdl(bl::ternary_pack_kernel<BL_W_I8>, static_cast<unsigned>(blocks), 256, 0, s, w, N, k, ldw, alpha, eps, out);
  return launch_status();
}

bl_status bitlinear_gemm(const void* a, bl_afmt afmt, const float* a_scale, const void* w, bl_wfmt wfmt,
                         const float* alpha, int64_t alpha_group, int64_t M, int64_t N, int64_t K, void* y_bf16,
                         int64_t ldy, int32_t* acc_out, void* stream) {
  NvtxRange nvtx_range("bitlinear_gemm");
  if (afmt != BL_A_I8 && afmt != BL_A_I4 && afmt != BL_A_E2M1) return BL_ERR_ARG;
  if (wfmt != BL_W_T2 && wfmt != BL_W_I8 && wfmt != BL_W_E2M1) return BL_ERR_ARG;
  if (alpha_group < 1 || alpha_group > 0x7FFFFFFFLL) return BL_ERR_ARG;
  if (M < 0 || N < 1 || K < 64 || (K & 63) || K > (1 << 20) || M > 0x7FFFFFFFLL || N > 0x7FFFFFFFLL)
    return BL_ERR_SHAPE;
  if (y_bf16 != nullptr && (ldy < N || (ldy & 7))) return BL_ERR_SHAPE;
  if (M == 0) return BL_OK;
  if (a == nullptr || a_scale == nullptr || w == nullptr || alpha == nullptr) return BL_ERR_NULL;
  if (y_bf16 == nullptr && acc_out == nullptr) return BL_ERR_NULL;
  if (!aligned16(a) || !aligned16(w) || (y_bf16 && !aligned16(y_bf16)) || (acc_out && !aligned16(acc_out)) ||
      (reinterpret_cast<uintptr_t>(a_scale) & 3u) || (reinterpret_cast<uintptr_t>(alpha) & 3u))
    return BL_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  const uint8_t* A = static_cast<const uint8_t*>(a);
  const uint8_t* W = static_cast<const uint8_t*>(w);
  uint16_t* Y = static_cast<uint16_t*>(y_bf16);

  if (wfmt == BL_W_E2M1) {
    // FP4 x FP4-coded ternary on the tensor cores (kind::mxf4, CTA pairs)
    if (afmt != BL_A_E2M1) return BL_ERR_ARG;
    if (!tc_kernel_ready()) return BL_ERR_CUDA;
    CUtensorMap ta, tb;
    if (!make_i8_map(&ta, A, static_cast<uint64_t>(M), static_cast<uint64_t>(K / 2), 128, bl::kTcBK) ||
        !make_i8_map(&tb, W, static_cast<uint64_t>(N), static_cast<uint64_t>(K / 2), bl::kF4BN / 2, bl::kTcBK))
      return BL_ERR_CUDA;
    bl::TcParams p;
    p.a_scale = a_scale;
    p.alpha = alpha;
    p.alpha_group = alpha_group;
    p.M = m;
    p.N = n;
    p.K = k;
    p.y = Y;
    p.ldy = ldy;
    p.acc = acc_out;
    p.num_m_blocks = (m + bl::kT2BM - 1) / bl::kT2BM;
    p.num_n_blocks = (n + bl::kF4BN - 1) / bl::kF4BN;
    p.num_tiles = p.num_m_blocks * p.num_n_blocks;
    p.num_kb = (k / 2 + bl::kTcBK - 1) / bl::kTcBK;
    const int pairs = p.num_tiles < sm_count() / 2 ? p.num_tiles : sm_count() / 2;
    launch_pdl(bl::gemm_tc2_kernel<true>, 2 * pairs, bl::kT2Threads, bl::kF4SmemBytes, s, ta, tb, p);
    return launch_status();
  }
  if (afmt == BL_A_I8 && wfmt == BL_W_I8 && M > bl::kTcBM) {
    // CTA-pair kernel: 256 x 256 tiles over clusters of two CTAs
    if (!tc_kernel_ready()) return BL_ERR_CUDA;
    CUtensorMap ta, tb;
    if (!make_i8_map(&ta, A, static_cast<uint64_t>(M), static_cast<uint64_t>(K), 128, bl::kTcBK) ||
        !make_i8_map(&tb, W, static_cast<uint64_t>(N), static_cast<uint64_t>(K), 128, bl::kTcBK))
      return BL_ERR_CUDA;
    bl::TcParams p;
    p.a_scale = a_scale;
    p.alpha = alpha;
    p.alpha_group = alpha_group;
    p.M = m;
    p.N = n;
    p.K = k;
    p.y = Y;
    p.ldy = ldy;
    p.acc = acc_out;
    p.num_m_blocks = (m + bl::kT2BM - 1) / bl::kT2BM;
    p.num_n_blocks = (n + bl::kT2BN - 1) / bl::kT2BN;
    p.num_tiles = p.num_m_blocks * p.num_n_blocks;
    p.num_kb = (k + bl::kTcBK - 1) / bl::kTcBK;
    const int pairs = p.num_tiles < sm_count() / 2 ? p.num_tiles : sm_count() / 2;
    launch_pdl(bl::gemm_tc2_kernel<false>, 2 * pairs, bl::kT2Threads, bl::kT2SmemBytes, s, ta, tb, p);
    return launch_status();
  }
  if (afmt == BL_A_I8 && wfmt == BL_W_I8) {
    if (!tc_kernel_ready()) return BL_ERR_CUDA;
    CUtensorMap ta, tb;
    if (!make_i8_map(&ta, A, static_cast<uint64_t>(M), static_cast<uint64_t>(K), bl::kTcBM, bl::kTcBK) ||
        !make_i8_map(&tb, W, static_cast<uint64_t>(N), static_cast<uint64_t>(K), bl::kTcBN, bl::kTcBK))
      return BL_ERR_CUDA;
    bl::TcParams p;
    p.a_scale = a_scale;
    p.alpha = alpha;
    p.alpha_group = alpha_group;
    p.M = m;
    p.N = n;
    p.K = k;
    p.y = Y;
    p.ldy = ldy;
    p.acc = acc_out;
    p.num_m_blocks = (m + bl::kTcBM - 1) / bl::kTcBM;
    p.num_n_blocks = (n + bl::kTcBN - 1) / bl::kTcBN;
    p.num_tiles = p.num_m_blocks * p.num_n_blocks;
    p.num_kb = (k + bl::kTcBK - 1) / bl::kTcBK;
    const int grid = p.num_tiles < sm_count() ? p.num_tiles : sm_count();
    launch_pdl(bl::gemm_tc_kernel, grid, bl::kTcThreads, bl::kTcSmemBytes, s, ta, tb, p);
    return launch_status();
  }
  if (wfmt == BL_W_T2 && gemv_applies(M, K, kGmMaxTokens)) {
    // up to 16 tokens: one pass over the 2-bit weights (warp-MMA from 3 tokens, else dp4a)
    if (afmt == BL_A_I8) return launch_gemv_any<bl::kSimtA_I8>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s);
    if (afmt == BL_A_I4) return launch_gemv_any<bl::kSimtA_I4>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s);
    return launch_gemv_any<bl::kSimtA_E2M1>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s);
  }
  if (afmt == BL_A_I8 && wfmt == BL_W_T2 && M >= bl::kTsMinTokens) {
    // 2-bit weights widened into tensor memory; tokens on the MMA's N side
    if (!tc_kernel_ready()) return BL_ERR_CUDA;
    const int nt = m <= 8 ? 8 : (m >= 256 ? 256 : ((m + 15) & ~15));
    const int sub = nt <= 32 ? 4 : (nt <= 96 ? 2 : 1);          // 256-code sub-stages per TMA stage
    CUtensorMap tx, tw;
    if (!make_i8_map(&tx, A, static_cast<uint64_t>(M), static_cast<uint64_t>(K), static_cast<uint32_t>(nt), 128) ||
        !make_u64_map(&tw, W, static_cast<uint64_t>(N), static_cast<uint64_t>(K / 4), bl::kTsBN,
                      static_cast<uint32_t>(sub * bl::kTsSubK / 4)))
      return BL_ERR_CUDA;
    bl::TsParams p;
    p.a_scale = a_scale;
    p.alpha = alpha;
    p.alpha_group = alpha_group;
    p.M = m;
    p.N = n;
    p.K = k;
    p.y = Y;
    p.ldy = ldy;
    p.acc = acc_out;
    p.nt = nt;
    p.num_n_tiles = (n + bl::kTsBN - 1) / bl::kTsBN;
    p.num_units = p.num_n_tiles * ((m + nt - 1) / nt);
    p.num_kb = (k + sub * bl::kTsSubK - 1) / (sub * bl::kTsSubK);
    p.stage_x = static_cast<uint32_t>(nt * sub * bl::kTsSubK);
    const uint32_t per_stage = p.stage_x + static_cast<uint32_t>(bl::kTsBN * sub * bl::kTsSubK / 4);
    int stages = static_cast<int>((208u * 1024u) / per_stage);
    p.stages = stages < 2 ? 2 : (stages > bl::kTsMaxStages ? bl::kTsMaxStages : stages);
    // the whole TMEM: up to four accumulators of nt columns, and as many 64-column A buffers as fit
    p.dslots = nt <= 32 ? 4u : (nt <= 64 ? 2u : 1u);
    const uint32_t ab = (512u - p.dslots * static_cast<uint32_t>(nt)) / bl::kTsACols;
    p.abufs = ab > static_cast<uint32_t>(bl::kTsMaxABufs) ? static_cast<uint32_t>(bl::kTsMaxABufs) : ab;
    const size_t smem = 1024 + static_cast<size_t>(p.stages) * per_stage + 512;   // + barriers
    const int grid = p.num_units < sm_count() ? p.num_units : sm_count();
    if (sub == 4) launch_pdl(bl::gemm_t2tc_kernel<4>, grid, bl::kTsThreads, smem, s, tx, tw, p);
    else if (sub == 2) launch_pdl(bl::gemm_t2tc_kernel<2>, grid, bl::kTsThreads, smem, s, tx, tw, p);
    else launch_pdl(bl::gemm_t2tc_kernel<1>, grid, bl::kTsThreads, smem, s, tx, tw, p);
    return launch_status();
  }
  // CUDA-core kernel: one row of A per tile must fit in shared memory
  if (K > kSimtMaxK) return BL_ERR_SHAPE;
  const bool t2 = wfmt == BL_W_T2;
  bool ok;
  switch (afmt) {
    case BL_A_I8:
      ok = t2 ? launch_simt<bl::kSimtA_I8, true>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s)
              : launch_simt<bl::kSimtA_I8, false>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s);
      break;
    case BL_A_I4:
      ok = t2 ? launch_simt<bl::kSimtA_I4, true>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s)
              : launch_simt<bl::kSimtA_I4, false>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s);
      break;
    default:
      ok = t2 ? launch_simt<bl::kSimtA_E2M1, true>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s)
              : launch_simt<bl::kSimtA_E2M1, false>(A, a_scale, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s);
      break;
  }
  if (!ok) return BL_ERR_CUDA;
  return launch_status();
}

bl_status bitlinear_quant_gemm(const void* x_bf16, int64_t ldx, bl_quant quant, float eps, const void* w,
                               bl_wfmt wfmt, const float* alpha, int64_t alpha_group, int64_t M, int64_t N, int64_t K,
                               void* y_bf16, int64_t ldy, int32_t* acc_out, void* workspace, size_t ws_bytes,
                               void* stream) {
  NvtxRange nvtx_range("bitlinear_quant_gemm");
  if (quant != BL_QUANT_INT4 && quant != BL_QUANT_FP4_E2M1) return BL_ERR_ARG;
  if (wfmt != BL_W_T2 && wfmt != BL_W_I8) return BL_ERR_ARG;
  if (alpha_group < 1 || alpha_group > 0x7FFFFFFFLL || !(eps >= 0.f)) return BL_ERR_ARG;
  if (M < 0 || N < 1 || K < 64 || (K & 63) || K > 16384 || ldx < K || (ldx & 7) || M > 0x7FFFFFFELL ||
      N > 0x7FFFFFFFLL)
    return BL_ERR_SHAPE;
  if (y_bf16 != nullptr && (ldy < N || (ldy & 7))) return BL_ERR_SHAPE;
  if (M == 0) return BL_OK;
  if (x_bf16 == nullptr || w == nullptr || alpha == nullptr) return BL_ERR_NULL;
  if (y_bf16 == nullptr && acc_out == nullptr) return BL_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(w) || (y_bf16 && !aligned16(y_bf16)) || (acc_out && !aligned16(acc_out)) ||
      (reinterpret_cast<uintptr_t>(alpha) & 3u))
    return BL_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  const bool fp4 = quant == BL_QUANT_FP4_E2M1;
  if (wfmt == BL_W_T2 && M <= kQgFusedMaxTokens && gemv_applies(M, K, kGvMaxTokens)) {
    // decode of 1-2 tokens: each GEMV CTA quantizes the token rows itself
    const uint8_t* X = static_cast<const uint8_t*>(x_bf16);
    const uint8_t* W = static_cast<const uint8_t*>(w);
    uint16_t* Y = static_cast<uint16_t*>(y_bf16);
    const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
    if (fp4)
      return launch_gemv_any<bl::kGvX_Fp4>(X, nullptr, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s, ldx, eps);
    return launch_gemv_any<bl::kGvX_Int4>(X, nullptr, W, alpha, alpha_group, m, n, k, Y, ldy, acc_out, s, ldx, eps);
  }
  // otherwise the quantizer writes int8 codes into the workspace for the GEMM
  if (workspace == nullptr) return BL_ERR_NULL;
  if (!aligned16(workspace)) return BL_ERR_ALIGN;
  if (ws_bytes < static_cast<size_t>(qg_workspace_bytes(M, K))) return BL_ERR_WORKSPACE;
  uint8_t* codes = static_cast<uint8_t*>(workspace);
  float* scale = reinterpret_cast<float*>(codes + qg_codes_bytes(M, K));
  const bl_status st = bitlinear_quant_a4(x_bf16, M, K, ldx, quant, BL_STORE_BYTES, eps, codes, scale, stream);
  if (st != BL_OK) return st;
  return bitlinear_gemm(codes, BL_A_I8, scale, w, wfmt, alpha, alpha_group, M, N, K, y_bf16, ldy, acc_out, stream);
}

bl_status bitlinear_gemm_gated(const void* a, bl_afmt afmt, const float* a_scale, const void* w, bl_wfmt wfmt,
                               const float* alpha, int64_t M, int64_t F, int64_t K, void* y_bf16, int64_t ldy,
                               int32_t* acc_out, void* stream) {
  NvtxRange nvtx_range("bitlinear_gemm_gated");
  if (afmt != BL_A_I8 && afmt != BL_A_I4 && afmt != BL_A_E2M1) return BL_ERR_ARG;
  if (wfmt != BL_W_T2) return BL_ERR_UNSUPPORTED;
  if (M < 0 || F < 1 || K < 64 || (K & 63) || F > 0x3FFFFFFFLL || ldy < 2 * F || (ldy & 7)) return BL_ERR_SHAPE;
  if (M == 0) return BL_OK;
  if (M > 2 || K > 4096) return BL_ERR_UNSUPPORTED;   // the decode kernel: one 4096-code round, 1-2 tokens
  if (a == nullptr || a_scale == nullptr || w == nullptr || alpha == nullptr || y_bf16 == nullptr) return BL_ERR_NULL;
  if (!aligned16(a) || !aligned16(w) || !aligned16(y_bf16) || (acc_out && !aligned16(acc_out)) ||
      (reinterpret_cast<uintptr_t>(a_scale) & 3u) || (reinterpret_cast<uintptr_t>(alpha) & 3u))
    return BL_ERR_ALIGN;
  cudaStream_t s = as_stream(stream);
  const int m = static_cast<int>(M), f = static_cast<int>(F), k = static_cast<int>(K);
  const uint8_t* A = static_cast<const uint8_t*>(a);
  const uint8_t* W = static_cast<const uint8_t*>(w);
  uint16_t* Y = static_cast<uint16_t*>(y_bf16);
  auto go = [&](auto kern, int mt) -> bl_status {
    const size_t smem = static_cast<size_t>(mt) * static_cast<size_t>(k);
    int per_sm = 0;
    if (!cuda_ok(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem))) return BL_ERR_CUDA;
    if (per_sm < 1) per_sm = 1;
    const int64_t passes = ((static_cast<int64_t>(f) + 3) / 4 + 7) / 8;
    const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm;
    const unsigned grid = static_cast<unsigned>(passes < cap ? passes : cap);
    launch_pdl(kern, grid, 256, smem, s, A, a_scale, W, alpha, m, f, k, Y, ldy, acc_out);
    return launch_status();
  };
  if (afmt == BL_A_I8) return m == 1 ? go(bl::gemv_gated_t2_kernel<bl::kSimtA_I8, 1>, 1)
                                     : go(bl::gemv_gated_t2_kernel<bl::kSimtA_I8, 2>, 2);
  if (afmt == BL_A_I4) return m == 1 ? go(bl::gemv_gated_t2_kernel<bl::kSimtA_I4, 1>, 1)
                                     : go(bl::gemv_gated_t2_kernel<bl::kSimtA_I4, 2>, 2);
  return m == 1 ? go(bl::gemv_gated_t2_kernel<bl::kSimtA_E2M1, 1>, 1) : go(bl::gemv_gated_t2_kernel<bl::kSimtA_E2M1, 2>, 2);
}

bl_status kv_quant3(const void* kv_bf16, int64_t T, int64_t H, int64_t D, int64_t ldt, int bits, int64_t bos_pos,
                    float eps, uint8_t* codes, float* scale, uint8_t* bos_codes, void* stream) {
  NvtxRange nvtx_range("kv_quant3");
  if (bits != 3 && bits != 4) return BL_ERR_ARG;
  if (T < 0 || H < 1 || (D != 32 && D != 64 && D != 128 && D != 256) || ldt < H * D || (ldt & 7))
    return BL_ERR_SHAPE;
  if (bos_pos < -1) return BL_ERR_ARG;
  if (!(eps >= 0.f)) return BL_ERR_ARG;
  if (T * H > 0x7FFFFFFFLL / 4 || H > 0x7FFFFFFF) return BL_ERR_SHAPE;   // 32-bit vector indices in the kernel
  if (T == 0) return BL_OK;
  const bool has_bos = bits == 3 && bos_pos >= 0 && bos_pos < T;
  if (kv_bf16 == nullptr || codes == nullptr || scale == nullptr || (has_bos && bos_codes == nullptr))
    return BL_ERR_NULL;
  if (!aligned16(kv_bf16) || !aligned16(codes) || !aligned16(scale) || (has_bos && !aligned16(bos_codes)))
    return BL_ERR_ALIGN;
  const int tpv = static_cast<int>(D / 32);
  // persistent grid: eight CTAs per SM at most, each thread group kKvItems vectors per round
  const int64_t groups = (T * H + bl::kKvItems - 1) / bl::kKvItems;
  const int64_t need = (groups * tpv + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const unsigned grid = static_cast<unsigned>(need < cap ? need : cap);
  const uint16_t* kv = static_cast<const uint16_t*>(kv_bf16);
  cudaStream_t s = as_stream(stream);
  const int64_t bos = has_bos ? bos_pos : -1;
  const int h = static_cast<int>(H);
  switch (tpv) {
    case 1: launch_pdl(bl::kv_quant_kernel<1>, grid, 256, 0, s, kv, T, h, ldt, bits, bos, eps, codes, scale, bos_codes); break;
    case 2: launch_pdl(bl::kv_quant_kernel<2>, grid, 256, 0, s, kv, T, h, ldt, bits, bos, eps, codes, scale, bos_codes); break;
    case 4: launch_pdl(bl::kv_quant_kernel<4>, grid, 256, 0, s, kv, T, h, ldt, bits, bos, eps, codes, scale, bos_codes); break;
    case 8: launch_pdl(bl::kv_quant_kernel<8>, grid, 256, 0, s, kv, T, h, ldt, bits, bos, eps, codes, scale, bos_codes); break;
    default: return BL_ERR_SHAPE;
  }
  return launch_status();
}

bl_status attention_lowbit(const uint8_t* q_codes, const float* q_scale, int64_t M, const uint8_t* k_codes,
                           const float* k_scale, const uint8_t* k_bos, const uint8_t* v_codes, const float* v_scale,
                           const uint8_t* v_bos, int64_t T, int64_t H, int64_t D, int kv_bits, int64_t bos_pos,
                           float softmax_scale, void* out_bf16, int64_t ldo, void* workspace, size_t ws_bytes,
                           void* stream) {
  NvtxRange nvtx_range("attention_lowbit");
  if (kv_bits != 3 && kv_bits != 4) return BL_ERR_ARG;
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f) return BL_ERR_ARG;
  if (bos_pos < -1) return BL_ERR_ARG;
  if ((D != 64 && D != 128) || H < 4 || (H & 3) || H * (D / 32) > bl::kAttnThreads) return BL_ERR_SHAPE;
  if (T < 1 || M < 0 || M > T || M > 65535 || T > 0x7FFFFFFFLL / 4 / H || ldo < H * D) return BL_ERR_SHAPE;
  if (M == 0) return BL_OK;
  const bool has_bos = kv_bits == 3 && bos_pos >= 0 && bos_pos < T;
  if (q_codes == nullptr || q_scale == nullptr || k_codes == nullptr || k_scale == nullptr || v_codes == nullptr ||
      v_scale == nullptr || out_bf16 == nullptr || workspace == nullptr || (has_bos && (k_bos == nullptr || v_bos == nullptr)))
    return BL_ERR_NULL;
  if (!aligned16(q_codes) || !aligned16(k_codes) || !aligned16(v_codes) || !aligned16(workspace) ||
      ((reinterpret_cast<uintptr_t>(q_scale) | reinterpret_cast<uintptr_t>(k_scale) |
        reinterpret_cast<uintptr_t>(v_scale)) & 3u) || (reinterpret_cast<uintptr_t>(out_bf16) & 1u))
    return BL_ERR_ALIGN;
  if (ws_bytes < attn_workspace_bytes(M, H, D)) return BL_ERR_WORKSPACE;
  bl::AttnParams a = {};
  a.q = q_codes;
  a.qs = q_scale;
  a.k = k_codes;
  a.ks = k_scale;
  a.v = v_codes;
  a.vs = v_scale;
  a.kbos = k_bos;
  a.vbos = v_bos;
  a.M = static_cast<int>(M);
  a.T = static_cast<int>(T);
  a.H = static_cast<int>(H);
  a.bos = has_bos ? static_cast<int>(bos_pos) : -1;
  a.coef = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634);   // log2(e)
  a.part = static_cast<float*>(workspace);
  a.out = static_cast<uint16_t*>(out_bf16);
  a.ldo = ldo;
  cudaStream_t s = as_stream(stream);
  if (D == 128) return kv_bits == 3 ? launch_attention<128, 3>(a, s) : launch_attention<128, 4>(a, s);
  return kv_bits == 3 ? launch_attention<64, 3>(a, s) : launch_attention<64, 4>(a, s);
}

}  // extern "C"
