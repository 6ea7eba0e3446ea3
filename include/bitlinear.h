/*
 * bitlinear.h -- C ABI of libbitlinear, the sm_100a (B200) implementation of the
 * BitLinear forward path of BitNet a4.8 ("BitNet a4.8: 4-bit Activations for
 * 1-bit LLMs", arXiv 2411.04965).
 *
 * Conventions for every entry point
 *   - All tensor arguments are DEVICE pointers owned by the caller.  The library
 *     allocates no device memory, keeps no per-call state and never frees
 *     caller memory.  Work is enqueued on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and is asynchronous: outputs are valid once the
 *     stream has reached that point.
 *   - bf16 tensors are IEEE bfloat16, row-major.  "ld" arguments are row
 *     strides in elements.  Pointers must be 16-byte aligned and row strides
 *     must keep every row 16-byte aligned (noted per call).
 *   - Arguments are validated on the host before anything is launched; a bad
 *     argument returns a status without touching the GPU.  A launch failure
 *     returns BL_ERR_CUDA.  Kernels bound every wait; a wait that runs out sets
 *     a device status word instead of hanging, and bitlinear_sync_status()
 *     reports it (BL_ERR_TIMEOUT).  No C++ exception crosses this boundary.
 *   - Quantizers work per token (one row of X).  NaN/Inf inputs are outside the
 *     contract (results unspecified).
 *   - eps is the paper's "small constant" (1e-5 in the tests).
 *   - Host threads: the first call that meets a kernel at a given shared-memory
 *     size on a device raises that kernel's shared-memory limit and caches the
 *     device's SM count; this setup is not synchronised between host threads.
 *     Make calls from one host thread, or run each operation and shape once on
 *     one thread before calling from several.
 */
#ifndef BITLINEAR_H_
#define BITLINEAR_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BL_API __attribute__((visibility("default")))
#else
#define BL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BL_OK = 0,
    BL_ERR_NULL = 1,          /* a required pointer is NULL */
    BL_ERR_ALIGN = 2,         /* a pointer or row stride breaks the 16-byte rule */
    BL_ERR_SHAPE = 3,         /* a size is out of range for this call */
    BL_ERR_ARG = 4,           /* an enum or scalar argument is invalid */
    BL_ERR_UNSUPPORTED = 5,   /* valid, but this build has no kernel for it */
    BL_ERR_CUDA = 6,          /* the CUDA runtime reported an error */
    BL_ERR_TIMEOUT = 7,       /* a kernel gave up on a bounded wait */
    BL_ERR_WORKSPACE = 8      /* workspace too small */
} bl_status;

/* Quantizer choice for the 4-bit activation path. */
typedef enum {
    BL_QUANT_INT4 = 0,        /* absmean INT4, Eq. 6-7 */
    BL_QUANT_FP4_E2M1 = 1,    /* MinMax FP4 E2M1, Eq. 8-9 */
    /* the ablation variants of Fig. 5 / Fig. 6 (formulas are readings, see bitlinear_quant_a4) */
    BL_QUANT_INT4_ABSMAX = 2,   /* INT4 absmax */
    BL_QUANT_INT4_ABSMEAN2 = 3, /* INT4 absmean with beta = 2 mean|x| */
    BL_QUANT_FP4_E1M2 = 4       /* MinMax FP4 E1M2 */
} bl_quant;

/* How 4-bit codes are stored. */
typedef enum {
    BL_STORE_PACKED = 0,      /* two codes per byte: element 2i in bits 0-3, 2i+1 in bits 4-7 */
    BL_STORE_BYTES = 1        /* one signed byte per element (tensor-core operand layout) */
} bl_store;

/* Activation operand formats accepted by bitlinear_gemm. */
typedef enum {
    BL_A_I8 = 0,              /* int8 per element: INT8 codes, INT4 codes in bytes, or FP4 as 2*value */
    BL_A_I4 = 1,              /* packed two's-complement INT4 nibbles (BL_STORE_PACKED of INT4) */
    BL_A_E2M1 = 2             /* packed E2M1 nibbles (BL_STORE_PACKED of FP4) */
} bl_afmt;

/* Ternary weight formats (both K-major: row n holds the K codes of output n). */
typedef enum {
    BL_W_T2 = 0,              /* 2-bit codes, 4 per byte, element 4i in bits 0-1: 0->00, +1->01, -1->11 */
    BL_W_I8 = 1,              /* one int8 in {-1,0,1} per element (tensor-core operand layout) */
    BL_W_E2M1 = 2             /* E2M1 nibbles, element 2i in bits 0-3: 0 -> 0x0, +1 -> 0x2, -1 -> 0xA
                                 (the FP4 tensor-core operand for BL_A_E2M1 activations) */
} bl_wfmt;

/*
 * bitlinear_quant_a4 -- 4-bit activation quantizer for the Gaussian-like inputs
 * (attention QKV and FFN Up/Gate inputs).
 * Paper: §3.4 "4-Bit Activation Quantization for Gaussian-Like Inputs".
 *   BL_QUANT_INT4 (Eq. 6-7): beta = mean|x| over the row (summed exactly in
 *     fp64 -- the contract covers rows whose |x| sum is exact in fp64, true for
 *     ordinary data), mult = fp32(sqrt7) / (beta + eps) in fp32,
 *     code = RoundClip(x * mult, -8, 7) with round-half-even.
 *     scale[m] = beta / fp32(sqrt7) (the dequant factor).
 *   BL_QUANT_FP4_E2M1 (Eq. 8-9, garbled on the page; reading used): p = the
 *     smallest integer with max|x| <= 6 * 2^p (p = 0 for a zero row); each
 *     x * 2^-p is rounded to the nearest E2M1 value {0,.5,1,1.5,2,3,4,6}, ties
 *     to the even encoding; codes are sign bit 3 + value bits 0-2, a zero
 *     magnitude is always +0.  scale[m] = 2^p.
 *   Ablation variants (Fig. 5, Fig. 6; the pages give no formulas, readings):
 *   BL_QUANT_INT4_ABSMAX: gamma = max|x|, mult = 7 / (gamma + eps),
 *     code = RoundClip(x * mult, -8, 7), scale[m] = gamma / 7 (Eq. 1's absmax
 *     quantizer with the 4-bit range).
 *   BL_QUANT_INT4_ABSMEAN2: BL_QUANT_INT4 with beta = 2 mean|x|.
 *   BL_QUANT_FP4_E1M2: magnitudes {0,.25,...,1.75} (1 exponent bit with bias 1,
 *     2 mantissa bits); p = the smallest integer with max|x| <= 1.75 * 2^p;
 *     nearest magnitude, ties to the even encoding; codes as for E2M1 (sign
 *     bit 3 + magnitude index bits 0-2); scale[m] = 2^p.
 * Storage: BL_STORE_PACKED writes M x K/2 bytes; BL_STORE_BYTES writes M x K
 *   int8 (INT4: the code itself; FP4 E2M1: 2 * value, an exact integer in
 *   [-12, 12], with scale[m] = 2^(p-1) so that value * 2^p = byte * scale;
 *   FP4 E1M2: 4 * value in [-7, 7] with scale[m] = 2^(p-2)).  The GEMM takes
 *   the bytes of every variant as BL_A_I8, the packed INT4 variants as
 *   BL_A_I4 and packed E2M1 as BL_A_E2M1.
 * x: [M x K] bf16 with row stride ldx.  codes: contiguous rows.  scale: [M] fp32.
 * Requires K % 8 == 0, 8 <= K <= 16384, ldx % 8 == 0, 16-byte aligned pointers.
 */
BL_API bl_status bitlinear_quant_a4(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                             bl_quant quant, bl_store store, float eps,
                             void* codes, float* scale, void* stream);

/*
 * bitlinear_rmsnorm_quant_a4 -- RMSNorm fused into the 4-bit quantizer: the
 * per-layer data flow puts an RMSNorm before each 4-bit quantization (paper:
 * §3.2, "RMSNorm -> 4-bit quantize -> attention QKV" and "-> FFN Up/Gate"); this
 * call reads x once and writes exactly the codes and scales that
 * bitlinear_quant_a4 writes for y = RMSNorm(x).
 * RMSNorm (the pages give no formula; reading used):
 *   ms = mean(x^2) over the row -- the exact mean of the squares, rounded once
 *        to fp32 (order-free; the contract covers rows whose squares, as
 *        multiples of the smallest one's last significant bit, sum below 2^90,
 *        true for ordinary data),
 *   r  = 1 / sqrt(ms + eps_norm),  y_k = bf16((x_k * r) * gamma_k),
 * each operation a single IEEE fp32 operation rounded to nearest even, the
 * last to bf16; gamma NULL means gamma_k = 1 (then y_k = bf16(x_k * r)).
 * Then quant as in bitlinear_quant_a4 (any bl_quant, either bl_store).
 * x: [M x K] bf16, row stride ldx.  gamma: [K] fp32 (nullable, 16-byte
 * aligned).  codes / scale as in bitlinear_quant_a4.
 * Requires K % 8 == 0, 8 <= K <= 16384, ldx % 8 == 0, eps_norm > 0 (finite).
 */
BL_API bl_status bitlinear_rmsnorm_quant_a4(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                            const float* gamma, float eps_norm, bl_quant quant, bl_store store,
                                            float eps, void* codes, float* scale, void* stream);

/*
 * bitlinear_quant_a4_per_tensor -- INT4 absmean with one scale for the whole
 * tensor: beta = mean|X| over all M x K entries (the per-tensor scaling of the
 * ablations, Fig. 5 / Fig. 6; also the literal reading of Eq. 6-7, whose mean
 * runs over all entries of X).  beta is the exact mean rounded once to fp32
 * (the exponent-bin sum of pack_ternary), then every row is quantized as by
 * BL_QUANT_INT4 with that beta: code = RoundClip(x * fp32(sqrt7)/(beta + eps),
 * -8, 7), scale[m] = beta / fp32(sqrt7) for every m.
 * x: [M x K] bf16, row stride ldx.  codes / scale as in bitlinear_quant_a4
 * (BL_STORE_PACKED or BL_STORE_BYTES).  beta: one device float, written.
 * workspace: bitlinear_workspace_size("quant_a4_per_tensor", M, K, 0) bytes
 * (2 KiB, 8-byte aligned, cleared by the call).
 * Requires K % 8 == 0, 8 <= K <= 16384, ldx % 8 == 0, M * K < 2^31.
 */
BL_API bl_status bitlinear_quant_a4_per_tensor(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                               bl_store store, float eps, void* codes, float* scale, float* beta,
                                               void* workspace, size_t ws_bytes, void* stream);

/*
 * bitlinear_sparsify_a8 -- Top-K sparsification then INT8 absmax quantization
 * for the outlier-heavy inputs (attention-output and FFN-down inputs).
 * Paper: §3.4 "Sparsification Pipeline for Outlier-Heavy Intermediate States",
 * Eq. 1 with Q_INT8:  codes = RoundClip(127/(gamma+eps) * x, -128, 127) * M,
 * gamma = max|x| over the row, M = Top_k(|x|).
 * Top-K reading: exactly k_keep survivors per row, ranked by |x| (the bf16
 * magnitude) descending; equal magnitudes are taken in increasing index order.
 * x: [M x K] bf16, row stride ldx.  codes: [M x K] int8 (0 where masked).
 * scale: [M] fp32 = gamma / 127.  mask (nullable): [M x ceil(K/32)] uint32,
 * bit j of word w is element 32w + j; bits past K are 0.
 * Requires 1 <= k_keep <= K, K % 8 == 0, K <= 16384, ldx % 8 == 0.
 */
BL_API bl_status bitlinear_sparsify_a8(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                int64_t k_keep, float eps, int8_t* codes, float* scale,
                                uint32_t* mask, void* stream);

/*
 * pack_ternary -- absmean ternary weight quantizer and packer.
 * Paper: §3.4 "Ternary Weight Quantization (BitLinear)", Eq. 2:
 *   alpha = mean|W| over the whole tensor, t = RoundClip(W / (alpha + eps), -1, 1).
 * alpha is the exact mean rounded once to fp32 (round-half-even): |w| values are
 * summed exactly in integer bins per fp32 exponent, then divided and rounded
 * with multi-word integer arithmetic on the device.  The division W/(alpha+eps)
 * is an IEEE fp32 division.
 * w: [N x K] fp32, row stride ldw.  alpha: one device float; read as the
 * input when alpha_given != 0, written otherwise.  w_out: BL_W_T2 -> N x K/4
 * bytes, BL_W_I8 -> N x K bytes, BL_W_E2M1 -> N x K/2 bytes (layouts in bl_wfmt).
 * workspace: device scratch of bitlinear_workspace_size("pack_ternary", N, K, 0)
 * bytes (2 KiB; cleared by the call itself).  Not needed when alpha_given != 0.
 * Requires K % 16 == 0, ldw % 4 == 0, N * K < 2^31.
 */
BL_API bl_status pack_ternary(const float* w, int64_t N, int64_t K, int64_t ldw, float eps,
                       int alpha_given, float* alpha, bl_wfmt wfmt, void* w_out,
                       void* workspace, size_t ws_bytes, void* stream);

/*
 * pack_ternary_noalloc -- pack_ternary for callers that cannot allocate device
 * memory.  The paper has no counterpart: this is an interface convenience.
 * Some callers may not allocate at all while they run -- an inference engine
 * that owns every byte of device memory and forbids allocation inside its
 * execute step (plugin interfaces, fixed-budget serving loops), or a C host
 * with no device allocator of its own.  This variant needs no workspace
 * argument: its scratch (the exponent bins of the exact |W| sum) is a
 * 2 KiB array inside the library, one per GPU that has loaded the library,
 * held until the process exits.  The caller still passes w, alpha and w_out.
 * Same arguments, layouts and results as pack_ternary (alpha and codes are
 * bit-identical); the scratch is cleared at the start of every call.
 * Limits: N * K < 2^31, so no 64-bit bin can overflow; larger tensors are
 * rejected with BL_ERR_SHAPE.  The first call on a device looks up the
 * array's device address (once per device) and caches it; make that first
 * call before any stream capture.  The cached address belongs to the device's
 * current primary context: after cudaDeviceReset() on that device it is stale,
 * so do not call this function again in that process after a reset.  Every
 * call on a device shares the one array, so calls that
 * can overlap on that GPU (different streams, no ordering between them) race
 * and must be serialized by the caller.  Allocates nothing.
 */
BL_API bl_status pack_ternary_noalloc(const float* w, int64_t N, int64_t K, int64_t ldw, float eps,
                                      int alpha_given, float* alpha, bl_wfmt wfmt, void* w_out,
                                      void* stream);

/*
 * bitlinear_gemm -- BitLinear product with integer accumulation and the
 * per-token x per-tensor dequant epilogue.
 * Paper: §3.4, Y = Q_x(X) . Q_w(W)^T (the equation above Eq. 6, and Eq. 1).
 *   acc[m,n] = sum_k a[m,k] * t[n,k]          exact int32
 *   y[m,n]   = bf16( acc[m,n] * a_scale[m] * alpha[n / alpha_group] )
 * For BL_A_E2M1 the codes' values are summed (exact: multiples of 0.5), and
 * acc_out holds 2 * the sum.
 * a: [M x K] in `afmt` (contiguous rows), a_scale: [M] fp32 (the scale the
 * quantizer wrote), w: [N x K] in `wfmt` (pack_ternary's output), alpha: fp32
 * array with one entry per group of alpha_group consecutive outputs
 * (alpha_group = N for one tensor; e.g. F for stacked Up|Gate weights).
 * y: [M x N] bf16 with row stride ldy (nullable).  acc_out: [M x N] int32,
 * row stride N (nullable; a test aid).
 * Kernels: BL_A_I8 x BL_W_I8 runs on the tcgen05 tensor cores (kind::i8,
 * TMA-fed, TMEM accumulators).  BL_W_T2 with M <= 16 (decode) runs on a GEMV
 * that reads the 2-bit weights once, for any activation format: 1 or 2 tokens
 * with dp4a (token slots 1/2/4/8 x K <= 147456, K <= 65536), 3 to 16 tokens on
 * warp-level integer MMA (16 weight rows x 8 or 16 token slots, slots x K <=
 * 180224), both on the offset codes c + 1 with the token's code sum subtracted.
 * BL_A_I8 x BL_W_T2 beyond those runs on the tensor cores, the 2-bit weights
 * widened to int8 into tensor memory as the MMA's A operand (the tokens are the
 * MMA's N side).  Other cases run on a CUDA-core kernel that reads
 * packed operands directly and needs K <= 196608 (BL_ERR_SHAPE beyond).
 * BL_A_E2M1 x BL_W_E2M1 (any M) runs on the tensor cores as kind::mxf4 with
 * unit block scales and fp32 accumulation, exact for these operands (every
 * partial sum is a multiple of 1/2 below 2^24); acc_out holds 2 * the sum.
 * BL_W_E2M1 weights take BL_A_E2M1 activations only.
 * Requires K % 64 == 0, K <= 2^20, ldy % 8 == 0, 1 <= alpha_group.
 */
BL_API bl_status bitlinear_gemm(const void* a, bl_afmt afmt, const float* a_scale,
                         const void* w, bl_wfmt wfmt, const float* alpha, int64_t alpha_group,
                         int64_t M, int64_t N, int64_t K,
                         void* y_bf16, int64_t ldy, int32_t* acc_out, void* stream);

/*
 * bitlinear_quant_gemm -- bitlinear_quant_a4 fused into the BitLinear GEMM:
 * y = bf16(Q(x) . t^T * scale[m] * alpha[n / alpha_group]) straight from the
 * bf16 rows x (paper: §3.4, Eq. 6-7 / 8-9 followed by Y = Q_x(X) . Q_w(W)^T).
 * The codes, the scale and acc_out are exactly those of bitlinear_quant_a4
 * followed by bitlinear_gemm (for FP4, acc_out holds 2 * the sum, as for
 * BL_A_E2M1 activations).
 * With BL_W_T2 weights and 1 or 2 tokens (a shape the decode GEMV takes; see
 * bitlinear_gemm) the quantization runs in the GEMV's prologue: every CTA reads
 * the M bf16 rows, reduces each token's statistic and quantizes into shared
 * memory, so no codes reach global memory and there is one launch (measured
 * faster there; from 3 tokens the repeated quantization in every CTA costs more
 * than the separate launch, so those run as two kernels).  Otherwise
 * it runs as bitlinear_quant_a4 (BL_STORE_BYTES) into `workspace` and then
 * bitlinear_gemm with BL_A_I8 codes; `workspace` then needs
 * bitlinear_workspace_size("quant_gemm", M, N, K) bytes (16-byte aligned) and
 * may be NULL otherwise.
 * x: [M x K] bf16, row stride ldx.  w: BL_W_T2 or BL_W_I8 (pack_ternary's
 * output).  y / acc_out / alpha / alpha_group as in bitlinear_gemm.
 * Requires K % 64 == 0, 64 <= K <= 16384, ldx % 8 == 0, ldy % 8 == 0.
 */
BL_API bl_status bitlinear_quant_gemm(const void* x_bf16, int64_t ldx, bl_quant quant, float eps,
                               const void* w, bl_wfmt wfmt, const float* alpha, int64_t alpha_group,
                               int64_t M, int64_t N, int64_t K,
                               void* y_bf16, int64_t ldy, int32_t* acc_out,
                               void* workspace, size_t ws_bytes, void* stream);

/*
 * bitlinear_gemm_gated -- the conditional Up projection (paper: §3.4 "Squared
 * ReLU Gating" and the FFN paragraph after Eq. 5: the Up projection only needs
 * the channels where ReLU^2(gate) != 0).  w = [W_up; W_gate] as for the stacked
 * Up|Gate bitlinear_gemm (F rows each, BL_W_T2), alpha = {alpha_up, alpha_gate}.
 *   y[m, F + n] = the Gate output, exactly as bitlinear_gemm writes it;
 *   y[m, n]     = the Up output where some token's gate output y[., F + n] is
 *                 > 0, else +0 (the Up row's bytes are then never read);
 *   acc_out likewise (0 for skipped Up entries).
 * relu2_glu(y[:, F:], y[:, :F], ...) then produces the same codes, mask and
 * scale as after the dense Up|Gate GEMM: h = up * max(0, gate)^2 is a zero on
 * the skipped channels either way.
 * a: M x K activation codes (afmt as for bitlinear_gemm); y: [M x ldy] bf16
 * with ldy >= 2F; acc_out: [M x 2F] int32 (nullable).
 * Requires K % 64 == 0.  Kernel: decode, M <= 2 and K <= 4096
 * (BL_ERR_UNSUPPORTED otherwise); weights only in BL_W_T2.
 */
BL_API bl_status bitlinear_gemm_gated(const void* a, bl_afmt afmt, const float* a_scale,
                               const void* w, bl_wfmt wfmt, const float* alpha,
                               int64_t M, int64_t F, int64_t K,
                               void* y_bf16, int64_t ldy, int32_t* acc_out, void* stream);

/*
 * relu2_glu -- squared-ReLU GLU fused with the down projection's
 * sparsify-then-quantize step.
 * Paper: §3.4 "Squared ReLU Gating and Conditional Computation in the FFN",
 * Eq. 5:  h = up (.) max(0, gate)^2, computed in fp32 as g2 = g*g, h = up*g2;
 * then Eq. 1 on h: gamma = max|h|, Top-K over |h| (fp32 magnitude, ties to
 * the lower index), codes = RoundClip(127/(gamma+eps) * h, -128, 127) * M.
 * k_keep = F keeps every entry (INT8 only).
 * gate, up: [M x F] bf16 with the shared row stride ld (e.g. the two halves of
 * a stacked Up|Gate output).  codes: [M x F] int8.  scale: [M] fp32 =
 * gamma / 127.  mask (nullable): [M x ceil(F/32)] uint32 as in sparsify_a8.
 * Requires 1 <= k_keep <= F, F % 8 == 0, F <= 16384, ld % 8 == 0.
 */
BL_API bl_status relu2_glu(const void* gate_bf16, const void* up_bf16, int64_t M, int64_t F, int64_t ld,
                    int64_t k_keep, float eps, int8_t* codes, float* scale, uint32_t* mask,
                    void* stream);

/*
 * kv_quant3 -- post-RoPE low-bit KV-cache quantizer.
 * Paper: §3.4 "Low-Bit KV Cache Quantization" (absmax to unsigned integers;
 * for 3-bit caches the beginning-of-sequence heads stay at 4 bits).
 * Reading: per (position t, head h) vector of D values, gamma = max|x|,
 * Q = 2^(b-1) - 1, c = RoundClip(Q/(gamma+eps) * x, -Q-1, Q), stored unsigned
 * as c + 2^(b-1); scale = gamma / Q.
 * kv: [T x H x D] bf16, stride ldt elements between positions (ldt >= H*D).
 * codes: [T x H x D*bits/8] bytes.  bits = 3: eight codes per 3 bytes, code j
 * of a group in bits 3j..3j+2 of a little-endian 24-bit word.  bits = 4: the
 * nibble layout of BL_STORE_PACKED.  scale: [T x H] fp32.
 * When bits == 3 and 0 <= bos_pos < T, position bos_pos is quantized at 4 bits
 * into bos_codes ([H x D/2] bytes, nibble layout), its scale is gamma/7, and
 * its 3-bit slot in `codes` is zero-filled.  bos_pos = -1: no BOS row.
 * Requires D in {32, 64, 128, 256}, ldt % 8 == 0, T * H < 2^29.
 */
BL_API bl_status kv_quant3(const void* kv_bf16, int64_t T, int64_t H, int64_t D, int64_t ldt, int bits,
                    int64_t bos_pos, float eps, uint8_t* codes, float* scale, uint8_t* bos_codes,
                    void* stream);

/*
 * attention_lowbit -- softmax attention of 4-bit queries over the low-bit KV
 * cache that kv_quant3 writes.
 * Paper: §3.4 "Low-Bit KV Cache Quantization" (post-RoPE Q, K and V quantized
 * by absmax to unsigned integers; 4-bit Q with 3-bit KV, the BOS position's
 * heads at 4 bits) and Table 3's "4-bit Q, 3-bit KV" / "4-bit QKV" rows.  The
 * pages give no attention formula; reading used (softmax over the dequantized
 * codes):
 *   q_hat = (q_code - 8) * q_scale,  k_hat_t = (k_code_t - 2^(b-1)) * k_scale_t,
 *   v_hat_t likewise (b = kv_bits; offset 8 at the BOS position of a 3-bit cache),
 *   s_t = softmax_scale * <q_hat, k_hat_t>,  out = sum_t softmax(s)_t * v_hat_t.
 * The M queries are the cache's last M positions: query m sits at position
 * T - M + m and attends positions 0 .. T - M + m (causal; M = 1 is decode).
 * q_codes: [M x H x D/2] bytes, 4-bit codes c + 8 (kv_quant3 with bits = 4 on
 * the query slice).  q_scale: [M x H] fp32.
 * k_codes / v_codes, k_scale / v_scale, k_bos / v_bos: as kv_quant3 writes them
 * for T positions (the BOS buffers are read only when kv_bits == 3 and
 * 0 <= bos_pos < T; bos_pos is ignored for 4-bit caches).
 * out: [M x ldo] bf16, row m holding head h's D values at h*D .. h*D + D-1
 * (the O projection's input layout), each rounded once to bf16.
 * Arithmetic: <q, k> exactly in integers, scores and the softmax in fp32 (base-2
 * exponentials), fp32 sums; against the fp64 definition the result is within
 * 2^-8 |out| + 2^-12 max_t |v_hat_t| per element.  The contract covers k_scale
 * and v_scale values between 2^-40 and 2^40 (the V sums carry a 2^64 factor).
 * workspace: bitlinear_workspace_size("attention_lowbit", M, H, D) bytes,
 * 16-byte aligned (partial results of the position chunks).
 * Requires D in {64, 128}, H % 4 == 0, H * D / 32 <= 256, 1 <= M <= min(T, 65535),
 * T * H < 2^29, ldo >= H * D; q_codes / k_codes / v_codes 16-byte aligned, the scales
 * 4-byte aligned.  M = 0 is a no-op.
 */
BL_API bl_status attention_lowbit(const uint8_t* q_codes, const float* q_scale, int64_t M, const uint8_t* k_codes,
                                  const float* k_scale, const uint8_t* k_bos, const uint8_t* v_codes,
                                  const float* v_scale, const uint8_t* v_bos, int64_t T, int64_t H, int64_t D,
                                  int kv_bits, int64_t bos_pos, float softmax_scale, void* out_bf16, int64_t ldo,
                                  void* workspace, size_t ws_bytes, void* stream);

/* Bytes of device workspace an operation needs ("pack_ternary", "quant_a4_per_tensor",
 * "quant_gemm"; "attention_lowbit" with M queries, N = H heads, K = D; 0 for the others). */
BL_API size_t bitlinear_workspace_size(const char* op, int64_t M, int64_t N, int64_t K);

/* Synchronizes `stream`, then reads and clears the calling device's status
 * word.  Returns BL_ERR_TIMEOUT if a kernel gave up on a bounded wait since the
 * last call, BL_ERR_CUDA on a runtime error, BL_OK otherwise. */
BL_API bl_status bitlinear_sync_status(void* stream);

/* Diagnostic of the failure handling (no counterpart in the paper): enqueues
 * one thread that waits, through the same bounded wait the tensor-core kernels
 * and the streaming GEMV use, on an mbarrier that nothing completes.  After the
 * wait limit (2 s) the thread gives up, records BL_ERR_TIMEOUT in the device
 * status word and returns; the next bitlinear_sync_status() reports
 * BL_ERR_TIMEOUT and clears it, and the context stays usable.  Returns the
 * launch status. */
BL_API bl_status bitlinear_selftest_timeout(void* stream);

/* Human-readable name of a status code (static storage). */
BL_API const char* bitlinear_status_string(bl_status status);

/* Name of the CUDA runtime error (static storage, e.g. "cudaErrorInvalidValue")
 * behind the last BL_ERR_CUDA that an entry point returned on the calling host
 * thread; "cudaSuccess" if there was none.  Not reset by later successful calls.
 * No counterpart in the paper: a diagnostic of this library. */
BL_API const char* bitlinear_last_cuda_error(void);

/* Library version string (static storage). */
BL_API const char* bitlinear_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H_ */
