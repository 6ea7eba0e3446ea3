"""CPU oracle for the BitLinear forward path of BitNet a4.8.

TEST INFRASTRUCTURE ONLY.  The plain, slow, obviously-correct definition of
what the CUDA path computes.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import it.  It shares nothing with the
CUDA path: the heavy loops are plain C in ``bitlinear_oracle.c`` (built with
gcc, no FMA contraction, no fast-math), the one step that needs more than
fp64 -- rounding the exact mean of |W| to fp32 -- is done here with Python
integers, and the storage layouts (nibbles, 2-bit and 3-bit packing) are
written from the layout statements of the public C header.

Equations follow arXiv 2411.04965 ("BitNet a4.8: 4-bit Activations for 1-bit
LLMs"), §3.4: Eq. 2 (ternary weights), Eq. 6-7 (INT4 absmean), Eq. 8-9 (FP4
MinMax), Eq. 1 with Q_INT8 (Top-K + INT8 absmax), Eq. 5 (ReLU^2-GLU) and the
"Low-Bit KV Cache Quantization" paragraph (the KV quantizer, and the attention
of 4-bit queries over the quantized cache).

Every function here is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from fractions import Fraction

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitlinear_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lib = None

EPS = 1e-5


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, IEEE fp32, no contraction) into _build/."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fno-tree-vectorize",
            "-std=c11", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        F = ctypes.c_float
        sigs = {
            "orc_quant_int4": [P, I64, I64, I64, F, P, P, P],
            "orc_quant_fp4": [P, I64, I64, I64, P, P, P, P],
            "orc_quant_int4_absmax": [P, I64, I64, I64, F, P, P, P],
            "orc_quant_int4_absmean2": [P, I64, I64, I64, F, P, P, P],
            "orc_quant_fp4_e1m2": [P, I64, I64, I64, P, P, P, P],
            "orc_sparsify_a8": [P, I64, I64, I64, I64, F, P, P, P, P],
            "orc_relu2_glu": [P, P, I64, I64, I64, I64, F, P, P, P, P, P],
            "orc_ternary_abs_bins": [P, I64, I64, I64, P],
            "orc_ternary_codes": [P, I64, I64, I64, F, F, P],
            "orc_gemm": [P, I64, P, P, P, I64, I64, I64, I64, P, I64, P, P],
            "orc_kv_quant": [P, I64, I64, I64, I64, ctypes.c_int, I64, F, P, P],
            "orc_rmsnorm_sumsq": [P, I64, I64, I64, P, P],
            "orc_rmsnorm_apply": [P, I64, I64, I64, P, P, F, P, P],
            "orc_quant_int4_given_beta": [P, I64, I64, I64, F, F, P, P],
            "orc_rounding_is_nearest": [],
        }
        for name, args in sigs.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        if lib.orc_rounding_is_nearest() != 1:
            raise RuntimeError("oracle needs round-to-nearest")
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"{what}: oracle precondition failed (code {rc})")


def _bf16_2d(x):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    if x.ndim != 2:
        raise ValueError("expected a 2-D bf16 (uint16) array")
    return x


# ---------------------------------------------------------------------------
# Quantizers
# ---------------------------------------------------------------------------
def quant_int4(x_bf16: np.ndarray, eps: float = EPS):
    """INT4 absmean per token (Eq. 6-7).  Returns (codes int8 [M,K] in
    [-8,7], beta fp32 [M], scale = beta/sqrt7 fp32 [M])."""
    x = _bf16_2d(x_bf16)
    M, K = x.shape
    codes = np.empty((M, K), np.int8)
    beta = np.empty(M, np.float32)
    scale = np.empty(M, np.float32)
    _check(_load().orc_quant_int4(_ptr(x), M, K, K, eps, _ptr(codes), _ptr(beta), _ptr(scale)),
           "quant_int4")
    return codes, beta, scale


def quant_fp4(x_bf16: np.ndarray):
    """FP4 E2M1 MinMax per token (Eq. 8-9, power-of-two reading).  Returns
    (code4 uint8 [M,K] E2M1 encodings, twice_value int8 [M,K], p int32 [M],
    scale = 2^p fp32 [M])."""
    x = _bf16_2d(x_bf16)
    M, K = x.shape
    code4 = np.empty((M, K), np.uint8)
    tv = np.empty((M, K), np.int8)
    p = np.empty(M, np.int32)
    scale = np.empty(M, np.float32)
    _check(_load().orc_quant_fp4(_ptr(x), M, K, K, _ptr(code4), _ptr(tv), _ptr(p), _ptr(scale)),
           "quant_fp4")
    return code4, tv, p, scale


def quant_int4_absmax(x_bf16: np.ndarray, eps: float = EPS):
    """INT4 absmax per token (the Fig. 6 ablation; reading: Eq. 1's absmax with
    the 4-bit range).  Returns (codes int8 [M,K], gamma fp32 [M], scale =
    gamma/7 fp32 [M])."""
    x = _bf16_2d(x_bf16)
    M, K = x.shape
    codes = np.empty((M, K), np.int8)
    gamma = np.empty(M, np.float32)
    scale = np.empty(M, np.float32)
    _check(_load().orc_quant_int4_absmax(_ptr(x), M, K, K, eps, _ptr(codes), _ptr(gamma), _ptr(scale)),
           "quant_int4_absmax")
    return codes, gamma, scale


def quant_int4_absmean2(x_bf16: np.ndarray, eps: float = EPS):
    """INT4 absmean with beta = 2 mean|x| per token (the Fig. 5 ablation).
    Returns (codes int8 [M,K], beta fp32 [M], scale = beta/sqrt7 fp32 [M])."""
    x = _bf16_2d(x_bf16)
    M, K = x.shape
    codes = np.empty((M, K), np.int8)
    beta = np.empty(M, np.float32)
    scale = np.empty(M, np.float32)
    _check(_load().orc_quant_int4_absmean2(_ptr(x), M, K, K, eps, _ptr(codes), _ptr(beta), _ptr(scale)),
           "quant_int4_absmean2")
    return codes, beta, scale


def quant_fp4_e1m2(x_bf16: np.ndarray):
    """FP4 E1M2 MinMax per token (the Fig. 6 ablation; reading: magnitudes
    {0,.25,...,1.75}, scale 2^p with max|x| <= 1.75*2^p).  Returns (code4 uint8
    [M,K], four_value int8 [M,K], p int32 [M], scale = 2^p fp32 [M])."""
    x = _bf16_2d(x_bf16)
    M, K = x.shape
    code4 = np.empty((M, K), np.uint8)
    fv = np.empty((M, K), np.int8)
    p = np.empty(M, np.int32)
    scale = np.empty(M, np.float32)
    _check(_load().orc_quant_fp4_e1m2(_ptr(x), M, K, K, _ptr(code4), _ptr(fv), _ptr(p), _ptr(scale)),
           "quant_fp4_e1m2")
    return code4, fv, p, scale


def sparsify_a8(x_bf16: np.ndarray, keep: int, eps: float = EPS):
    """Top-K (exactly `keep` per token, ties to the lower index) then INT8
    absmax (Eq. 1).  Returns (codes int8 [M,K], mask uint8 [M,K], gamma fp32
    [M], scale = gamma/127 fp32 [M])."""
    x = _bf16_2d(x_bf16)
    M, K = x.shape
    codes = np.empty((M, K), np.int8)
    mask = np.empty((M, K), np.uint8)
    gamma = np.empty(M, np.float32)
    scale = np.empty(M, np.float32)
    _check(_load().orc_sparsify_a8(_ptr(x), M, K, K, keep, eps, _ptr(codes), _ptr(mask),
                                   _ptr(gamma), _ptr(scale)), "sparsify_a8")
    return codes, mask, gamma, scale


def relu2_glu(gate_bf16: np.ndarray, up_bf16: np.ndarray, keep: int, eps: float = EPS,
              want_h: bool = False):
    """h = up * max(0, gate)^2 in fp32 (Eq. 5), then Top-K + INT8 on h.
    Returns (codes, mask, gamma, scale[, h])."""
    gate = _bf16_2d(gate_bf16)
    up = _bf16_2d(up_bf16)
    if gate.shape != up.shape:
        raise ValueError("gate/up shape mismatch")
    M, F = gate.shape
    codes = np.empty((M, F), np.int8)
    mask = np.empty((M, F), np.uint8)
    gamma = np.empty(M, np.float32)
    scale = np.empty(M, np.float32)
    h = np.empty((M, F), np.float32) if want_h else None
    _check(_load().orc_relu2_glu(_ptr(gate), _ptr(up), M, F, F, keep, eps, _ptr(codes), _ptr(mask),
                                 _ptr(h), _ptr(gamma), _ptr(scale)), "relu2_glu")
    return (codes, mask, gamma, scale, h) if want_h else (codes, mask, gamma, scale)


# ---------------------------------------------------------------------------
# RMSNorm ahead of the 4-bit quantizer (§3.2's data flow), and per-tensor INT4
# ---------------------------------------------------------------------------
def rmsnorm(x_bf16: np.ndarray, gamma=None, eps_norm: float = 1e-6):
    """y = bf16((x * r) * g), r = 1 / sqrt(ms + eps_norm) per row, ms the exact
    mean of x^2 rounded once to fp32, the rest single fp32 operations (see
    bitlinear_oracle.c).  Returns (y bf16 bits uint16 [M,K], r fp32 [M])."""
    x = _bf16_2d(x_bf16)
    M, K = x.shape
    g = None if gamma is None else np.ascontiguousarray(gamma, dtype=np.float32)
    if g is not None and g.shape != (K,):
        raise ValueError("gamma must have K entries")
    if not eps_norm > 0:
        raise ValueError("eps_norm must be positive")
    hi = np.empty(M, np.float64)
    lo = np.empty(M, np.float64)
    _check(_load().orc_rmsnorm_sumsq(_ptr(x), M, K, K, _ptr(hi), _ptr(lo)), "rmsnorm_sumsq")
    ms = np.array([round_fraction_to_f32((Fraction(float(h)) + Fraction(float(l))) / K) for h, l in zip(hi, lo)],
                  np.float32)
    y = np.empty((M, K), np.uint16)
    r = np.empty(M, np.float32)
    _check(_load().orc_rmsnorm_apply(_ptr(x), M, K, K, _ptr(ms), _ptr(g), np.float32(eps_norm), _ptr(y), _ptr(r)),
           "rmsnorm_apply")
    return y, r


def rmsnorm_quant(x_bf16: np.ndarray, gamma=None, eps_norm: float = 1e-6, quant: str = "int4", eps: float = EPS):
    """The 4-bit quantizer applied to the RMSNorm output: quant_int4 (returns
    (codes, beta, scale)) or quant_fp4 (returns (code4, twice, p, scale)) of
    rmsnorm(x)."""
    y, _ = rmsnorm(x_bf16, gamma, eps_norm)
    if quant == "int4":
        return quant_int4(y, eps)
    if quant == "fp4":
        return quant_fp4(y)
    raise ValueError(quant)


def tensor_abs_mean_bf16(x_bf16: np.ndarray) -> np.float32:
    """The exact mean of |x| over every entry of a bf16 tensor, rounded once to
    fp32 (the bf16 values are exact in fp32, so the exponent-bin sum of
    ternary_alpha applies unchanged)."""
    x = _bf16_2d(x_bf16)
    return ternary_alpha((x.astype(np.uint32) << 16).view(np.float32))


def quant_int4_per_tensor(x_bf16: np.ndarray, eps: float = EPS):
    """INT4 absmean with beta = mean|X| over the whole tensor (per-tensor
    scaling).  Returns (codes int8 [M,K], beta fp32, scale fp32 [M], every
    entry beta/sqrt7)."""
    x = _bf16_2d(x_bf16)
    M, K = x.shape
    beta = tensor_abs_mean_bf16(x)
    codes = np.empty((M, K), np.int8)
    scale = np.empty(M, np.float32)
    _check(_load().orc_quant_int4_given_beta(_ptr(x), M, K, K, np.float32(beta), eps, _ptr(codes), _ptr(scale)),
           "quant_int4_given_beta")
    return codes, beta, scale


# ---------------------------------------------------------------------------
# Ternary weights (Eq. 2)
# ---------------------------------------------------------------------------
def round_fraction_to_f32(q: Fraction) -> np.float32:
    """Round an exact non-negative rational to the nearest fp32, ties to even
    (normal and subnormal range; overflow raises)."""
    if q < 0:
        raise ValueError("non-negative only")
    if q == 0:
        return np.float32(0.0)
    # e = floor(log2(q)), found exactly from the integer bit lengths
    e = q.numerator.bit_length() - q.denominator.bit_length()
    if Fraction(2) ** e > q:
        e -= 1
    lsb = max(e - 23, -149)
    m = round(q / Fraction(2) ** lsb)          # Fraction.__round__ ties to even
    val = float(m) * 2.0 ** lsb                # exact: m <= 2^24
    if val >= 2.0 ** 128:
        raise OverflowError("mean |W| overflows fp32")
    return np.float32(val)


def ternary_alpha(w: np.ndarray) -> np.float32:
    """alpha = mean(|W|) over the whole tensor: the exact mean, rounded once
    to fp32.  The C side accumulates the exact integer sum per fp32 exponent."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    bins = np.zeros(256, np.uint64)
    _check(_load().orc_ternary_abs_bins(_ptr(w), N, K, K, _ptr(bins)), "ternary_abs_bins")
    total = Fraction(0)
    for e in range(256):
        if bins[e]:
            total += Fraction(int(bins[e])) * Fraction(2) ** (max(e, 1) - 150)
    return round_fraction_to_f32(total / (N * K))


def ternary_codes(w: np.ndarray, alpha: float, eps: float = EPS) -> np.ndarray:
    """t = RoundClip(w / (alpha + eps), -1, 1), fp32 division."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    t = np.empty((N, K), np.int8)
    _check(_load().orc_ternary_codes(_ptr(w), N, K, K, np.float32(alpha), eps, _ptr(t)),
           "ternary_codes")
    return t


def ternary_quantize(w: np.ndarray, eps: float = EPS):
    alpha = ternary_alpha(w)
    return ternary_codes(w, alpha, eps), alpha


# ---------------------------------------------------------------------------
# BitLinear matmul
# ---------------------------------------------------------------------------
def gemm(a_codes: np.ndarray, a_scale: np.ndarray, t_codes: np.ndarray, alpha, alpha_group: int = 0,
         rows=None, want_y: bool = True):
    """acc = A . T^T exactly (int64 checked into int32), y = bf16(acc * s_m * alpha).
    `alpha` is one value or an array indexed by n // alpha_group.
    Returns (acc int32 [R,N], y bf16 bits uint16 [R,N] or None)."""
    a = np.ascontiguousarray(a_codes, dtype=np.int8)
    t = np.ascontiguousarray(t_codes, dtype=np.int8)
    M, K = a.shape
    N, K2 = t.shape
    if K != K2:
        raise ValueError("K mismatch")
    al = np.atleast_1d(np.asarray(alpha, dtype=np.float32)).copy()
    group = alpha_group if alpha_group > 0 else N
    if al.size * group < N:
        raise ValueError("alpha too short")
    sc = np.ascontiguousarray(a_scale, dtype=np.float32)
    rr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    R = M if rr is None else rr.size
    acc = np.empty((R, N), np.int32)
    y = np.empty((R, N), np.uint16) if want_y else None
    _check(_load().orc_gemm(_ptr(a), K, _ptr(sc), _ptr(t), _ptr(al), group, M, N, K, _ptr(rr), R,
                            _ptr(acc), _ptr(y)), "gemm")
    return acc, y


# ---------------------------------------------------------------------------
# KV cache
# ---------------------------------------------------------------------------
def kv_quant(kv_bf16: np.ndarray, bits: int = 3, bos_pos: int = 0, eps: float = EPS):
    """Absmax per (position, head) to unsigned b-bit codes; position bos_pos
    at 4 bits when bits == 3.  kv: [T, H, D].  Returns (codes_u uint8
    [T,H,D], scale fp32 [T,H])."""
    kv = np.ascontiguousarray(kv_bf16, dtype=np.uint16)
    T, H, D = kv.shape
    codes = np.empty((T, H, D), np.uint8)
    scale = np.empty((T, H), np.float32)
    _check(_load().orc_kv_quant(_ptr(kv), T, H, D, H * D, bits, bos_pos, eps, _ptr(codes),
                                _ptr(scale)), "kv_quant")
    return codes, scale


# ---------------------------------------------------------------------------
# Low-bit attention over the quantized cache
# ---------------------------------------------------------------------------
def attention_lowbit(q_codes_u: np.ndarray, q_scale: np.ndarray, k_codes_u: np.ndarray, k_scale: np.ndarray,
                     v_codes_u: np.ndarray, v_scale: np.ndarray, kv_bits: int = 3, bos_pos: int = -1,
                     softmax_scale=None, heads=None) -> np.ndarray:
    """Attention of 4-bit queries over a 3- or 4-bit key/value cache, in fp64
    (§3.4 "Low-Bit KV Cache Quantization": post-RoPE Q, K and V quantized by
    absmax to unsigned integers; Table 3's "4-bit Q, 3-bit KV" and "4-bit QKV"
    rows).  The pages give the quantizer, not the attention; the reading used is
    softmax attention over the dequantized codes:

      q_hat = (q_code - 8) * q_scale                      (4-bit Q)
      k_hat_t = (k_code_t - 2^(b-1)) * k_scale_t          (b = kv_bits; the BOS
      v_hat_t = (v_code_t - 2^(b-1)) * v_scale_t           position of a 3-bit
                                                           cache is 4-bit: offset 8)
      s_t = softmax_scale * <q_hat, k_hat_t>,  p = softmax(s) over the allowed t,
      o = sum_t p_t * v_hat_t.

    The M queries are the cache's last M positions: query m sits at position
    T - M + m and attends positions 0 .. T - M + m (causal).
    q_codes_u: [M, H, D] unsigned 4-bit codes; q_scale: [M, H].  k_codes_u,
    v_codes_u: [T, H, D] unsigned codes as ``kv_quant`` returns them; k_scale,
    v_scale: [T, H].  softmax_scale: fp32 value (default fp32(1/sqrt(D))).
    heads: optional list of heads to compute (others are left NaN).
    Returns o: fp64 [M, H, D]."""
    q = np.asarray(q_codes_u)
    k = np.asarray(k_codes_u)
    v = np.asarray(v_codes_u)
    M, H, D = q.shape
    T = k.shape[0]
    if k.shape != (T, H, D) or v.shape != (T, H, D) or kv_bits not in (3, 4) or not 1 <= M <= T:
        raise ValueError("attention_lowbit: bad shapes or kv_bits")
    if softmax_scale is None:
        softmax_scale = np.float32(1.0 / np.sqrt(D))
    sm = float(np.float32(softmax_scale))
    offset = np.full(T, float(1 << (kv_bits - 1)))
    if kv_bits == 3 and 0 <= bos_pos < T:
        offset[bos_pos] = 8.0
    qs = np.asarray(q_scale, np.float32).astype(np.float64)
    ks = np.asarray(k_scale, np.float32).astype(np.float64)
    vs = np.asarray(v_scale, np.float32).astype(np.float64)
    out = np.full((M, H, D), np.nan)
    for h in (range(H) if heads is None else heads):
        k_hat = (k[:, h, :].astype(np.float64) - offset[:, None]) * ks[:, h, None]
        v_hat = (v[:, h, :].astype(np.float64) - offset[:, None]) * vs[:, h, None]
        for m in range(M):
            last = T - M + m
            q_hat = (q[m, h, :].astype(np.float64) - 8.0) * qs[m, h]
            s = sm * (k_hat[:last + 1] @ q_hat)
            e = np.exp(s - s.max())
            out[m, h] = (e @ v_hat[:last + 1]) / e.sum()
    return out


# ---------------------------------------------------------------------------
# Storage layouts, written from the C header's layout statements.
# ---------------------------------------------------------------------------
def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit fields per byte along the last axis: element 2i in bits 0-3,
    element 2i+1 in bits 4-7 (two's complement for INT4, the E2M1 encoding
    for FP4)."""
    c = np.asarray(codes).astype(np.int16) & 0xF
    lo = c[..., 0::2]
    hi = c[..., 1::2]
    return (lo | (hi << 4)).astype(np.uint8)


def pack_ternary2(t: np.ndarray) -> np.ndarray:
    """Four 2-bit ternary codes per byte along K: element 4i in bits 0-1;
    0 -> 00, +1 -> 01, -1 -> 11."""
    c = np.asarray(t).astype(np.int16) & 0x3
    out = c[..., 0::4] | (c[..., 1::4] << 2) | (c[..., 2::4] << 4) | (c[..., 3::4] << 6)
    return out.astype(np.uint8)


def pack_ternary_e2m1(t: np.ndarray) -> np.ndarray:
    """Ternary codes as E2M1 nibbles along K (the FP4 tensor-core weight layout):
    0 -> 0x0 (+0), +1 -> 0x2 (exponent 1, mantissa 0), -1 -> 0xA (sign | 0x2);
    element 2i in bits 0-3."""
    c = np.asarray(t).astype(np.int16)
    e = np.where(c > 0, 0x2, np.where(c < 0, 0xA, 0x0)).astype(np.int16)
    return pack_nibbles(e)


def pack_mask_bits(mask: np.ndarray) -> np.ndarray:
    """Mask bits per row in uint32 words: bit j of word w is element 32w + j;
    rows padded to a whole number of words."""
    m = np.asarray(mask).astype(np.uint8)
    M, K = m.shape
    W = (K + 31) // 32
    padded = np.zeros((M, W * 32), np.uint8)
    padded[:, :K] = m
    bits = padded.reshape(M, W, 32).astype(np.uint64)
    words = np.zeros((M, W), np.uint64)
    for j in range(32):
        words |= bits[:, :, j] << np.uint64(j)
    return words.astype(np.uint32)


def pack_kv3(codes_u: np.ndarray) -> np.ndarray:
    """Eight 3-bit codes per 3 bytes along the last axis: code j of a group in
    bits 3j..3j+2 of a little-endian 24-bit word."""
    c = np.asarray(codes_u).astype(np.uint32)
    *lead, D = c.shape
    g = c.reshape(*lead, D // 8, 8)
    word = np.zeros(g.shape[:-1], np.uint32)
    for j in range(8):
        word |= g[..., j] << np.uint32(3 * j)
    out = np.stack([(word >> s) & 0xFF for s in (0, 8, 16)], axis=-1).astype(np.uint8)
    return out.reshape(*lead, D // 8 * 3)
