"""Python binding of libbitlinear, the sm_100a implementation of the BitNet a4.8
BitLinear forward path (arXiv 2411.04965, §3.4).

Argument marshalling only: every function below forwards device pointers,
sizes and the current CUDA stream to the C entry point of the same name in
``libbitlinear.so`` (declared in ``include/bitlinear.h``) and raises on a
non-OK status.  All arithmetic runs in the library's kernels.  Device memory
is allocated by the caller (PyTorch tensors); nothing here falls back to a
CPU or PyTorch implementation -- if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitlinear.so")

# enums of include/bitlinear.h
BL_OK = 0
STATUS_NAMES = ["BL_OK", "BL_ERR_NULL", "BL_ERR_ALIGN", "BL_ERR_SHAPE", "BL_ERR_ARG", "BL_ERR_UNSUPPORTED",
                "BL_ERR_CUDA", "BL_ERR_TIMEOUT", "BL_ERR_WORKSPACE"]
BL_ERR_CUDA = STATUS_NAMES.index("BL_ERR_CUDA")
BL_QUANT_INT4, BL_QUANT_FP4_E2M1, BL_QUANT_INT4_ABSMAX, BL_QUANT_INT4_ABSMEAN2, BL_QUANT_FP4_E1M2 = 0, 1, 2, 3, 4
BL_STORE_PACKED, BL_STORE_BYTES = 0, 1
BL_A_I8, BL_A_I4, BL_A_E2M1 = 0, 1, 2
BL_W_T2, BL_W_I8, BL_W_E2M1 = 0, 1, 2

EXPORTED = ["bitlinear_quant_a4", "bitlinear_rmsnorm_quant_a4", "bitlinear_quant_a4_per_tensor",
            "bitlinear_sparsify_a8", "pack_ternary", "pack_ternary_noalloc", "bitlinear_gemm",
            "bitlinear_quant_gemm", "bitlinear_gemm_gated", "relu2_glu", "kv_quant3", "attention_lowbit",
            "bitlinear_workspace_size",
            "bitlinear_sync_status", "bitlinear_selftest_timeout", "bitlinear_status_string",
            "bitlinear_last_cuda_error", "bitlinear_version"]

_lib = None


class BitLinearError(RuntimeError):
    def __init__(self, fn: str, status: int, cuda_error: str = ""):
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else f"status {status}"
        detail = f" ({cuda_error})" if cuda_error else ""
        super().__init__(f"{fn} failed: {name}{detail}")
        self.status = status
        self.cuda_error = cuda_error


def lib():
    """Load libbitlinear.so (built in-tree by ``build.py``); raise if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m ternary_bit_activation_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, F, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int
        sig = {
            "bitlinear_quant_a4": [P, I64, I64, I64, I, I, F, P, P, P],
            "bitlinear_rmsnorm_quant_a4": [P, I64, I64, I64, P, F, I, I, F, P, P, P],
            "bitlinear_quant_a4_per_tensor": [P, I64, I64, I64, I, F, P, P, P, P, ctypes.c_size_t, P],
            "bitlinear_sparsify_a8": [P, I64, I64, I64, I64, F, P, P, P, P],
            "pack_ternary": [P, I64, I64, I64, F, I, P, I, P, P, ctypes.c_size_t, P],
            "pack_ternary_noalloc": [P, I64, I64, I64, F, I, P, I, P, P],
            "bitlinear_gemm": [P, I, P, P, I, P, I64, I64, I64, I64, P, I64, P, P],
            "bitlinear_quant_gemm": [P, I64, I, F, P, I, P, I64, I64, I64, I64, P, I64, P, P, ctypes.c_size_t, P],
            "bitlinear_gemm_gated": [P, I, P, P, I, P, I64, I64, I64, P, I64, P, P],
            "relu2_glu": [P, P, I64, I64, I64, I64, F, P, P, P, P],
            "kv_quant3": [P, I64, I64, I64, I64, I, I64, F, P, P, P, P],
            "attention_lowbit": [P, P, I64, P, P, P, P, P, P, I64, I64, I64, I, I64, F, P, I64, P, ctypes.c_size_t,
                                 P],
            "bitlinear_sync_status": [P],
            "bitlinear_selftest_timeout": [P],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.bitlinear_workspace_size.argtypes = [ctypes.c_char_p, I64, I64, I64]
        L.bitlinear_workspace_size.restype = ctypes.c_size_t
        L.bitlinear_status_string.argtypes = [I]
        L.bitlinear_status_string.restype = ctypes.c_char_p
        L.bitlinear_last_cuda_error.argtypes = []
        L.bitlinear_last_cuda_error.restype = ctypes.c_char_p
        L.bitlinear_version.argtypes = []
        L.bitlinear_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(fn: str, rc: int):
    if rc != BL_OK:
        raise BitLinearError(fn, rc, last_cuda_error() if rc == BL_ERR_CUDA else "")


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------
def bitlinear_quant_a4(x, codes, scale, quant=BL_QUANT_INT4, store=BL_STORE_PACKED, eps=1e-5, M=None, K=None,
                       ldx=None, stream=None):
    """INT4 absmean (Eq. 6-7) or FP4 E2M1 MinMax (Eq. 8-9) per token."""
    M = x.shape[0] if M is None else M
    K = x.shape[1] if K is None else K
    ldx = x.stride(0) if ldx is None else ldx
    _check("bitlinear_quant_a4", lib().bitlinear_quant_a4(_ptr(x), M, K, ldx, quant, store, eps, _ptr(codes),
                                                          _ptr(scale), _stream(stream)))


def bitlinear_rmsnorm_quant_a4(x, codes, scale, gamma=None, eps_norm=1e-6, quant=BL_QUANT_INT4,
                               store=BL_STORE_PACKED, eps=1e-5, ldx=None, stream=None):
    """RMSNorm (x * r * gamma, r = 1/sqrt(mean(x^2) + eps_norm)) fused into the
    4-bit quantizer: the codes and scales of bitlinear_quant_a4 on RMSNorm(x)."""
    M, K = x.shape
    ldx = x.stride(0) if ldx is None else ldx
    _check("bitlinear_rmsnorm_quant_a4", lib().bitlinear_rmsnorm_quant_a4(
        _ptr(x), M, K, ldx, _ptr(gamma), eps_norm, quant, store, eps, _ptr(codes), _ptr(scale), _stream(stream)))


def bitlinear_quant_a4_per_tensor(x, codes, scale, beta, workspace, store=BL_STORE_PACKED, eps=1e-5, ldx=None,
                                  stream=None):
    """INT4 absmean with beta = the exact mean |x| over the whole tensor."""
    M, K = x.shape
    ldx = x.stride(0) if ldx is None else ldx
    ws = workspace.numel() * workspace.element_size()
    _check("bitlinear_quant_a4_per_tensor", lib().bitlinear_quant_a4_per_tensor(
        _ptr(x), M, K, ldx, store, eps, _ptr(codes), _ptr(scale), _ptr(beta), _ptr(workspace), ws, _stream(stream)))


def bitlinear_sparsify_a8(x, k_keep, codes, scale, mask=None, eps=1e-5, stream=None):
    """Top-K (exactly k_keep per token) then INT8 absmax (Eq. 1)."""
    M, K = x.shape
    _check("bitlinear_sparsify_a8", lib().bitlinear_sparsify_a8(_ptr(x), M, K, x.stride(0), k_keep, eps, _ptr(codes),
                                                                _ptr(scale), _ptr(mask), _stream(stream)))


def pack_ternary(w, alpha, w_out, wfmt=BL_W_T2, workspace=None, alpha_given=False, eps=1e-5, stream=None):
    """Absmean ternary quantization (Eq. 2) into the 2-bit, int8 or E2M1 layout."""
    N, K = w.shape
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pack_ternary", lib().pack_ternary(_ptr(w), N, K, w.stride(0), eps, 1 if alpha_given else 0, _ptr(alpha),
                                              wfmt, _ptr(w_out), _ptr(workspace), ws, _stream(stream)))


def pack_ternary_noalloc(w, alpha, w_out, wfmt=BL_W_T2, alpha_given=False, eps=1e-5, stream=None):
    """pack_ternary without a workspace argument, for callers that cannot
    allocate device memory: the scratch lives in the library (one 2 KiB array
    per GPU).  Calls that may overlap on one GPU must be serialized."""
    N, K = w.shape
    _check("pack_ternary_noalloc", lib().pack_ternary_noalloc(_ptr(w), N, K, w.stride(0), eps,
                                                              1 if alpha_given else 0, _ptr(alpha), wfmt,
                                                              _ptr(w_out), _stream(stream)))


def bitlinear_gemm(a, a_scale, w, alpha, M, N, K, y=None, acc=None, afmt=BL_A_I8, wfmt=BL_W_I8, alpha_group=None,
                   ldy=None, stream=None):
    """y = bf16(acc * a_scale[m] * alpha[n // alpha_group]), acc = A . T^T exact."""
    group = N if alpha_group is None else alpha_group
    ldy = (y.stride(0) if y is not None else N) if ldy is None else ldy
    _check("bitlinear_gemm", lib().bitlinear_gemm(_ptr(a), afmt, _ptr(a_scale), _ptr(w), wfmt, _ptr(alpha), group,
                                                  M, N, K, _ptr(y), ldy, _ptr(acc), _stream(stream)))


def bitlinear_quant_gemm(x, w, alpha, M, N, K, y=None, acc=None, quant=BL_QUANT_INT4, wfmt=BL_W_T2, eps=1e-5,
                         alpha_group=None, ldx=None, ldy=None, workspace=None, stream=None):
    """bitlinear_quant_a4 fused into bitlinear_gemm: y from the bf16 rows x."""
    group = N if alpha_group is None else alpha_group
    ldx = x.stride(0) if ldx is None else ldx
    ldy = (y.stride(0) if y is not None else N) if ldy is None else ldy
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("bitlinear_quant_gemm", lib().bitlinear_quant_gemm(_ptr(x), ldx, quant, eps, _ptr(w), wfmt, _ptr(alpha),
                                                              group, M, N, K, _ptr(y), ldy, _ptr(acc),
                                                              _ptr(workspace), ws_bytes, _stream(stream)))


def bitlinear_gemm_gated(a, a_scale, w, alpha, M, F, K, y, acc=None, afmt=BL_A_I8, wfmt=BL_W_T2, ldy=None,
                         stream=None):
    """Gate rows of [W_up; W_gate] first, Up rows only where some token's gate > 0."""
    ldy = y.stride(0) if ldy is None else ldy
    _check("bitlinear_gemm_gated", lib().bitlinear_gemm_gated(_ptr(a), afmt, _ptr(a_scale), _ptr(w), wfmt,
                                                              _ptr(alpha), M, F, K, _ptr(y), ldy, _ptr(acc),
                                                              _stream(stream)))


def relu2_glu(gate, up, k_keep, codes, scale, mask=None, eps=1e-5, M=None, F=None, ld=None, stream=None):
    """h = up * relu(gate)^2 (Eq. 5), then Top-K + INT8 (Eq. 1) on h."""
    M = gate.shape[0] if M is None else M
    F = gate.shape[1] if F is None else F
    ld = gate.stride(0) if ld is None else ld
    _check("relu2_glu", lib().relu2_glu(_ptr(gate), _ptr(up), M, F, ld, k_keep, eps, _ptr(codes), _ptr(scale),
                                        _ptr(mask), _stream(stream)))


def kv_quant3(kv, T, H, D, codes, scale, bos_codes=None, bits=3, bos_pos=0, eps=1e-5, ldt=None, stream=None):
    """Absmax per (position, head) to unsigned 3/4-bit codes; BOS row at 4 bits."""
    ldt = H * D if ldt is None else ldt
    _check("kv_quant3", lib().kv_quant3(_ptr(kv), T, H, D, ldt, bits, bos_pos, eps, _ptr(codes), _ptr(scale),
                                        _ptr(bos_codes), _stream(stream)))


def attention_lowbit(q_codes, q_scale, M, k_codes, k_scale, v_codes, v_scale, T, H, D, out, workspace,
                     k_bos=None, v_bos=None, kv_bits=3, bos_pos=0, softmax_scale=None, ldo=None, ws_bytes=None,
                     stream=None):
    """Softmax attention of M 4-bit queries (the cache's last M positions) over
    the kv_quant3 cache of T positions; out: [M x ldo] bf16."""
    ldo = H * D if ldo is None else ldo
    if softmax_scale is None:
        softmax_scale = float(1.0 / (D ** 0.5))
    if ws_bytes is None:
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("attention_lowbit", lib().attention_lowbit(_ptr(q_codes), _ptr(q_scale), M, _ptr(k_codes), _ptr(k_scale),
                                                      _ptr(k_bos), _ptr(v_codes), _ptr(v_scale), _ptr(v_bos), T, H,
                                                      D, kv_bits, bos_pos, softmax_scale, _ptr(out), ldo,
                                                      _ptr(workspace), ws_bytes, _stream(stream)))


def workspace_size(op: str, M: int = 0, N: int = 0, K: int = 0) -> int:
    return int(lib().bitlinear_workspace_size(op.encode(), M, N, K))


def sync_status(stream=None):
    """Synchronize and raise if a kernel reported a timeout since the last check."""
    _check("bitlinear_sync_status", lib().bitlinear_sync_status(_stream(stream)))


def selftest_timeout(stream=None):
    """Enqueue a bounded wait that runs out (about 2 s); the next sync_status()
    raises BitLinearError with status BL_ERR_TIMEOUT."""
    _check("bitlinear_selftest_timeout", lib().bitlinear_selftest_timeout(_stream(stream)))


def status_string(status: int) -> str:
    return lib().bitlinear_status_string(status).decode()


def last_cuda_error() -> str:
    """Name of the CUDA error behind the last BL_ERR_CUDA on this thread."""
    return lib().bitlinear_last_cuda_error().decode()


def version() -> str:
    return lib().bitlinear_version().decode()
