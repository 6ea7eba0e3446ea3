"""Helpers shared by the GPU parity tests: move seeded host inputs to the
device, pull results back as numpy, and the bf16 tolerance of the GEMM
output."""
import numpy as np
import torch

import synth


def device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


def to_dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    elif a.dtype == np.uint32:
        a = a.view(np.int32)
    elif a.dtype == np.uint64:
        a = a.view(np.int64)
    return torch.from_numpy(a).to(device())


def empty(shape, dtype) -> torch.Tensor:
    return torch.empty(shape, dtype=dtype, device=device())


def host(t: torch.Tensor, np_dtype=None) -> np.ndarray:
    torch.cuda.synchronize()
    a = t.detach().cpu().numpy()
    return a.view(np_dtype) if np_dtype is not None else a


def bf16_rows_rel_err(y_gpu_bits: np.ndarray, exact: np.ndarray) -> float:
    """max over rows of  max_n |y_gpu - exact| / ||exact_row||_2  (fp64)."""
    y = synth.bf16_bits_to_f32(y_gpu_bits).astype(np.float64)
    num = np.abs(y - exact).max(axis=1)
    den = np.linalg.norm(exact, axis=1)
    den = np.where(den == 0, 1.0, den)
    return float((num / den).max())


# bf16 outputs: relative error per row (max |err| over the row's fp64 norm)
BF16_ROW_TOL = 1e-2


# Out-of-bounds write check without a sanitizer: an output tensor sits inside a
# larger byte buffer; the margins on both sides and the tensor itself start as
# CANARY bytes, and after the call the margins must still hold them.
CANARY = 0xA5
CANARY_PAD = 4096       # bytes on each side; a multiple of 16 keeps the tensor aligned


def canaried(shape, dtype, dev=None):
    """(tensor of `shape` and `dtype`, the buffer around it), all bytes CANARY."""
    dev = device() if dev is None else dev
    nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    buf = torch.full((2 * CANARY_PAD + nbytes,), CANARY, dtype=torch.uint8, device=dev)
    return buf[CANARY_PAD:CANARY_PAD + nbytes].view(dtype).view(*shape), buf


def canary_margins_intact(t: torch.Tensor, buf: torch.Tensor) -> bool:
    """True if no byte of buf outside tensor t differs from CANARY."""
    if buf.is_cuda:
        torch.cuda.synchronize()
    b = buf.cpu().numpy()
    nbytes = t.numel() * t.element_size()
    return bool(np.all(b[:CANARY_PAD] == CANARY) and np.all(b[CANARY_PAD + nbytes:] == CANARY))


def canary_bytes(t: torch.Tensor) -> np.ndarray:
    """The bytes of tensor t, row by row (uint8 [rows x row bytes])."""
    if t.is_cuda:
        torch.cuda.synchronize()
    a = t.detach().cpu().contiguous().view(torch.uint8).numpy()
    return a.reshape(t.shape[0], -1) if t.dim() > 1 else a.reshape(1, -1)
