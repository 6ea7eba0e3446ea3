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
