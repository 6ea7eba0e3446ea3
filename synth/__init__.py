"""Seeded synthetic inputs for the BitLinear forward path of BitNet a4.8.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no quantizer, no Top-K, no matmul).  Both the CUDA path
and the CPU oracle are fed the same bytes from here, so there is no RNG skew
between them.

Value distributions follow what the BitNet a4.8 paper reports about the inputs
of each projection (§3.4, "Activation Distribution Analysis", Fig. 2):

* the attention QKV and FFN Up/Gate inputs are roughly Gaussian -> N(0, 1);
* the attention-output and FFN-down inputs are sharply peaked with long
  tails -> Student-t with nu = 3;
* latent weights are drawn N(0, 0.02) and ternarized by the method itself.

The shapes are the 700M / 3B / 7B decoder-layer shapes (hidden size, FFN width,
heads) at which the paper's tables are reported.  Every generator is a pure
function of its seed: numpy ``Generator(PCG64(seed))``.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Tuple

import numpy as np


# ----------------------------------------------------------------------------
# bf16 storage.  bf16 is stored as raw uint16 bit patterns; conversion from the
# fp32 draws rounds to nearest, ties to even, which is the storage format's own
# definition (the top 16 bits of an IEEE binary32).
# ----------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round-to-nearest-even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    if np.isnan(a).any():
        raise ValueError("NaN inputs are not generated")
    u = a.view(np.uint32)
    rounding_bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    # u + bias stays below 2^32 for every finite value (the top exponent is 0xFE)
    return ((u + rounding_bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def gaussian_bf16(g: np.random.Generator, shape, sigma: float = 1.0,
                  outlier_channels=(), outlier_scale: float = 1.0) -> np.ndarray:
    x = g.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    for c in outlier_channels:
        x[..., c] *= np.float32(outlier_scale)
    return f32_to_bf16_bits(x)


def student_t_bf16(g: np.random.Generator, shape, nu: float = 3.0) -> np.ndarray:
    x = g.standard_t(nu, size=shape)
    return f32_to_bf16_bits(x.astype(np.float32))


def latent_weights_f32(g: np.random.Generator, n: int, k: int, sigma: float = 0.02) -> np.ndarray:
    w = g.standard_normal(size=(n, k), dtype=np.float32)
    w *= np.float32(sigma)
    return w


# ----------------------------------------------------------------------------
# Workload recipes.
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class LayerShape:
    name: str
    hidden: int
    heads: int
    ffn: int
    tokens: int          # M = batch x sequence
    topk_pct_o: int      # Top-K percentage for the attention-output input
    topk_pct_down: int   # Top-K percentage for the down-projection input (100 = no Top-K)

    @property
    def head_dim(self) -> int:
        return self.hidden // self.heads

    def matrices(self) -> Dict[str, Tuple[int, int]]:
        """BitLinear weight shapes [N x K] of one decoder layer.  Up and Gate
        are stacked into one [2F x d] operand (Up rows first, Gate rows second)."""
        d, f = self.hidden, self.ffn
        return {"qkv": (3 * d, d), "o": (d, d), "upgate": (2 * f, d), "down": (d, f)}


TINY = LayerShape("tiny", hidden=256, heads=4, ffn=256, tokens=16, topk_pct_o=50, topk_pct_down=50)
L700M = LayerShape("700M", hidden=1536, heads=24, ffn=4096, tokens=8 * 512, topk_pct_o=50, topk_pct_down=50)
L3B = LayerShape("3B", hidden=3200, heads=32, ffn=8640, tokens=16 * 2048, topk_pct_o=50, topk_pct_down=50)
L7B = LayerShape("7B", hidden=4096, heads=32, ffn=11008, tokens=8 * 4096, topk_pct_o=50, topk_pct_down=50)
DECODE_TOKENS: List[int] = [1, 2, 4, 8, 16, 32, 64, 128, 256]
KV_SHAPE = (32768, 32, 128)   # positions x heads x head_dim

SHAPES = {s.name: s for s in (TINY, L700M, L3B, L7B)}
SEEDS = {"tiny": 0, "700M": 1, "3B": 2, "7B": 3, "decode": 4}


def k_keep(k: int, pct: int) -> int:
    """Number of survivors of a k%-Top-K over a row of ``k`` entries."""
    return (k * pct) // 100


def tiny_inputs(seed: int = 0):
    """16 tokens x 256 features, N(0,1) with two outlier channels x20; weights
    [256 x 256] ~ N(0, 0.02)."""
    g = rng(seed)
    x = gaussian_bf16(g, (16, 256), outlier_channels=(5, 200), outlier_scale=20.0)
    w = latent_weights_f32(g, 256, 256)
    return x, w


def layer_activations(shape: LayerShape, seed: int, tokens: int | None = None):
    """Per-layer activation inputs: attention input (Gaussian), attention-output
    input (Student-t), FFN input (Gaussian)."""
    m = shape.tokens if tokens is None else tokens
    g = rng(seed)
    x_attn = gaussian_bf16(g, (m, shape.hidden))
    x_o = student_t_bf16(g, (m, shape.hidden))
    x_ffn = gaussian_bf16(g, (m, shape.hidden))
    return x_attn, x_o, x_ffn


def layer_weights(shape: LayerShape, seed: int):
    """Latent fp32 weights of one layer, each drawn N(0, 0.02)."""
    g = rng(seed + 1000)
    out = {}
    for name, (n, k) in shape.matrices().items():
        if name == "upgate":
            f = n // 2
            out["up"] = latent_weights_f32(g, f, k)
            out["gate"] = latent_weights_f32(g, f, k)
        else:
            out[name] = latent_weights_f32(g, n, k)
    return out


def glu_inputs(m: int, f: int, seed: int, gate_shift: float = 0.0):
    """Gate and Up projections' outputs as bf16 [m x f] each (Gaussian; an
    optional negative shift of the gate raises the fraction of zero ReLU^2
    outputs toward the paper's reported gate sparsity)."""
    g = rng(seed + 2000)
    gate = g.standard_normal(size=(m, f), dtype=np.float32)
    if gate_shift:
        gate += np.float32(gate_shift)
    gate = f32_to_bf16_bits(gate)
    up = gaussian_bf16(g, (m, f))
    return gate, up


def kv_inputs(seed: int, positions: int = KV_SHAPE[0], heads: int = KV_SHAPE[1],
              head_dim: int = KV_SHAPE[2]):
    """Post-RoPE K and V, bf16 [positions x heads x head_dim] ~ N(0, 1)."""
    g = rng(seed + 3000)
    k = gaussian_bf16(g, (positions, heads, head_dim))
    v = gaussian_bf16(g, (positions, heads, head_dim))
    return k, v
