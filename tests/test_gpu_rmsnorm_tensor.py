"""GPU parity of the RMSNorm-fused 4-bit quantizer (bitlinear_rmsnorm_quant_a4)
and of the per-tensor INT4 quantizer (bitlinear_quant_a4_per_tensor) against the
CPU oracle, through the C ABI: codes, scales and beta bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_bit_activation_b200 as tba
from gpu_util import CANARY, canaried, canary_bytes, canary_margins_intact, empty, host, to_dev

pytestmark = pytest.mark.gpu

EPS = 1e-5
EPS_N = 1e-6

QUANTS = {tba.BL_QUANT_INT4: "int4", tba.BL_QUANT_FP4_E2M1: "fp4"}


def rows(name):
    g = synth.rng(abs(hash(name)) % 1000)
    if name == "gauss_M37_K1536":
        return synth.gaussian_bf16(g, (37, 1536))
    if name == "studentt_K3200":
        return synth.student_t_bf16(g, (9, 3200))
    if name == "K8_min":
        return synth.gaussian_bf16(g, (5, 8))
    if name == "K16384_max":
        return synth.gaussian_bf16(g, (3, 16384))
    if name == "wide_in_contract":
        x = synth.gaussian_bf16(g, (6, 4096))
        x[0, :3] = synth.f32_to_bf16_bits(np.array([1e-6, 3e3, -7e-7], np.float32))   # squares span ~80 bits
        x[1] = synth.f32_to_bf16_bits(np.full(4096, 2.0 ** -60, np.float32))          # tiny constant row
        x[2, ::2] = 0
        return x
    if name == "midpoint_rows":
        # mean(x^2) exactly on an fp32 midpoint (6 + 2^-22 over 8 = 0.75 + 2^-25: ties to
        # 0.75), just above it (+ 2^-60: rounds up), and the same with zeros past the
        # squares: the fast sum cannot settle these, the exact path must
        f = lambda v: synth.f32_to_bf16_bits(np.array([v], np.float32))
        r = [f([1, 1, 1, 1, 1, 1, 2.0 ** -11, 0]), f([1, 1, 1, 1, 1, 1, 2.0 ** -11, 2.0 ** -30]),
             f([-1, 1, -1, 1, -1, 1, -2.0 ** -11, 0]), f([0.5, 0.5, 0.5, 0.5, 0.5, 0.5, 2.0 ** -12, 0])]
        return np.concatenate(r)
    if name == "zeros_consts":
        return np.concatenate([np.zeros((2, 256), np.uint16),
                               synth.f32_to_bf16_bits(np.full((2, 256), -0.75, np.float32)),
                               synth.student_t_bf16(g, (4, 256))])
    raise KeyError(name)


ROWS = ["gauss_M37_K1536", "studentt_K3200", "K8_min", "K16384_max", "wide_in_contract", "midpoint_rows",
        "zeros_consts"]


def gamma_for(K, kind):
    if kind == "none":
        return None
    g = synth.rng(K)
    return (1.0 + 0.3 * g.standard_normal(K)).astype(np.float32)


def run_rmsnorm_quant(x, gamma, quant, store):
    M, K = x.shape
    codes = empty((M, K // 2 if store == tba.BL_STORE_PACKED else K), torch.uint8)
    scale = empty((M,), torch.float32)
    tba.bitlinear_rmsnorm_quant_a4(to_dev(x), codes, scale, gamma=None if gamma is None else to_dev(gamma),
                                   eps_norm=EPS_N, quant=quant, store=store, eps=EPS)
    tba.sync_status()
    return host(codes), host(scale)


def expected(x, gamma, quant, store):
    """The oracle's codes in the layout of `store`, and the scale the call writes."""
    y, _ = oracle.rmsnorm(x, gamma, EPS_N)
    if quant == tba.BL_QUANT_INT4:
        c, _, s = oracle.quant_int4(y, EPS)
        return (oracle.pack_nibbles(c) if store == tba.BL_STORE_PACKED else c.view(np.uint8)), s
    code4, twice, _, s = oracle.quant_fp4(y)
    if store == tba.BL_STORE_PACKED:
        return oracle.pack_nibbles(code4), s
    return twice.view(np.uint8), (s / 2).astype(np.float32)


@pytest.mark.parametrize("name", ROWS)
@pytest.mark.parametrize("gk", ["none", "weight"])
@pytest.mark.parametrize("quant", list(QUANTS), ids=list(QUANTS.values()))
@pytest.mark.parametrize("store", [tba.BL_STORE_PACKED, tba.BL_STORE_BYTES], ids=["packed", "bytes"])
def test_rmsnorm_quant_parity(name, gk, quant, store):
    x = rows(name)
    gamma = gamma_for(x.shape[1], gk)
    codes, scale = run_rmsnorm_quant(x, gamma, quant, store)
    c_ref, s_ref = expected(x, gamma, quant, store)
    assert np.array_equal(codes, c_ref)
    assert np.array_equal(scale.view(np.uint32), s_ref.view(np.uint32))


@pytest.mark.parametrize("variant", [tba.BL_QUANT_INT4_ABSMAX, tba.BL_QUANT_INT4_ABSMEAN2, tba.BL_QUANT_FP4_E1M2],
                         ids=["int4_absmax", "int4_absmean2", "fp4_e1m2"])
def test_rmsnorm_quant_variants(variant):
    x = rows("studentt_K3200")
    gamma = gamma_for(3200, "weight")
    codes, scale = run_rmsnorm_quant(x, gamma, variant, tba.BL_STORE_BYTES)
    y, _ = oracle.rmsnorm(x, gamma, EPS_N)
    if variant == tba.BL_QUANT_INT4_ABSMAX:
        c, _, s = oracle.quant_int4_absmax(y, EPS)
        ref = c.view(np.uint8)
    elif variant == tba.BL_QUANT_INT4_ABSMEAN2:
        c, _, s = oracle.quant_int4_absmean2(y, EPS)
        ref = c.view(np.uint8)
    else:
        _, four, _, s = oracle.quant_fp4_e1m2(y)
        ref, s = four.view(np.uint8), (s / 4).astype(np.float32)
    assert np.array_equal(codes, ref)
    assert np.array_equal(scale.view(np.uint32), s.view(np.uint32))


@pytest.mark.slow
def test_rmsnorm_quant_full_7b():
    """The QKV input of a 7B prefill step: 32768 x 4096, with a norm weight, every row."""
    x = synth.gaussian_bf16(synth.rng(71), (32768, 4096))
    gamma = gamma_for(4096, "weight")
    codes, scale = run_rmsnorm_quant(x, gamma, tba.BL_QUANT_INT4, tba.BL_STORE_BYTES)
    c_ref, s_ref = expected(x, gamma, tba.BL_QUANT_INT4, tba.BL_STORE_BYTES)
    assert np.array_equal(codes, c_ref)
    assert np.array_equal(scale.view(np.uint32), s_ref.view(np.uint32))


# ---------------------------------------------------------------------------
# per-tensor INT4
# ---------------------------------------------------------------------------
def run_per_tensor(x, store):
    M, K = x.shape
    codes = empty((M, K // 2 if store == tba.BL_STORE_PACKED else K), torch.uint8)
    scale = empty((M,), torch.float32)
    beta = empty((1,), torch.float32)
    ws = empty((tba.workspace_size("quant_a4_per_tensor") // 8,), torch.int64)
    tba.bitlinear_quant_a4_per_tensor(to_dev(x), codes, scale, beta, ws, store=store, eps=EPS)
    tba.sync_status()
    return host(codes), host(scale), host(beta)


PT_CASES = [("tiny", lambda: synth.tiny_inputs(0)[0]),
            ("one_row", lambda: synth.gaussian_bf16(synth.rng(81), (1, 3200))),
            ("M700_K1536", lambda: synth.gaussian_bf16(synth.rng(82), (700, 1536))),
            ("heavy_tailed_K4096", lambda: synth.student_t_bf16(synth.rng(83), (300, 4096))),
            ("K8", lambda: synth.gaussian_bf16(synth.rng(84), (9, 8))),
            ("zeros", lambda: np.zeros((4, 64), np.uint16))]


@pytest.mark.parametrize("name,make", PT_CASES, ids=[c[0] for c in PT_CASES])
@pytest.mark.parametrize("store", [tba.BL_STORE_PACKED, tba.BL_STORE_BYTES], ids=["packed", "bytes"])
def test_quant_per_tensor_parity(name, make, store):
    x = make()
    codes, scale, beta = run_per_tensor(x, store)
    c_ref, b_ref, s_ref = oracle.quant_int4_per_tensor(x, EPS)
    assert beta.view(np.uint32)[0] == np.float32(b_ref).view(np.uint32)
    assert np.array_equal(codes, oracle.pack_nibbles(c_ref) if store == tba.BL_STORE_PACKED else c_ref.view(np.uint8))
    assert np.array_equal(scale.view(np.uint32), s_ref.view(np.uint32))
    # two calls in a row give the same beta (the workspace is cleared by the call)
    assert run_per_tensor(x, store)[2].view(np.uint32)[0] == beta.view(np.uint32)[0]


@pytest.mark.slow
def test_quant_per_tensor_full_7b():
    x = synth.gaussian_bf16(synth.rng(85), (32768, 4096))
    codes, scale, beta = run_per_tensor(x, tba.BL_STORE_BYTES)
    c_ref, b_ref, s_ref = oracle.quant_int4_per_tensor(x, EPS)
    assert beta.view(np.uint32)[0] == np.float32(b_ref).view(np.uint32)
    assert np.array_equal(codes.view(np.int8), c_ref)
    assert np.array_equal(scale.view(np.uint32), s_ref.view(np.uint32))


# ---------------------------------------------------------------------------
# no writes outside the outputs
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("store", [tba.BL_STORE_PACKED, tba.BL_STORE_BYTES], ids=["packed", "bytes"])
@pytest.mark.parametrize("M,K", [(37, 1536), (9, 3200), (5, 8)])
def test_new_quantizers_in_bounds(store, M, K):
    x = to_dev(synth.gaussian_bf16(synth.rng(M + K), (M, K)))
    width = K // 2 if store == tba.BL_STORE_PACKED else K
    codes = canaried((M, width), torch.uint8)
    scale = canaried((M,), torch.float32)
    tba.bitlinear_rmsnorm_quant_a4(x, codes[0], scale[0], gamma=to_dev(gamma_for(K, "weight")), eps_norm=EPS_N,
                                   store=store, eps=EPS)
    tba.sync_status()
    for t, buf in (codes, scale):
        assert canary_margins_intact(t, buf) and np.any(canary_bytes(t) != CANARY)
    codes = canaried((M, width), torch.uint8)
    scale = canaried((M,), torch.float32)
    beta = canaried((1,), torch.float32)
    ws = canaried((tba.workspace_size("quant_a4_per_tensor"),), torch.uint8)
    tba.bitlinear_quant_a4_per_tensor(x, codes[0], scale[0], beta[0], ws[0], store=store, eps=EPS)
    tba.sync_status()
    for t, buf in (codes, scale, beta):
        assert canary_margins_intact(t, buf) and np.any(canary_bytes(t) != CANARY)
    assert canary_margins_intact(*ws)


def test_rmsnorm_midpoint_rows_take_the_exact_mean():
    # the oracle's r for these rows follows ms = 0.75 (the tie to even) and 0.75 + 2^-24
    y, r = oracle.rmsnorm(rows("midpoint_rows"), None, EPS_N)
    s0 = np.sqrt(np.float32(0.75) + np.float32(EPS_N), dtype=np.float32)
    s1 = np.sqrt(np.float32(0.75 + 2.0 ** -24) + np.float32(EPS_N), dtype=np.float32)
    assert float(r[0]) == float(np.float32(1) / s0) and float(r[1]) == float(np.float32(1) / s1)
    codes, scale = run_rmsnorm_quant(rows("midpoint_rows"), None, tba.BL_QUANT_INT4, tba.BL_STORE_BYTES)
    c_ref, s_ref = expected(rows("midpoint_rows"), None, tba.BL_QUANT_INT4, tba.BL_STORE_BYTES)
    assert np.array_equal(codes, c_ref) and np.array_equal(scale.view(np.uint32), s_ref.view(np.uint32))
