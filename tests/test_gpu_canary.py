"""No call of the path writes outside its output buffers.  Each output lies
inside a canary-filled byte buffer (gpu_util.canaried); after the call, on
ragged shapes, the margins before and after every output, and the unused tail
of each row of a strided GEMM output, must still hold the canary.  The values
themselves are compared with the oracle by the parity tests; here the outputs
only have to have been written."""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_bit_activation_b200 as tba
from gpu_util import CANARY, canaried, canary_bytes, canary_margins_intact, empty, to_dev

pytestmark = pytest.mark.gpu

EPS = 1e-5


def check(*outputs):
    tba.sync_status()
    for t, buf in outputs:
        assert canary_margins_intact(t, buf)
        assert np.any(canary_bytes(t) != CANARY)


@pytest.mark.parametrize("quant", [tba.BL_QUANT_INT4, tba.BL_QUANT_FP4_E2M1], ids=["int4", "fp4"])
@pytest.mark.parametrize("store", [tba.BL_STORE_PACKED, tba.BL_STORE_BYTES], ids=["packed", "bytes"])
@pytest.mark.parametrize("M,K", [(37, 1536), (9, 3200), (5, 8)])
def test_quant_a4_in_bounds(quant, store, M, K):
    x = synth.gaussian_bf16(synth.rng(M + K), (M, K))
    codes = canaried((M, K // 2 if store == tba.BL_STORE_PACKED else K), torch.uint8)
    scale = canaried((M,), torch.float32)
    tba.bitlinear_quant_a4(to_dev(x), codes[0], scale[0], quant=quant, store=store, eps=EPS)
    check(codes, scale)


@pytest.mark.parametrize("M,K,keep", [(9, 40, 13), (7, 3200, 1600), (12, 4096, 2048)])
def test_sparsify_a8_in_bounds(M, K, keep):
    x = synth.student_t_bf16(synth.rng(K + keep), (M, K))
    codes = canaried((M, K), torch.int8)
    scale = canaried((M,), torch.float32)
    mask = canaried((M, (K + 31) // 32), torch.int32)
    tba.bitlinear_sparsify_a8(to_dev(x), keep, codes[0], scale[0], mask[0], eps=EPS)
    check(codes, scale, mask)


@pytest.mark.parametrize("M,F,keep,shift", [(5, 40, 7, 0.0), (6, 11008, 5504, -0.454), (7, 2048, 300, 0.0)])
def test_relu2_glu_in_bounds(M, F, keep, shift):
    gate, up = synth.glu_inputs(M, F, seed=F + M, gate_shift=shift)
    both = np.zeros((M, 2 * F), np.uint16)
    both[:, :F] = up
    both[:, F:] = gate
    d = to_dev(both)
    codes = canaried((M, F), torch.int8)
    scale = canaried((M,), torch.float32)
    mask = canaried((M, (F + 31) // 32), torch.int32)
    tba.relu2_glu(d[:, F:], d[:, :F], keep, codes[0], scale[0], mask[0], eps=EPS, M=M, F=F, ld=2 * F)
    check(codes, scale, mask)


@pytest.mark.parametrize("D", [32, 128])
@pytest.mark.parametrize("bits,bos_pos", [(3, 0), (4, -1)])
def test_kv_quant3_in_bounds(D, bits, bos_pos):
    T, H = 37, 5
    k, _ = synth.kv_inputs(D, positions=T, heads=H, head_dim=D)
    d = to_dev(np.ascontiguousarray(k.reshape(T, H * D)))
    codes = canaried((T, H, D * bits // 8), torch.uint8)
    scale = canaried((T, H), torch.float32)
    bos = canaried((H, D // 2), torch.uint8)
    tba.kv_quant3(d, T, H, D, codes[0], scale[0], bos_codes=bos[0], bits=bits, bos_pos=bos_pos, eps=EPS,
                  ldt=d.stride(0))
    outputs = [codes, scale] + ([bos] if bos_pos >= 0 else [])
    check(*outputs)
    if bos_pos < 0:
        assert canary_margins_intact(*bos) and np.all(canary_bytes(bos[0]) == CANARY)   # untouched


@pytest.mark.parametrize("wfmt,width", [(tba.BL_W_I8, 1), (tba.BL_W_T2, 4), (tba.BL_W_E2M1, 2)],
                         ids=["i8", "t2", "e2m1"])
def test_pack_ternary_in_bounds(wfmt, width):
    N, K = 37, 336
    w = (synth.rng(31).standard_normal((N, K)) * 0.02).astype(np.float32)
    out = canaried((N, K // width), torch.uint8)
    alpha = canaried((1,), torch.float32)
    ws = empty((tba.workspace_size("pack_ternary") // 8,), torch.int64)
    tba.pack_ternary(to_dev(w), alpha[0], out[0], wfmt, ws, eps=EPS)
    check(out, alpha)


# (M, N, K, weight layout): the tensor-core GEMM with int8 weights, the decode
# tensor-core kernel, the dp4a / warp-MMA GEMVs and the streaming GEMV on 2-bit weights
GEMM_CASES = [
    (200, 300, 320, tba.BL_W_I8),
    (257, 520, 3200, tba.BL_W_I8),
    (8, 300, 320, tba.BL_W_T2),
    (3, 37, 11008, tba.BL_W_T2),
    (9, 130, 832, tba.BL_W_T2),
    (1, 4736, 640, tba.BL_W_T2),
    (2, 96, 640, tba.BL_W_T2),
]


@pytest.mark.parametrize("M,N,K,wfmt", GEMM_CASES, ids=[f"{c[0]}x{c[1]}x{c[2]}_{'i8' if c[3] == tba.BL_W_I8 else 't2'}"
                                                         for c in GEMM_CASES])
def test_gemm_in_bounds(M, N, K, wfmt):
    g = synth.rng(M * 7 + N + K)
    a = g.integers(-128, 128, (M, K)).astype(np.int8)
    scale = (g.random(M) * 0.1 + 1e-3).astype(np.float32)
    t = g.integers(-1, 2, (N, K)).astype(np.int8)
    w = oracle.pack_ternary2(t) if wfmt == tba.BL_W_T2 else t
    ldy = (N + 7) // 8 * 8
    y = canaried((M, ldy), torch.int16)
    acc = canaried((M, N), torch.int32)
    al = to_dev(np.array([0.0211], np.float32))
    tba.bitlinear_gemm(to_dev(a), to_dev(scale), to_dev(w), al, M, N, K, y=y[0], acc=acc[0], afmt=tba.BL_A_I8,
                       wfmt=wfmt, ldy=ldy)
    check(y, acc)
    # the columns between N and the row stride are not part of the output
    assert np.all(canary_bytes(y[0])[:, 2 * N:] == CANARY)


def test_pack_ternary_noalloc_in_bounds():
    N, K = 37, 336
    w = (synth.rng(32).standard_normal((N, K)) * 0.02).astype(np.float32)
    for wfmt, width in ((tba.BL_W_T2, 4), (tba.BL_W_E2M1, 2)):
        out = canaried((N, K // width), torch.uint8)
        alpha = canaried((1,), torch.float32)
        tba.pack_ternary_noalloc(to_dev(w), alpha[0], out[0], wfmt, eps=EPS)
        check(out, alpha)


# (M, N, K): the fused-prologue decode GEMV (M <= 8, 2-bit weights) and the
# quantizer-into-workspace path (M > 8, or int8 weights)
QG_CASES = [(1, 300, 832, tba.BL_W_T2), (2, 37, 4096, tba.BL_W_T2), (7, 130, 640, tba.BL_W_T2),
            (13, 300, 320, tba.BL_W_T2), (200, 300, 320, tba.BL_W_I8)]


@pytest.mark.parametrize("quant", [tba.BL_QUANT_INT4, tba.BL_QUANT_FP4_E2M1], ids=["int4", "fp4"])
@pytest.mark.parametrize("M,N,K,wfmt", QG_CASES, ids=[f"{c[0]}x{c[1]}x{c[2]}" for c in QG_CASES])
def test_quant_gemm_in_bounds(quant, M, N, K, wfmt):
    g = synth.rng(M * 11 + N + K)
    x = synth.gaussian_bf16(g, (M, K))
    t = g.integers(-1, 2, (N, K)).astype(np.int8)
    w = oracle.pack_ternary2(t) if wfmt == tba.BL_W_T2 else t
    ldy = (N + 7) // 8 * 8
    y = canaried((M, ldy), torch.int16)
    acc = canaried((M, N), torch.int32)
    ws_bytes = tba.workspace_size("quant_gemm", M, N, K)
    ws = canaried((ws_bytes,), torch.uint8)
    al = to_dev(np.array([0.0211], np.float32))
    tba.bitlinear_quant_gemm(to_dev(x), to_dev(w), al, M, N, K, y=y[0], acc=acc[0], quant=quant, wfmt=wfmt,
                             eps=EPS, ldy=ldy, workspace=ws[0])
    check(y, acc)
    assert canary_margins_intact(*ws)
    assert np.all(canary_bytes(y[0])[:, 2 * N:] == CANARY)


@pytest.mark.parametrize("M,F,K", [(1, 37, 640), (2, 300, 4096), (2, 4, 64)])
def test_gemm_gated_in_bounds(M, F, K):
    g = synth.rng(M * 13 + F + K)
    a = g.integers(-8, 8, (M, K)).astype(np.int8)
    scale = (g.random(M) * 0.1 + 1e-3).astype(np.float32)
    t = g.integers(-1, 2, (2 * F, K)).astype(np.int8)
    ldy = (2 * F + 7) // 8 * 8 + 8
    y = canaried((M, ldy), torch.int16)
    acc = canaried((M, 2 * F), torch.int32)
    al = to_dev(np.array([0.0211, 0.0187], np.float32))
    tba.bitlinear_gemm_gated(to_dev(a), to_dev(scale), to_dev(oracle.pack_ternary2(t)), al, M, F, K, y[0],
                             acc=acc[0], ldy=ldy)
    check(y, acc)
    assert np.all(canary_bytes(y[0])[:, 4 * F:] == CANARY)


@pytest.mark.parametrize("M,N,K", [(200, 300, 320), (37, 230, 576), (300, 450, 4160)])
def test_gemm_fp4_mxf4_in_bounds(M, N, K):
    g = synth.rng(M * 17 + N + K)
    x = synth.gaussian_bf16(g, (M, K))
    codes, _, _, p2 = oracle.quant_fp4(x)
    a = oracle.pack_nibbles(codes)
    t = g.integers(-1, 2, (N, K)).astype(np.int8)
    ldy = (N + 7) // 8 * 8
    y = canaried((M, ldy), torch.int16)
    acc = canaried((M, N), torch.int32)
    al = to_dev(np.array([0.0211], np.float32))
    tba.bitlinear_gemm(to_dev(a), to_dev(p2.astype(np.float32)), to_dev(oracle.pack_ternary_e2m1(t)), al, M, N, K,
                       y=y[0], acc=acc[0], afmt=tba.BL_A_E2M1, wfmt=tba.BL_W_E2M1, ldy=ldy)
    check(y, acc)
    assert np.all(canary_bytes(y[0])[:, 2 * N:] == CANARY)
