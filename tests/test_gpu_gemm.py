"""GPU parity of the ternary packer and the BitLinear GEMM (tcgen05 and
CUDA-core kernels) against the CPU oracle, through the C ABI.  alpha, packed
codes and int32 accumulators are compared bit for bit; bf16 outputs per row
within 1e-2 of the fp64 product (max |err| over the row's norm)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_bit_activation_b200 as tba
from gpu_util import BF16_ROW_TOL, bf16_rows_rel_err, empty, host, to_dev

pytestmark = pytest.mark.gpu

EPS = 1e-5


def run_pack(w, wfmt, alpha_in=None):
    N, K = w.shape
    wd = to_dev(w)
    width = {tba.BL_W_T2: K // 4, tba.BL_W_E2M1: K // 2}.get(wfmt, K)
    out = empty((N, width), torch.uint8)
    ws = empty((tba.workspace_size("pack_ternary", 0, N, K) // 8,), torch.int64)
    alpha = empty((1,), torch.float32)
    if alpha_in is not None:
        alpha.fill_(float(alpha_in))
    tba.pack_ternary(wd, alpha, out, wfmt=wfmt, workspace=ws, alpha_given=alpha_in is not None, eps=EPS)
    tba.sync_status()
    return host(out), host(alpha)[0]


def _wide_range_weights():
    # magnitudes from 2^-140 (subnormal) to 2^120, both signs
    g = synth.rng(26)
    e = g.integers(-140, 121, (64, 512))
    m = 1.0 + g.random((64, 512))
    sgn = np.where(g.random((64, 512)) < 0.5, -1.0, 1.0)
    return (sgn * m * np.exp2(e.astype(np.float64))).astype(np.float32)


def _tiny_first_weights():
    # every lane's first weight is tiny, so its window sits far below the rest
    w = synth.latent_weights_f32(synth.rng(27), 64, 1024)
    w[:, ::4] = np.float32(1e-30)
    return w


PACK_CASES = [
    ("tiny_256x256", lambda: synth.tiny_inputs(0)[1]),
    ("700M_qkv", lambda: synth.latent_weights_f32(synth.rng(21), 4608, 1536)),
    ("odd_rows_K3200", lambda: synth.latent_weights_f32(synth.rng(22), 33, 3200)),
    ("tiny_values", lambda: (synth.latent_weights_f32(synth.rng(23), 16, 64) * np.float32(1e-36))),
    ("constant", lambda: np.full((8, 64), -0.0213, np.float32)),
    ("wide_exponent_range", lambda: _wide_range_weights()),
    ("tiny_first_then_normal", lambda: _tiny_first_weights()),
    ("near_max_magnitude", lambda: (synth.latent_weights_f32(synth.rng(25), 8, 256) * np.float32(1e38))),
    ("zeros", lambda: np.zeros((4, 64), np.float32)),
]


@pytest.mark.parametrize("name,make", PACK_CASES, ids=[c[0] for c in PACK_CASES])
@pytest.mark.parametrize("wfmt", [tba.BL_W_T2, tba.BL_W_I8], ids=["t2", "i8"])
def test_pack_ternary_parity(name, make, wfmt):
    w = make()
    out, alpha = run_pack(w, wfmt)
    t_ref, a_ref = oracle.ternary_quantize(w, EPS)
    assert np.float32(alpha).view(np.uint32) == np.float32(a_ref).view(np.uint32), (alpha, a_ref)
    if wfmt == tba.BL_W_T2:
        assert np.array_equal(out, oracle.pack_ternary2(t_ref))
    else:
        assert np.array_equal(out.view(np.int8), t_ref)


def test_pack_ternary_alpha_given():
    w = synth.latent_weights_f32(synth.rng(24), 64, 256)
    for a in (0.011, 0.016, 0.05):
        out, alpha = run_pack(w, tba.BL_W_I8, alpha_in=a)
        assert alpha == np.float32(a)
        assert np.array_equal(out.view(np.int8), oracle.ternary_codes(w, np.float32(a), EPS))


def exact_y(a_codes, a_scale, t_codes, alpha, group, rows):
    al = np.atleast_1d(np.asarray(alpha, np.float64))
    N = t_codes.shape[0]
    acc = a_codes[rows].astype(np.int64) @ t_codes.astype(np.int64).T
    col_alpha = al[np.arange(N) // group]
    return acc, acc.astype(np.float64) * a_scale[rows, None].astype(np.float64) * col_alpha[None, :]


def run_gemm(a_dev, afmt, scale, w_dev, wfmt, alpha, M, N, K, group=None, want_acc=True, ldy=None):
    ldy = (N + 7) // 8 * 8 if ldy is None else ldy     # rows of y stay 16-byte aligned
    y = empty((M, ldy), torch.int16)
    acc = empty((M, N), torch.int32) if want_acc else None
    al = to_dev(np.atleast_1d(np.asarray(alpha, np.float32)))
    tba.bitlinear_gemm(a_dev, to_dev(scale), w_dev, al, M, N, K, y=y, acc=acc, afmt=afmt, wfmt=wfmt,
                       alpha_group=group, ldy=ldy)
    tba.sync_status()
    return (host(acc) if want_acc else None), host(y, np.uint16)[:, :N]


GEMM_TC_CASES = [
    ("tiny_16x256x256", 16, 256, 256),
    ("one_row", 1, 256, 128),
    ("K_tail_200x300x320", 200, 300, 320),
    ("multi_tile_384x768x1536", 384, 768, 1536),
    ("ragged_257x520x3200", 257, 520, 3200),
    ("many_tiles_1300x2304x1024", 1300, 2304, 1024),
]


@pytest.mark.parametrize("name,M,N,K", GEMM_TC_CASES, ids=[c[0] for c in GEMM_TC_CASES])
def test_gemm_tc_parity(name, M, N, K):
    g = synth.rng(M * 7 + N + K)
    a = g.integers(-128, 128, (M, K)).astype(np.int8)
    t = g.integers(-1, 2, (N, K)).astype(np.int8)
    scale = (g.random(M) * 0.1 + 1e-3).astype(np.float32)
    alpha = np.float32(0.0173)
    acc, y = run_gemm(to_dev(a), tba.BL_A_I8, scale, to_dev(t), tba.BL_W_I8, alpha, M, N, K)
    acc_ref, _ = oracle.gemm(a, scale, t, alpha, want_y=False)
    assert np.array_equal(acc, acc_ref)
    _, ex = exact_y(a, scale, t, alpha, N, np.arange(M))
    assert bf16_rows_rel_err(y, ex) <= BF16_ROW_TOL
    _, y_or = oracle.gemm(a, scale, t, alpha, rows=np.arange(min(M, 8)))
    yo = synth.bf16_bits_to_f32(y_or).astype(np.float64)
    yg = synth.bf16_bits_to_f32(y[:min(M, 8)]).astype(np.float64)
    assert np.all(np.abs(yg - yo) <= np.abs(yo) * 2.0 ** -7 + 1e-30)   # within one bf16 ulp


def test_gemm_tc_alpha_groups_and_ldy():
    # stacked Up|Gate weights with one alpha per tensor; output written into a wider row
    M, F, K = 130, 384, 512
    g = synth.rng(31)
    a = g.integers(-8, 8, (M, K)).astype(np.int8)
    t = g.integers(-1, 2, (2 * F, K)).astype(np.int8)
    scale = (g.random(M) + 0.5).astype(np.float32)
    alpha = np.array([0.0151, 0.0213], np.float32)
    acc, y = run_gemm(to_dev(a), tba.BL_A_I8, scale, to_dev(t), tba.BL_W_I8, alpha, M, 2 * F, K, group=F,
                      ldy=2 * F + 64)
    acc_ref, _ = oracle.gemm(a, scale, t, alpha, alpha_group=F, want_y=False)
    assert np.array_equal(acc, acc_ref)
    _, ex = exact_y(a, scale, t, alpha, F, np.arange(M))
    assert bf16_rows_rel_err(y, ex) <= BF16_ROW_TOL


def test_bitlinear_end_to_end_tiny():
    # the tiny configuration end to end: quantize X (INT4 and Top-K/INT8),
    # pack W, multiply -- all on the GPU -- against the oracle chain
    x, w = synth.tiny_inputs(0)
    M, K = x.shape
    N = w.shape[0]
    xd = to_dev(x)
    w8, alpha = run_pack(w, tba.BL_W_I8)
    t_ref, a_ref = oracle.ternary_quantize(w, EPS)
    codes = empty((M, K), torch.uint8)
    scale = empty((M,), torch.float32)
    tba.bitlinear_quant_a4(xd, codes, scale, quant=tba.BL_QUANT_INT4, store=tba.BL_STORE_BYTES, eps=EPS)
    al = to_dev(np.array([alpha], np.float32))
    y = empty((M, N), torch.int16)
    acc = empty((M, N), torch.int32)
    tba.bitlinear_gemm(codes, scale, to_dev(w8), al, M, N, K, y=y, acc=acc)
    tba.sync_status()
    c_ref, _, s_ref = oracle.quant_int4(x, EPS)
    acc_ref, y_ref = oracle.gemm(c_ref, s_ref, t_ref, a_ref)
    assert np.array_equal(host(acc), acc_ref)
    _, ex = exact_y(c_ref, s_ref, t_ref, a_ref, N, np.arange(M))
    assert bf16_rows_rel_err(host(y, np.uint16), ex) <= BF16_ROW_TOL
    # Top-K 50% + INT8 path
    keep = synth.k_keep(K, 50)
    c8 = empty((M, K), torch.int8)
    s8 = empty((M,), torch.float32)
    tba.bitlinear_sparsify_a8(xd, keep, c8, s8, None, eps=EPS)
    tba.bitlinear_gemm(c8, s8, to_dev(w8), al, M, N, K, y=y, acc=acc)
    tba.sync_status()
    c8_ref, _, _, s8_ref = oracle.sparsify_a8(x, keep, EPS)
    acc_ref, _ = oracle.gemm(c8_ref, s8_ref, t_ref, a_ref, want_y=False)
    assert np.array_equal(host(acc), acc_ref)


@pytest.mark.parametrize("M", [1, 2, 3, 8, 17])
@pytest.mark.parametrize("afmt", ["i8", "i4", "e2m1"])
@pytest.mark.parametrize("wfmt", [tba.BL_W_T2, tba.BL_W_I8], ids=["t2", "i8w"])
def test_gemm_simt_parity(M, afmt, wfmt):
    N, K = 96, 640
    g = synth.rng(M + 100)
    x = synth.gaussian_bf16(g, (M, K))
    w = synth.latent_weights_f32(g, N, K)
    t_ref, a_ref = oracle.ternary_quantize(w, EPS)
    wq = oracle.pack_ternary2(t_ref) if wfmt == tba.BL_W_T2 else t_ref.view(np.uint8)
    if afmt == "i8":
        a_codes, _, _, scale = oracle.sparsify_a8(x, K // 2, EPS)
        a_dev, af, acc_codes = to_dev(a_codes), tba.BL_A_I8, a_codes
        acc_scale = scale
    elif afmt == "i4":
        c, _, scale = oracle.quant_int4(x, EPS)
        a_dev, af, acc_codes = to_dev(oracle.pack_nibbles(c)), tba.BL_A_I4, c
        acc_scale = scale
    else:
        code4, twice, _, scale = oracle.quant_fp4(x)
        a_dev, af, acc_codes = to_dev(oracle.pack_nibbles(code4)), tba.BL_A_E2M1, twice
        acc_scale = (scale.astype(np.float64) / 2).astype(np.float32)
    acc, y = run_gemm(a_dev, af, scale, to_dev(wq), wfmt, a_ref, M, N, K)
    acc_ref, _ = oracle.gemm(acc_codes, acc_scale, t_ref, a_ref, want_y=False)
    assert np.array_equal(acc, acc_ref)
    _, ex = exact_y(acc_codes, acc_scale, t_ref, a_ref, N, np.arange(M))
    assert bf16_rows_rel_err(y, ex) <= BF16_ROW_TOL


# 2-bit weights x int8 activations on the tensor cores beyond the decode GEMVs
# (more than 16 tokens, or rows too long to stage the GEMV's token slots):
# weights widened into tensor memory, tokens on the MMA's N side (8 for M = 8,
# else a multiple of 16 up to 256 per token block).  The cases with up to 16
# tokens and shorter rows run on the warp-MMA GEMV.
GEMM_T2TC_CASES = [
    ("M8_long_K_24576_tc", 8, 136, 24576),
    ("M12_long_K_12288_tc", 12, 136, 12288),
    ("M16_long_K_11328_tc", 16, 300, 11328),
    ("M8_min_K", 8, 128, 64),
    ("M8_ragged_N_K_tail", 8, 300, 320),
    ("M8_two_tiles", 8, 256, 4096),
    ("M12_K_tail_1088", 12, 136, 1088),
    ("M9_nt16", 9, 130, 832),
    ("M33_nt48", 33, 384, 768),
    ("M100_nt112", 100, 200, 2048),
    ("M256_nt256", 256, 129, 512),
    ("M300_two_token_blocks", 300, 256, 256),
    ("M64_K11008_down", 64, 160, 11008),
]


@pytest.mark.parametrize("name,M,N,K", GEMM_T2TC_CASES, ids=[c[0] for c in GEMM_T2TC_CASES])
def test_gemm_t2_tensor_core_parity(name, M, N, K):
    g = synth.rng(M * 13 + N + K)
    a = g.integers(-128, 128, (M, K)).astype(np.int8)
    t = g.integers(-1, 2, (N, K)).astype(np.int8)
    scale = (g.random(M) * 0.1 + 1e-3).astype(np.float32)
    alpha = np.float32(0.0173)
    acc, y = run_gemm(to_dev(a), tba.BL_A_I8, scale, to_dev(oracle.pack_ternary2(t)), tba.BL_W_T2, alpha, M, N, K)
    acc_ref, _ = oracle.gemm(a, scale, t, alpha, want_y=False)
    assert np.array_equal(acc, acc_ref)
    _, ex = exact_y(a, scale, t, alpha, N, np.arange(M))
    assert bf16_rows_rel_err(y, ex) <= BF16_ROW_TOL


def test_gemm_t2_tensor_core_alpha_groups_and_ldy():
    M, F, K = 24, 192, 1024
    g = synth.rng(33)
    a = g.integers(-8, 8, (M, K)).astype(np.int8)
    t = g.integers(-1, 2, (2 * F, K)).astype(np.int8)
    scale = (g.random(M) + 0.5).astype(np.float32)
    alpha = np.array([0.0151, 0.0213], np.float32)
    acc, y = run_gemm(to_dev(a), tba.BL_A_I8, scale, to_dev(oracle.pack_ternary2(t)), tba.BL_W_T2, alpha, M,
                      2 * F, K, group=F, ldy=2 * F + 64)
    acc_ref, _ = oracle.gemm(a, scale, t, alpha, alpha_group=F, want_y=False)
    assert np.array_equal(acc, acc_ref)
    _, ex = exact_y(a, scale, t, alpha, F, np.arange(M))
    assert bf16_rows_rel_err(y, ex) <= BF16_ROW_TOL


# FP4: E2M1 activations x E2M1-coded ternary weights on the tensor cores
# (kind::mxf4, unit block scales, exact fp32 sums; acc holds twice the sum)
@pytest.mark.parametrize("name,make", PACK_CASES[:4], ids=[c[0] for c in PACK_CASES[:4]])
def test_pack_ternary_e2m1_parity(name, make):
    w = make()
    out, alpha = run_pack(w, tba.BL_W_E2M1)
    t_ref, a_ref = oracle.ternary_quantize(w, EPS)
    assert np.float32(alpha).view(np.uint32) == np.float32(a_ref).view(np.uint32)
    assert np.array_equal(out, oracle.pack_ternary_e2m1(t_ref))


GEMM_FP4_CASES = [
    ("one_row", 1, 224, 128),
    ("K_tail_130x300x320", 130, 300, 320),
    ("two_pair_tiles_300x448x1024", 300, 448, 1024),
    ("ragged_257x520x3200", 257, 520, 3200),
    ("many_tiles_1300x2304x1024", 1300, 2304, 1024),
    ("K11008_512x256", 512, 256, 11008),
]


@pytest.mark.parametrize("name,M,N,K", GEMM_FP4_CASES, ids=[c[0] for c in GEMM_FP4_CASES])
def test_gemm_fp4_mxf4_parity(name, M, N, K):
    g = synth.rng(M * 5 + N + K)
    x = synth.gaussian_bf16(g, (M, K), outlier_channels=(3,), outlier_scale=8.0)
    w = synth.latent_weights_f32(g, N, K)
    t_ref, a_ref = oracle.ternary_quantize(w, EPS)
    code4, twice, _, scale = oracle.quant_fp4(x)
    acc, y = run_gemm(to_dev(oracle.pack_nibbles(code4)), tba.BL_A_E2M1, scale,
                      to_dev(oracle.pack_ternary_e2m1(t_ref)), tba.BL_W_E2M1, a_ref, M, N, K)
    acc_scale = (scale.astype(np.float64) / 2).astype(np.float32)
    acc_ref, _ = oracle.gemm(twice, acc_scale, t_ref, a_ref, want_y=False)
    assert np.array_equal(acc, acc_ref)
    _, ex = exact_y(twice, acc_scale, t_ref, a_ref, N, np.arange(M))
    assert bf16_rows_rel_err(y, ex) <= BF16_ROW_TOL


def test_gemm_fp4_end_to_end_alpha_groups():
    # FP4 quantizer -> packed codes -> stacked Up|Gate E2M1 weights, one alpha each
    M, F, K = 200, 448, 1536
    g = synth.rng(35)
    x = synth.gaussian_bf16(g, (M, K))
    wu, wg = synth.latent_weights_f32(g, F, K), synth.latent_weights_f32(g, F, K)
    tu, au = oracle.ternary_quantize(wu, EPS)
    tg, ag = oracle.ternary_quantize(wg, EPS)
    codes = empty((M, K // 2), torch.uint8)
    scale = empty((M,), torch.float32)
    tba.bitlinear_quant_a4(to_dev(x), codes, scale, quant=tba.BL_QUANT_FP4_E2M1, store=tba.BL_STORE_PACKED, eps=EPS)
    wdev = empty((2 * F, K // 2), torch.uint8)
    alpha = empty((2,), torch.float32)
    ws = empty((tba.workspace_size("pack_ternary") // 8,), torch.int64)
    tba.pack_ternary(to_dev(wu), alpha[0:1], wdev[:F], tba.BL_W_E2M1, ws, eps=EPS)
    tba.pack_ternary(to_dev(wg), alpha[1:2], wdev[F:], tba.BL_W_E2M1, ws, eps=EPS)
    y = empty((M, 2 * F), torch.int16)
    acc = empty((M, 2 * F), torch.int32)
    tba.bitlinear_gemm(codes, scale, wdev, alpha, M, 2 * F, K, y=y, acc=acc, afmt=tba.BL_A_E2M1,
                       wfmt=tba.BL_W_E2M1, alpha_group=F)
    tba.sync_status()
    code4, twice, _, s_ref = oracle.quant_fp4(x)
    assert np.array_equal(host(codes), oracle.pack_nibbles(code4))
    t = np.concatenate([tu, tg])
    al = np.array([au, ag], np.float32)
    acc_scale = (s_ref.astype(np.float64) / 2).astype(np.float32)
    acc_ref, _ = oracle.gemm(twice, acc_scale, t, al, alpha_group=F, want_y=False)
    assert np.array_equal(host(acc), acc_ref)
    _, ex = exact_y(twice, acc_scale, t, al, F, np.arange(M))
    assert bf16_rows_rel_err(host(y, np.uint16), ex) <= BF16_ROW_TOL


# up to 16 tokens against 2-bit weights: the decode GEMVs (dp4a for 1-2 tokens,
# warp-level MMA with 8 or 16 token slots for 3-16).  Rows are split over warps
# (K = 11008: 3 rounds / 11 batches; K = 36864: 9 rounds), so the shapes cover
# one and many rounds, a ragged last round, and N that fills no CTA; token slots
# x K = 36864 beyond the staged-activation limit take the tiled CUDA-core
# kernel or, for INT8 activations and more than 8 tokens, the tensor cores.
# For 1-2 tokens, rows up to K = 11328 and at most 32 rows per SM the
# streaming GEMV runs (every shape here with N <= 4736).
GEMV_SHAPES = [(1, 64), (7, 320), (130, 4096), (258, 4160), (37, 11008), (96, 640), (40, 36864), (4736, 640),
               (23680, 640)]


def gemv_inputs(g, afmt, M, K):
    """(device codes, afmt, the integer codes the sums use, scale passed, scale of those sums)"""
    if afmt == "i8":
        a = g.integers(-128, 128, (M, K)).astype(np.int8)
        scale = (g.random(M) * 0.1 + 1e-3).astype(np.float32)
        return to_dev(a), tba.BL_A_I8, a, scale, scale
    x = synth.gaussian_bf16(g, (M, K))
    if afmt == "i4":
        c, _, scale = oracle.quant_int4(x, EPS)
        return to_dev(oracle.pack_nibbles(c)), tba.BL_A_I4, c, scale, scale
    code4, twice, _, scale = oracle.quant_fp4(x)
    return (to_dev(oracle.pack_nibbles(code4)), tba.BL_A_E2M1, twice, scale,
            (scale.astype(np.float64) / 2).astype(np.float32))


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 9, 16])
@pytest.mark.parametrize("afmt", ["i8", "i4", "e2m1"])
@pytest.mark.parametrize("N,K", GEMV_SHAPES)
def test_gemv_t2_parity(M, afmt, N, K):
    g = synth.rng(M * 1000 + N + K + len(afmt))
    a_dev, af, codes, scale, sum_scale = gemv_inputs(g, afmt, M, K)
    t = g.integers(-1, 2, (N, K)).astype(np.int8)
    alpha = np.float32(0.0211)
    acc, y = run_gemm(a_dev, af, scale, to_dev(oracle.pack_ternary2(t)), tba.BL_W_T2, alpha, M, N, K)
    acc_ref, _ = oracle.gemm(codes, sum_scale, t, alpha, want_y=False)
    assert np.array_equal(acc, acc_ref)
    _, ex = exact_y(codes, sum_scale, t, alpha, N, np.arange(M))
    assert bf16_rows_rel_err(y, ex) <= BF16_ROW_TOL


# the largest sums the GEMV meets: every activation -128 against rows of all
# +1, all -1, all 0 and random signs, at the longest K it takes
@pytest.mark.parametrize("M,K", [(1, 65536), (2, 65536), (4, 32768), (8, 16384), (1, 16384), (3, 18432), (16, 11264)])
def test_gemv_t2_extreme_sums(M, K):
    N = 12
    g = synth.rng(M + K)
    a = np.full((M, K), -128, np.int8)
    t = np.zeros((N, K), np.int8)
    t[0], t[1] = 1, -1
    t[3:] = g.integers(-1, 2, (N - 3, K))
    scale = np.full(M, 1e-6, np.float32)
    alpha = np.float32(0.5)
    acc, y = run_gemm(to_dev(a), tba.BL_A_I8, scale, to_dev(oracle.pack_ternary2(t)), tba.BL_W_T2, alpha, M, N, K)
    acc_ref, _ = oracle.gemm(a, scale, t, alpha, want_y=False)
    assert np.array_equal(acc, acc_ref)
    assert acc[0, 0] == -128 * K and acc[0, 1] == 128 * K and acc[0, 2] == 0
    _, ex = exact_y(a, scale, t, alpha, N, np.arange(M))
    assert bf16_rows_rel_err(y, ex) <= BF16_ROW_TOL


@pytest.mark.parametrize("M", [1, 3, 8])
def test_gemv_t2_alpha_groups_and_ldy(M):
    F, K = 100, 4096
    g = synth.rng(40 + M)
    a_dev, af, codes, scale, sum_scale = gemv_inputs(g, "i4", M, K)
    t = g.integers(-1, 2, (2 * F, K)).astype(np.int8)
    alpha = np.array([0.0151, 0.0213], np.float32)
    acc, y = run_gemm(a_dev, af, scale, to_dev(oracle.pack_ternary2(t)), tba.BL_W_T2, alpha, M, 2 * F, K,
                      group=F, ldy=2 * F + 64)
    acc_ref, _ = oracle.gemm(codes, sum_scale, t, alpha, alpha_group=F, want_y=False)
    assert np.array_equal(acc, acc_ref)
    _, ex = exact_y(codes, sum_scale, t, alpha, F, np.arange(M))
    assert bf16_rows_rel_err(y, ex) <= BF16_ROW_TOL


# past the GEMV's K limit the tiled CUDA-core kernel stages fewer rows of A
# per tile; past its own limit the call is refused before any launch
def test_gemm_t2_long_k_cuda_core():
    M, N, K = 3, 16, 131072
    g = synth.rng(77)
    a_dev, af, codes, scale, sum_scale = gemv_inputs(g, "i4", M, K)
    t = g.integers(-1, 2, (N, K)).astype(np.int8)
    acc, y = run_gemm(a_dev, af, scale, to_dev(oracle.pack_ternary2(t)), tba.BL_W_T2, np.float32(0.02), M, N, K)
    acc_ref, _ = oracle.gemm(codes, sum_scale, t, np.float32(0.02), want_y=False)
    assert np.array_equal(acc, acc_ref)
    K = 196608 + 64
    with pytest.raises(tba.BitLinearError) as e:
        run_gemm(to_dev(np.zeros((1, K), np.int8)), tba.BL_A_I8, np.ones(1, np.float32),
                 to_dev(np.zeros((2, K // 4), np.uint8)), tba.BL_W_T2, np.float32(1.0), 1, 2, K)
    assert tba.STATUS_NAMES[e.value.status] == "BL_ERR_SHAPE"


# bitlinear_quant_gemm: the INT4 / FP4 quantizer fused into the GEMM.  For 1-2
# tokens against 2-bit weights it runs in the decode GEMV's prologue (every CTA
# quantizes the token rows itself); otherwise as quantizer + GEMM through the
# workspace.  Either way the result must be the oracle's quantizer followed by
# its matmul, and y must be bit-identical to the two separate calls.
QG_CASES = [(1, 96, 640), (2, 130, 4096), (3, 37, 11008), (5, 258, 4160), (8, 40, 16384), (16, 136, 1024),
            (40, 200, 4096)]


@pytest.mark.parametrize("quant", ["int4", "fp4"])
@pytest.mark.parametrize("wfmt", [tba.BL_W_T2, tba.BL_W_I8], ids=["t2", "i8w"])
@pytest.mark.parametrize("M,N,K", QG_CASES)
def test_quant_gemm_parity(quant, wfmt, M, N, K):
    g = synth.rng(M * 31 + N + K + len(quant))
    x = synth.gaussian_bf16(g, (M, K))
    x[:, 5] = synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(x[:, 5]) * 20)   # an outlier channel
    if M >= 2:
        x[1] = 0                                                               # an all-zero token
    w = synth.latent_weights_f32(g, N, K)
    t, a_ref = oracle.ternary_quantize(w, EPS)
    wq = oracle.pack_ternary2(t) if wfmt == tba.BL_W_T2 else t.view(np.uint8)
    q = tba.BL_QUANT_INT4 if quant == "int4" else tba.BL_QUANT_FP4_E2M1
    if quant == "int4":
        codes, _, scale = oracle.quant_int4(x, EPS)
        sum_scale = scale
    else:
        _, codes, _, scale = oracle.quant_fp4(x)
        sum_scale = (scale.astype(np.float64) / 2).astype(np.float32)
    ldx = K + 64
    xp = np.zeros((M, ldx), np.uint16)
    xp[:, :K] = x
    xd, wd = to_dev(xp), to_dev(wq)
    al = to_dev(np.array([a_ref], np.float32))
    ldy = (N + 7) // 8 * 8
    y, acc = empty((M, ldy), torch.int16), empty((M, N), torch.int32)
    ws = empty((tba.workspace_size("quant_gemm", M, N, K) // 8 + 1,), torch.int64)
    tba.bitlinear_quant_gemm(xd, wd, al, M, N, K, y=y, acc=acc, quant=q, wfmt=wfmt, eps=EPS, ldx=ldx, workspace=ws)
    tba.sync_status()
    acc_ref, _ = oracle.gemm(codes, sum_scale, t, a_ref, want_y=False)
    assert np.array_equal(host(acc), acc_ref)
    _, ex = exact_y(codes, sum_scale, t, a_ref, N, np.arange(M))
    y_fused = host(y, np.uint16)[:, :N]
    assert bf16_rows_rel_err(y_fused, ex) <= BF16_ROW_TOL
    # the same two steps as separate calls
    c8, s8 = empty((M, K), torch.int8), empty((M,), torch.float32)
    tba.bitlinear_quant_a4(xd, c8, s8, q, tba.BL_STORE_BYTES, EPS, M=M, K=K, ldx=ldx)
    y2 = empty((M, ldy), torch.int16)
    tba.bitlinear_gemm(c8, s8, wd, al, M, N, K, y=y2, wfmt=wfmt)
    tba.sync_status()
    assert np.array_equal(host(y2, np.uint16)[:, :N], y_fused)


def test_quant_gemm_needs_workspace_beyond_the_gemv():
    M, N, K = 16, 64, 256
    x = to_dev(np.zeros((M, K), np.uint16))
    w = to_dev(np.zeros((N, K // 4), np.uint8))
    al = to_dev(np.ones(1, np.float32))
    y = empty((M, N), torch.int16)
    with pytest.raises(tba.BitLinearError) as e:
        tba.bitlinear_quant_gemm(x, w, al, M, N, K, y=y)
    assert tba.STATUS_NAMES[e.value.status] == "BL_ERR_NULL"
    # from 3 tokens the quantizer runs separately, through the workspace
    with pytest.raises(tba.BitLinearError) as e:
        tba.bitlinear_quant_gemm(x[:3], w, al, 3, N, K, y=y[:3])
    assert tba.STATUS_NAMES[e.value.status] == "BL_ERR_NULL"
    # the decode GEMV with the quantizer in its prologue (1-2 tokens) needs none
    tba.bitlinear_quant_gemm(x[:2], w, al, 2, N, K, y=y[:2])
    tba.sync_status()
    assert np.array_equal(host(y[:2], np.uint16), np.zeros((2, N), np.uint16))


# the conditional Up projection: Gate rows first, Up rows only where some
# token's gate output is > 0; ReLU^2-GLU must then give exactly what it gives
# after the dense Up|Gate GEMM
@pytest.mark.parametrize("M", [1, 2])
@pytest.mark.parametrize("F,K,zero_frac", [(96, 640, 0.0), (1000, 4096, 0.0), (1000, 4096, 0.675), (37, 64, 0.0),
                                           (2048, 1536, 1.0)])
def test_gemm_gated_conditional_up(M, F, K, zero_frac):
    g = synth.rng(M * 7 + F + K)
    x = synth.gaussian_bf16(g, (M, K))
    c, _, s_ref = oracle.quant_int4(x, EPS)
    wu, wg = synth.latent_weights_f32(g, F, K), synth.latent_weights_f32(g, F, K)
    tu, au = oracle.ternary_quantize(wu, EPS)
    tg, ag = oracle.ternary_quantize(wg, EPS)
    # all-zero Gate rows give exactly-zero gate outputs: inactive channels at a
    # chosen share (0.675: the pages' Gate sparsity; 1.0: no Up row is read)
    tg[g.random(F) < zero_frac] = 0
    t = np.concatenate([tu, tg])
    al = np.array([au, ag], np.float32)
    a_dev, s_dev, w_dev, al_dev = to_dev(c), to_dev(s_ref), to_dev(oracle.pack_ternary2(t)), to_dev(al)
    ldy = (2 * F + 15) // 8 * 8
    # dense reference path: the stacked Up|Gate GEMM
    y_dense = empty((M, ldy), torch.int16)
    acc_dense = empty((M, 2 * F), torch.int32)
    tba.bitlinear_gemm(a_dev, s_dev, w_dev, al_dev, M, 2 * F, K, y=y_dense, acc=acc_dense, wfmt=tba.BL_W_T2,
                       alpha_group=F, ldy=ldy)
    y_g = empty((M, ldy), torch.int16)
    acc_g = empty((M, 2 * F), torch.int32)
    tba.bitlinear_gemm_gated(a_dev, s_dev, w_dev, al_dev, M, F, K, y_g, acc=acc_g, ldy=ldy)
    tba.sync_status()
    yd, yg = host(y_dense, np.uint16)[:, :2 * F], host(y_g, np.uint16)[:, :2 * F]
    ad, ag_ = host(acc_dense), host(acc_g)
    acc_ref, _ = oracle.gemm(c, s_ref, t, al, alpha_group=F, want_y=False)
    # the Gate half: exactly the dense GEMM's, and the oracle's sums
    assert np.array_equal(yg[:, F:], yd[:, F:])
    assert np.array_equal(ag_[:, F:], acc_ref[:, F:])
    # the Up half: the oracle's sums on active channels, zeros elsewhere
    gate_bits = yg[:, F:]
    active = ((gate_bits & 0x8000) == 0) & (gate_bits != 0)
    active = active.any(axis=0)
    assert np.array_equal(ag_[:, :F], np.where(active[None, :], acc_ref[:, :F], 0))
    assert np.array_equal(yg[:, :F], np.where(active[None, :], yd[:, :F], 0))
    if zero_frac == 0.0:
        assert 0 < active.sum() < F
    if zero_frac == 1.0:
        assert not active.any() and not ag_[:, :F].any()
    # ReLU^2-GLU + Top-K 50% + INT8 gives identical codes, scale and mask (rows of
    # a multiple of 8 values; F = 37 checks the ragged last channel group only)
    if F % 8:
        return
    keep = synth.k_keep(F, 50)
    outs = []
    for y in (y_dense, y_g):
        h8 = empty((M, F), torch.int8)
        h8_s = empty((M,), torch.float32)
        mask = empty((M, (F + 31) // 32), torch.int32)
        tba.relu2_glu(y[:, F:2 * F], y[:, :F], keep, h8, h8_s, mask, EPS, M=M, F=F, ld=ldy)
        tba.sync_status()
        outs.append((host(h8), host(h8_s).view(np.uint32), host(mask)))
    for u, v in zip(*outs):
        assert np.array_equal(u, v)


def test_sync_status_clean():
    tba.sync_status()
