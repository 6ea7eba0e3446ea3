"""GPU parity of the activation quantizers and the KV quantizer against the CPU
oracle, through the C ABI.  Codes, masks and scales are compared bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_bit_activation_b200 as tba
from gpu_util import empty, host, to_dev

pytestmark = pytest.mark.gpu

EPS = 1e-5


def run_quant_a4(x, quant, store):
    M, K = x.shape
    xd = to_dev(x)
    nbytes = K // 2 if store == tba.BL_STORE_PACKED else K
    codes = empty((M, nbytes), torch.uint8)
    scale = empty((M,), torch.float32)
    tba.bitlinear_quant_a4(xd, codes, scale, quant=quant, store=store, eps=EPS)
    tba.sync_status()
    return host(codes), host(scale)


QUANT_CASES = [
    ("tiny", lambda: synth.tiny_inputs(0)[0]),
    ("ragged_M37_K1536", lambda: synth.gaussian_bf16(synth.rng(1), (37, 1536))),
    ("K3200_tail_chunk", lambda: synth.gaussian_bf16(synth.rng(2), (9, 3200))),
    ("K8_min", lambda: synth.gaussian_bf16(synth.rng(3), (5, 8))),
    ("K16384_max", lambda: synth.gaussian_bf16(synth.rng(4), (3, 16384))),
    ("zeros_and_consts", lambda: np.concatenate([np.zeros((2, 256), np.uint16),
                                                 synth.f32_to_bf16_bits(np.full((2, 256), -0.75, np.float32)),
                                                 synth.student_t_bf16(synth.rng(5), (4, 256))])),
]


@pytest.mark.parametrize("name,make", QUANT_CASES, ids=[c[0] for c in QUANT_CASES])
@pytest.mark.parametrize("store", [tba.BL_STORE_PACKED, tba.BL_STORE_BYTES], ids=["packed", "bytes"])
def test_quant_int4_parity(name, make, store):
    x = make()
    codes, scale = run_quant_a4(x, tba.BL_QUANT_INT4, store)
    c_ref, beta_ref, s_ref = oracle.quant_int4(x, EPS)
    if store == tba.BL_STORE_PACKED:
        assert np.array_equal(codes, oracle.pack_nibbles(c_ref))
    else:
        assert np.array_equal(codes.view(np.int8), c_ref)
    assert np.array_equal(scale.view(np.uint32), s_ref.view(np.uint32))


@pytest.mark.parametrize("name,make", QUANT_CASES, ids=[c[0] for c in QUANT_CASES])
@pytest.mark.parametrize("store", [tba.BL_STORE_PACKED, tba.BL_STORE_BYTES], ids=["packed", "bytes"])
def test_quant_fp4_parity(name, make, store):
    x = make()
    codes, scale = run_quant_a4(x, tba.BL_QUANT_FP4_E2M1, store)
    code4, twice, p, s_ref = oracle.quant_fp4(x)
    if store == tba.BL_STORE_PACKED:
        assert np.array_equal(codes, oracle.pack_nibbles(code4))
        assert np.array_equal(scale.view(np.uint32), s_ref.view(np.uint32))
    else:
        assert np.array_equal(codes.view(np.int8), twice)
        half = (s_ref.astype(np.float64) / 2).astype(np.float32)
        assert np.array_equal(scale.view(np.uint32), half.view(np.uint32))


# the ablation variants (Fig. 5 / Fig. 6) as flags of the same quantizer
@pytest.mark.parametrize("name,make", QUANT_CASES, ids=[c[0] for c in QUANT_CASES])
@pytest.mark.parametrize("store", [tba.BL_STORE_PACKED, tba.BL_STORE_BYTES], ids=["packed", "bytes"])
@pytest.mark.parametrize("variant", ["int4_absmax", "int4_absmean2"])
def test_quant_int4_variant_parity(name, make, store, variant):
    x = make()
    quant = tba.BL_QUANT_INT4_ABSMAX if variant == "int4_absmax" else tba.BL_QUANT_INT4_ABSMEAN2
    codes, scale = run_quant_a4(x, quant, store)
    ref = oracle.quant_int4_absmax if variant == "int4_absmax" else oracle.quant_int4_absmean2
    c_ref, _, s_ref = ref(x, EPS)
    if store == tba.BL_STORE_PACKED:
        assert np.array_equal(codes, oracle.pack_nibbles(c_ref))
    else:
        assert np.array_equal(codes.view(np.int8), c_ref)
    assert np.array_equal(scale.view(np.uint32), s_ref.view(np.uint32))


@pytest.mark.parametrize("name,make", QUANT_CASES, ids=[c[0] for c in QUANT_CASES])
@pytest.mark.parametrize("store", [tba.BL_STORE_PACKED, tba.BL_STORE_BYTES], ids=["packed", "bytes"])
def test_quant_fp4_e1m2_parity(name, make, store):
    x = make()
    codes, scale = run_quant_a4(x, tba.BL_QUANT_FP4_E1M2, store)
    code4, four, p, s_ref = oracle.quant_fp4_e1m2(x)
    if store == tba.BL_STORE_PACKED:
        assert np.array_equal(codes, oracle.pack_nibbles(code4))
        assert np.array_equal(scale.view(np.uint32), s_ref.view(np.uint32))
    else:
        assert np.array_equal(codes.view(np.int8), four)
        quarter = (s_ref.astype(np.float64) / 4).astype(np.float32)
        assert np.array_equal(scale.view(np.uint32), quarter.view(np.uint32))


def test_quant_fp4_e1m2_extreme_exponents_and_gemm():
    vals = [1e-39, 3e-38, 1e-20, 0.011, 1.75, 1.765625, 1e4, 3e38]
    rows = []
    for v in vals:
        r = synth.gaussian_bf16(synth.rng(8), (1, 64))
        f = np.clip(synth.bf16_bits_to_f32(r), -4, 4) * np.float32(v / 8)
        rows.append(synth.f32_to_bf16_bits(f))
    x = np.concatenate(rows)
    codes, scale = run_quant_a4(x, tba.BL_QUANT_FP4_E1M2, tba.BL_STORE_BYTES)
    code4, four, p, s_ref = oracle.quant_fp4_e1m2(x)
    assert np.array_equal(codes.view(np.int8), four)
    # the bytes feed the INT8 GEMM: acc = sum of 4 * value * t
    g = synth.rng(9)
    M, K = x.shape
    N = 48
    t = g.integers(-1, 2, (N, K)).astype(np.int8)
    y = empty((M, N), torch.int16)
    acc = empty((M, N), torch.int32)
    tba.bitlinear_gemm(to_dev(codes.view(np.int8)), to_dev(scale), to_dev(oracle.pack_ternary2(t)),
                       to_dev(np.array([0.02], np.float32)), M, N, K, y=y, acc=acc, wfmt=tba.BL_W_T2)
    tba.sync_status()
    acc_ref, _ = oracle.gemm(four, scale, t, np.float32(0.02), want_y=False)
    assert np.array_equal(host(acc), acc_ref)


def test_quant_fp4_extreme_exponents():
    # rows whose max spans bf16's whole exponent range, subnormals included
    vals = [1e-39, 3e-38, 1e-20, 0.011, 6.0, 6.03125, 1e4, 3e38]
    rows = []
    for v in vals:
        r = synth.gaussian_bf16(synth.rng(7), (1, 64))
        f = np.clip(synth.bf16_bits_to_f32(r), -4, 4) * np.float32(v / 8)
        rows.append(synth.f32_to_bf16_bits(f))
    x = np.concatenate(rows)
    for store in (tba.BL_STORE_PACKED, tba.BL_STORE_BYTES):
        codes, scale = run_quant_a4(x, tba.BL_QUANT_FP4_E2M1, store)
        code4, twice, p, s_ref = oracle.quant_fp4(x)
        if store == tba.BL_STORE_PACKED:
            assert np.array_equal(codes, oracle.pack_nibbles(code4))
            assert np.array_equal(scale.view(np.uint32), s_ref.view(np.uint32))
        else:
            assert np.array_equal(codes.view(np.int8), twice)


def run_sparsify(x, keep):
    M, K = x.shape
    xd = to_dev(x)
    codes = empty((M, K), torch.int8)
    scale = empty((M,), torch.float32)
    mask = empty((M, (K + 31) // 32), torch.int32)
    tba.bitlinear_sparsify_a8(xd, keep, codes, scale, mask, eps=EPS)
    tba.sync_status()
    return host(codes), host(scale), host(mask, np.uint32)


def check_topk(codes, scale, mask, ref):
    c_ref, m_ref, g_ref, s_ref = ref
    assert np.array_equal(mask, oracle.pack_mask_bits(m_ref))
    assert np.array_equal(codes, c_ref)
    assert np.array_equal(scale.view(np.uint32), s_ref.view(np.uint32))


TOPK_CASES = [
    ("tiny_50pct", lambda: synth.tiny_inputs(0)[0], 128),
    ("700M_O_input", lambda: synth.student_t_bf16(synth.rng(11), (64, 1536)), 768),
    ("K3200_tail", lambda: synth.student_t_bf16(synth.rng(12), (7, 3200)), 1600),
    ("K8640_down", lambda: synth.student_t_bf16(synth.rng(13), (5, 8640)), 4320),
    ("K11008_down", lambda: synth.student_t_bf16(synth.rng(14), (5, 11008)), 5504),
    ("keep1", lambda: synth.student_t_bf16(synth.rng(15), (6, 512)), 1),
    ("keep_all", lambda: synth.student_t_bf16(synth.rng(16), (6, 512)), 512),
    ("K40_ragged_mask_word", lambda: synth.student_t_bf16(synth.rng(17), (9, 40)), 13),
    ("K4096_7B_O", lambda: synth.student_t_bf16(synth.rng(19), (12, 4096)), 2048),
    ("K4104_two_warps", lambda: synth.student_t_bf16(synth.rng(20), (5, 4104)), 2052),
    ("K16384_four_warps", lambda: synth.student_t_bf16(synth.rng(21), (3, 16384)), 8192),
    ("gaussian_keep_small", lambda: synth.gaussian_bf16(synth.rng(22), (9, 1024)), 37),
]


@pytest.mark.parametrize("name,make,keep", TOPK_CASES, ids=[c[0] for c in TOPK_CASES])
def test_sparsify_a8_parity(name, make, keep):
    x = make()
    codes, scale, mask = run_sparsify(x, keep)
    check_topk(codes, scale, mask, oracle.sparsify_a8(x, keep, EPS))


def test_sparsify_a8_heavy_ties():
    g = synth.rng(18)
    x = synth.student_t_bf16(g, (8, 2048))
    x[0, :] = synth.f32_to_bf16_bits(np.full(2048, 0.5, np.float32))            # one value
    x[1, ::2] = 0                                                                  # half zeros
    x[2, :] = synth.f32_to_bf16_bits(np.round(synth.bf16_bits_to_f32(x[2]) * 2) / 2)   # coarse grid
    x[3, :1500] = 0x8000                                                           # -0 and +0 tie
    for keep in (1, 700, 1024, 1500, 2047):
        codes, scale, mask = run_sparsify(x, keep)
        check_topk(codes, scale, mask, oracle.sparsify_a8(x, keep, EPS))


def test_sparsify_a8_zero_and_constant_rows():
    x = synth.student_t_bf16(synth.rng(23), (4, 4096))
    x[0] = 0                                                  # gamma = 0: every code 0
    x[1] = synth.f32_to_bf16_bits(np.full(4096, -3.0, np.float32))
    x[2, 100:] = 0
    for keep in (1, 50, 100, 2048, 4095, 4096):
        codes, scale, mask = run_sparsify(x, keep)
        check_topk(codes, scale, mask, oracle.sparsify_a8(x, keep, EPS))


@pytest.mark.parametrize("K", [4096, 1000, 40])
def test_sparsify_a8_subnormal_and_extreme_rows(K):
    """Rows whose threshold falls among bf16 subnormals, on the subnormal /
    normal boundary, or among values spread over the whole exponent range: the
    magnitude ranking must order subnormals exactly (no flush to zero)."""
    g = synth.rng(K + 5)
    x = synth.student_t_bf16(g, (6, K))
    sign = (g.integers(0, 2, (6, K)) << 15).astype(np.uint16)
    x[0] = sign[0] | g.integers(1, 0x80, K).astype(np.uint16)                       # all subnormal
    x[1] = sign[1] | np.where(g.random(K) < 0.5, g.integers(1, 0x80, K),
                              g.integers(0x80, 0x100, K)).astype(np.uint16)       # subnormal and smallest normals
    x[2] = sign[2] | g.integers(1, 0x7F7F, K).astype(np.uint16)                      # whole exponent range
    x[3] = sign[3] | np.full(K, 0x0005, np.uint16)                                   # one subnormal value
    x[3, ::7] = 0x0003
    x[4, : K // 2] = 0x0001                                                          # smallest subnormal ties
    for keep in sorted({1, K // 3, K // 2, K - 1}):
        ref = oracle.sparsify_a8(x, keep, EPS)
        codes, scale, mask = run_sparsify(x, keep)
        check_topk(codes, scale, mask, ref)


def test_sparsify_a8_without_mask():
    """Without a mask the codes and scales are the same (dropped zeros among the
    ties need no ranking then)."""
    x = synth.student_t_bf16(synth.rng(24), (9, 4096))
    x[1, ::2] = 0
    x[2, :3000] = 0x8000
    for keep in (1, 1500, 2048, 3000, 4095):
        ref = oracle.sparsify_a8(x, keep, EPS)
        xd = to_dev(x)
        codes = empty(x.shape, torch.int8)
        scale = empty((x.shape[0],), torch.float32)
        tba.bitlinear_sparsify_a8(xd, keep, codes, scale, None, eps=EPS)
        tba.sync_status()
        assert np.array_equal(host(codes), ref[0])
        assert np.array_equal(host(scale).view(np.uint32), ref[3].view(np.uint32))


def run_relu2(gate, up, keep, ld_pad=0):
    M, F = gate.shape
    both = np.zeros((M, 2 * F + ld_pad), np.uint16)
    both[:, :F] = up
    both[:, F + ld_pad:2 * F + ld_pad] = gate
    d = to_dev(both)
    up_d = d[:, :F]
    gate_d = d[:, F + ld_pad:]
    codes = empty((M, F), torch.int8)
    scale = empty((M,), torch.float32)
    mask = empty((M, (F + 31) // 32), torch.int32)
    tba.relu2_glu(gate_d, up_d, keep, codes, scale, mask, eps=EPS, M=M, F=F, ld=d.stride(0))
    tba.sync_status()
    return host(codes), host(scale), host(mask, np.uint32)


RELU_CASES = [
    ("tiny", 16, 256, 128, 0.0),
    ("700M_F4096", 32, 4096, 2048, -0.454),
    ("3B_F8640", 6, 8640, 4320, -0.454),
    ("7B_F11008", 6, 11008, 5504, -0.454),
    ("keep_all", 8, 1024, 1024, 0.0),
    ("F40_ragged", 5, 40, 7, 0.0),
    ("F2048_one_warp_select", 7, 2048, 300, 0.0),
    ("F11008_select_nonzero", 5, 11008, 2000, 0.0),
    ("F11008_half", 6, 11008, 5504, 0.0),
    ("F12296_eight_warps", 3, 12296, 6148, 0.0),
    ("F16384_max", 3, 16384, 8192, -0.454),
]


@pytest.mark.parametrize("name,M,F,keep,shift", RELU_CASES, ids=[c[0] for c in RELU_CASES])
def test_relu2_glu_parity(name, M, F, keep, shift):
    gate, up = synth.glu_inputs(M, F, seed=F + M, gate_shift=shift)
    codes, scale, mask = run_relu2(gate, up, keep, ld_pad=8)
    check_topk(codes, scale, mask, oracle.relu2_glu(gate, up, keep, EPS))


def test_relu2_glu_ties_and_no_mask():
    M, F = 6, 4096
    gate, up = synth.glu_inputs(M, F, seed=99, gate_shift=0.0)
    one = synth.f32_to_bf16_bits(np.full(F, 1.0, np.float32))
    gate[0], up[0] = one, one                                  # every h equal: no list, all ties
    up[1] = synth.f32_to_bf16_bits(np.round(synth.bf16_bits_to_f32(up[1]) * 4) / 4)   # coarse: many ties
    gate[2] = 0                                                # all h zero
    gate[3, ::3] = one[::3]                                    # a third equal to up
    for keep in (1, 1000, 2048, 3000, 4095):
        ref = oracle.relu2_glu(gate, up, keep, EPS)
        codes, scale, mask = run_relu2(gate, up, keep)
        check_topk(codes, scale, mask, ref)
        # without a mask the codes and scales must not change
        both = np.zeros((M, 2 * F), np.uint16)
        both[:, :F] = up
        both[:, F:] = gate
        d = to_dev(both)
        c2 = empty((M, F), torch.int8)
        s2 = empty((M,), torch.float32)
        tba.relu2_glu(d[:, F:], d[:, :F], keep, c2, s2, None, eps=EPS, M=M, F=F, ld=2 * F)
        tba.sync_status()
        assert np.array_equal(host(c2), ref[0])
        assert np.array_equal(host(s2).view(np.uint32), ref[3].view(np.uint32))


def test_relu2_glu_subnormal_cut():
    # h = up * relu(gate)^2 subnormal in fp32 for part of each row, and the cut among
    # those values: the selection's first digit (the exponent) is then 0, the digit
    # the zero keys share, so the zeros stay candidates in the later digits
    g = synth.rng(123)
    M, F = 4, 2048
    gate = np.where(g.random((M, F)) < 0.5, -1.0, 1.0) * g.uniform(0.5, 1.5, (M, F))
    up = g.standard_normal((M, F))
    small = g.random((M, F)) < 0.6                    # these positions get a subnormal h
    gate = np.where(small, gate * 1e-15, gate)
    up = np.where(small, up * 1e-10, up)
    gate_b = synth.f32_to_bf16_bits(gate.astype(np.float32))
    up_b = synth.f32_to_bf16_bits(up.astype(np.float32))
    h = synth.bf16_bits_to_f32(up_b).astype(np.float32) * np.maximum(synth.bf16_bits_to_f32(gate_b), 0) ** 2
    nz = (h != 0).sum(axis=1)
    normal = (np.abs(h) >= np.float32(2.0 ** -126)).sum(axis=1)
    keep = int(normal.max() + (nz.min() - normal.max()) // 2)   # between the normal and the nonzero counts
    assert (normal < keep).all() and (nz > keep).all()
    ref = oracle.relu2_glu(gate_b, up_b, keep, EPS)
    codes, scale, mask = run_relu2(gate_b, up_b, keep)
    check_topk(codes, scale, mask, ref)


def run_kv(kv, bits, bos_pos, ldt_pad=0):
    T, H, D = kv.shape
    buf = np.zeros((T, H * D + ldt_pad), np.uint16)
    buf[:, :H * D] = kv.reshape(T, H * D)
    d = to_dev(buf)
    codes = empty((T, H, D * bits // 8), torch.uint8)
    scale = empty((T, H), torch.float32)
    bos = empty((H, D // 2), torch.uint8)
    tba.kv_quant3(d, T, H, D, codes, scale, bos_codes=bos, bits=bits, bos_pos=bos_pos, eps=EPS, ldt=d.stride(0))
    tba.sync_status()
    return host(codes), host(scale), host(bos)


@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("bits,bos_pos", [(3, 0), (3, 5), (3, -1), (4, -1)])
def test_kv_quant_parity(D, bits, bos_pos):
    k, _ = synth.kv_inputs(D, positions=37, heads=5, head_dim=D)
    codes, scale, bos = run_kv(k, bits, bos_pos, ldt_pad=8)
    cu, s_ref = oracle.kv_quant(k, bits=bits, bos_pos=bos_pos, eps=EPS)
    assert np.array_equal(scale.view(np.uint32), s_ref.view(np.uint32))
    for t in range(k.shape[0]):
        if bits == 3 and t == bos_pos:
            assert np.array_equal(bos, oracle.pack_nibbles(cu[t]))
            assert not codes[t].any()
        elif bits == 3:
            assert np.array_equal(codes[t], oracle.pack_kv3(cu[t]))
        else:
            assert np.array_equal(codes[t], oracle.pack_nibbles(cu[t]))
