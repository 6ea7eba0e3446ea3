"""Pins for the CPU oracle: hand-worked examples from the paper's equations,
closed forms, invariants and brute force on tiny inputs -- never the oracle's
own formula retyped.  CPU only."""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth
from conftest import read_golden

EPS = 1e-5


def bf16(vals):
    return synth.f32_to_bf16_bits(np.asarray(vals, np.float32))


def bf16_val(bits):
    return synth.bf16_bits_to_f32(bits)


# ----------------------------------------------------------------------------
# INT4 absmean (Eq. 6-7)
# ----------------------------------------------------------------------------
def test_int4_hand_examples():
    g = read_golden("int4_hand.txt")
    for xs, codes, beta in zip(g["x"], g["codes"], g["beta"]):
        c, b, s = oracle.quant_int4(bf16([xs]))
        assert c[0].tolist() == [int(v) for v in codes]
        assert abs(float(b[0]) - beta[0]) < 1e-6
        assert abs(float(s[0]) - beta[0] / math.sqrt(7)) < 1e-6


def test_int4_constant_row_closed_form():
    # x = c everywhere: beta = |c| exactly, sqrt7*c/(|c|+eps) ~ +-2.6457 -> +-3
    for c in (0.75, -3.0, 1e-3, 96.0):
        codes, beta, _ = oracle.quant_int4(bf16([[c] * 64]))
        assert float(beta[0]) == float(bf16_val(bf16([c]))[0].__abs__())
        assert set(codes[0].tolist()) == {3 if c > 0 else -3}


def test_int4_zero_row():
    codes, beta, scale = oracle.quant_int4(np.zeros((1, 32), np.uint16))
    assert not codes.any() and beta[0] == 0 and scale[0] == 0


def test_int4_brute_force_nearest_code():
    # Each code is the nearest of the 16 INT4 values to x*sqrt7/(beta+eps),
    # ties to the even one (brute force over the code set).
    x = synth.gaussian_bf16(synth.rng(11), (8, 96), outlier_channels=(3,), outlier_scale=9.0)
    codes, beta, _ = oracle.quant_int4(x)
    xf = bf16_val(x).astype(np.float32)
    for m in range(x.shape[0]):
        mult = np.float32(np.float32(math.sqrt(7)) / (np.float32(beta[m]) + np.float32(EPS)))
        for k in range(x.shape[1]):
            v = float(np.float32(xf[m, k] * mult))
            best = min(range(-8, 8), key=lambda c: (abs(v - c), c % 2))
            assert codes[m, k] == best
    assert codes.min() >= -8 and codes.max() <= 7


def test_int4_beta_is_correctly_rounded_mean():
    x = synth.gaussian_bf16(synth.rng(5), (4, 4096))
    _, beta, _ = oracle.quant_int4(x)
    for m in range(4):
        mean = math.fsum(abs(float(v)) for v in bf16_val(x[m])) / 4096
        assert abs(float(beta[m]) - mean) <= abs(mean) * 2 ** -24


def test_int4_rejects_inexact_sums():
    # a row whose |x| sum cannot be held exactly in fp64
    row = bf16([[1e30, 1e-30] + [0.0] * 30])
    with pytest.raises(ValueError):
        oracle.quant_int4(row)


# ----------------------------------------------------------------------------
# FP4 E2M1 (Eq. 8-9)
# ----------------------------------------------------------------------------
def test_fp4_hand_example():
    g = read_golden("fp4_hand.txt")
    code4, tv, p, scale = oracle.quant_fp4(bf16(g["x"]))
    assert p[0] == int(g["p"][0][0])
    assert (tv[0] / 2.0).tolist() == g["values"][0]
    assert code4[0].tolist() == [int(v) for v in g["codes"][0]]
    assert scale[0] == 1.0


@pytest.mark.parametrize("gmax,p", [(6.0, 0), (6.03125, 1), (3.0, -1), (3.015625, 0),
                                    (12.0, 1), (0.75, -3), (1.5, -2), (1e-3, -12)])
def test_fp4_scale_exponent_closed_form(gmax, p):
    # p = ceil(log2(max|x| / 6)): the smallest power of two that covers the max
    row = bf16([[gmax, -gmax / 4, 0.0, gmax / 3]])
    g = float(bf16_val(row)[0, 0])
    _, _, pp, scale = oracle.quant_fp4(row)
    assert pp[0] == p
    assert g <= 6 * 2.0 ** p and g > 6 * 2.0 ** (p - 1)
    assert scale[0] == np.float32(2.0 ** p)


def test_fp4_exhaustive_bf16_against_midpoint_table():
    # Every positive and negative finite bf16 below 6 at p = 0, against a rounding
    # written from the grid midpoints and the even-encoding tie rule.
    mids = [(0.25, 0, 0), (0.75, 1, 2), (1.25, 2, 2), (1.75, 3, 4), (2.5, 4, 4),
            (3.5, 5, 6), (5.0, 6, 6)]       # (midpoint, code below, code at tie)

    def table_code(v):
        a = abs(v)
        code = 7
        for mid, below, tie in mids:
            if a < mid:
                code = below
                break
            if a == mid:
                code = tie
                break
        return code

    bits = np.arange(0, 0x8000, dtype=np.uint16)
    vals = bf16_val(bits)
    keep = np.isfinite(vals) & (vals <= 6.0)
    bits = bits[keep]
    for sign in (0, 0x8000):
        b = (bits | sign).astype(np.uint16)
        row = np.concatenate([b, bf16([6.0])]).reshape(1, -1)   # pin max |x| = 6 -> p = 0
        code4, tv, p, _ = oracle.quant_fp4(row)
        assert p[0] == 0
        v = bf16_val(row[0])
        for j in range(row.shape[1]):
            mag_code = table_code(float(v[j]))
            expect = mag_code | (8 if (v[j] < 0 and mag_code != 0) else 0)
            assert code4[0, j] == expect, (float(v[j]), code4[0, j], expect)
        grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
        assert np.array_equal(np.abs(tv[0]) / 2.0, grid[code4[0] & 7])


# ----------------------------------------------------------------------------
# Top-K + INT8 (Eq. 1)
# ----------------------------------------------------------------------------
def test_topk_int8_hand_example():
    g = read_golden("topk_int8_hand.txt")
    codes, mask, gamma, scale = oracle.sparsify_a8(bf16(g["x"]), int(g["keep"][0][0]))
    assert mask[0].tolist() == [int(v) for v in g["mask"][0]]
    assert codes[0].tolist() == [int(v) for v in g["codes"][0]]
    assert gamma[0] == g["gamma"][0][0]
    assert abs(scale[0] - 3 / 127) < 1e-8
    assert oracle.pack_mask_bits(mask)[0, 0] == int(g["mask_word"][0][0])


def _check_topk_invariants(mag, mask, keep):
    """Exactly keep survivors; every survivor's magnitude >= every dropped one's;
    at the threshold magnitude, survivors precede the dropped by index."""
    kept = np.flatnonzero(mask)
    dropped = np.flatnonzero(mask == 0)
    assert kept.size == keep
    if dropped.size and kept.size:
        thr = mag[kept].min()
        assert thr >= mag[dropped].max()
        tk = kept[mag[kept] == thr]
        td = dropped[mag[dropped] == thr]
        if td.size:
            assert tk.max() < td.min()


def test_topk_invariants_heavy_tailed_and_ties():
    g = synth.rng(3)
    x = synth.student_t_bf16(g, (6, 512))
    x[1, ::3] = 0                      # many tied zeros
    x[2, :] = bf16([[0.5] * 512])[0]   # all tied
    for keep in (1, 128, 256, 511, 512):
        codes, mask, gamma, _ = oracle.sparsify_a8(x, keep)
        mag = np.abs(bf16_val(x).astype(np.float64))
        for m in range(6):
            _check_topk_invariants(mag[m], mask[m], keep)
            assert gamma[m] == mag[m].max()
            assert np.all(codes[m][mask[m] == 0] == 0)
            assert codes[m].min() >= -127 and codes[m].max() <= 127


def test_topk_brute_force_tiny():
    # all subsets of size keep: the chosen one is the unique lexicographic maximum
    # of (sorted magnitudes desc, then smaller indices)
    import itertools
    g = synth.rng(9)
    for trial in range(20):
        x = bf16(np.round(g.standard_normal(7) * 2) / 2)       # many ties
        mag = np.abs(bf16_val(x).astype(np.float64))
        keep = 1 + trial % 6
        _, mask, _, _ = oracle.sparsify_a8(x.reshape(1, -1), keep)
        best = max(itertools.combinations(range(7), keep),
                   key=lambda s: (sorted(mag[list(s)], reverse=True), [-i for i in s]))
        assert sorted(np.flatnonzero(mask[0]).tolist()) == list(best)


def test_int8_codes_bruteforce_nearest():
    x = synth.student_t_bf16(synth.rng(4), (3, 200))
    codes, mask, gamma, _ = oracle.sparsify_a8(x, 200)
    xf = bf16_val(x)
    for m in range(3):
        mult = np.float32(np.float32(127.0) / (np.float32(gamma[m]) + np.float32(EPS)))
        for k in range(200):
            v = float(np.float32(xf[m, k] * mult))
            assert abs(v - codes[m, k]) <= 0.5
            if abs(v - codes[m, k]) == 0.5:
                assert codes[m, k] % 2 == 0


# ----------------------------------------------------------------------------
# ReLU^2-GLU (Eq. 5)
# ----------------------------------------------------------------------------
def test_relu2_glu_hand_example():
    g = read_golden("relu2glu_hand.txt")
    gate, up = bf16(g["gate"]), bf16(g["up"])
    for keep, mask_e, codes_e in zip(g["keep"], g["mask"], g["codes"]):
        codes, mask, gamma, _, h = oracle.relu2_glu(gate, up, int(keep[0]), want_h=True)
        assert h[0].tolist() == g["h"][0]
        assert mask[0].tolist() == [int(v) for v in mask_e]
        assert codes[0].tolist() == [int(v) for v in codes_e]
        assert gamma[0] == 4.5


def test_relu2_glu_closed_form():
    g = synth.rng(21)
    gate = synth.gaussian_bf16(g, (4, 300))
    up = synth.gaussian_bf16(g, (4, 300))
    _, mask, _, _, h = oracle.relu2_glu(gate, up, 150, want_h=True)
    gf = bf16_val(gate).astype(np.float64)
    uf = bf16_val(up).astype(np.float64)
    exact = uf * np.maximum(gf, 0) ** 2
    assert np.all(h[gf <= 0] == 0)                       # gate <= 0 gives exactly 0
    assert np.all(np.abs(h - exact) <= np.abs(exact) * 2 ** -22)   # two fp32 roundings
    for m in range(4):
        _check_topk_invariants(np.abs(h[m].astype(np.float64)), mask[m], 150)


# ----------------------------------------------------------------------------
# Ternary weights (Eq. 2)
# ----------------------------------------------------------------------------
def test_ternary_hand_example():
    g = read_golden("ternary_hand.txt")
    w = np.array(g["w"], np.float32)
    t, alpha = oracle.ternary_quantize(w)
    assert abs(float(alpha) - g["alpha"][0][0]) < 1e-9
    assert t.tolist() == [[int(v) for v in r] for r in g["codes"]]
    assert oracle.pack_ternary2(t)[0, 0] == int(g["packed_row0"][0][0])


def test_ternary_alpha_exact_cases():
    # means that are exactly representable must come out exactly
    w = np.array([[1, -2], [3, -4]], np.float32) * np.float32(0.125)
    assert oracle.ternary_alpha(w) == np.float32(0.3125)
    w = np.full((7, 33), -0.0213, np.float32)
    assert oracle.ternary_alpha(w) == np.float32(0.0213)
    assert oracle.ternary_alpha(np.zeros((3, 8), np.float32)) == 0.0
    # subnormal entries are summed too
    tiny = np.float32(2.0 ** -140)
    assert oracle.ternary_alpha(np.full((2, 2), tiny, np.float32)) == tiny


def test_ternary_alpha_against_fsum():
    w = synth.latent_weights_f32(synth.rng(8), 64, 96)
    a = float(oracle.ternary_alpha(w))
    mean = math.fsum(abs(float(v)) for v in w.ravel()) / w.size
    assert abs(a - mean) <= mean * 2 ** -24


def test_round_fraction_to_f32_matches_numpy_single_rounding():
    g = synth.rng(1)
    vals = np.concatenate([g.standard_normal(2000) * 10.0 ** g.integers(-40, 38, 2000),
                           [2.0 ** -149, 2.0 ** -149 * 1.5, 2.0 ** -126 * 0.75, 1.0 + 2.0 ** -24]])
    for v in np.abs(vals):
        if v == 0 or v >= 3.4e38:
            continue
        assert oracle.round_fraction_to_f32(Fraction(float(v))) == np.float32(v)


def test_ternary_codes_bruteforce():
    w = synth.latent_weights_f32(synth.rng(6), 16, 64)
    t, alpha = oracle.ternary_quantize(w)
    d = np.float32(np.float32(alpha) + np.float32(EPS))
    for n in range(16):
        for k in range(64):
            q = float(np.float32(w[n, k] / d))
            best = min((-1, 0, 1), key=lambda c: (abs(q - c), c % 2))
            assert t[n, k] == best
    # about 31% of Gaussian weights land on 0 (|w| < alpha/2, alpha ~ 0.8 sigma)
    frac0 = np.mean(t == 0)
    assert 0.2 < frac0 < 0.45


# ----------------------------------------------------------------------------
# GEMM (Y = Q_x(X) Q_w(W)^T)
# ----------------------------------------------------------------------------
def test_gemm_hand_example():
    gi = read_golden("int4_hand.txt")
    gt = read_golden("ternary_hand.txt")
    gg = read_golden("gemm_hand.txt")
    c, _, s = oracle.quant_int4(bf16([gi["x"][0]]))
    t, alpha = oracle.ternary_quantize(np.array(gt["w"], np.float32))
    acc, y = oracle.gemm(c, s, t, alpha)
    assert acc[0].tolist() == [int(v) for v in gg["acc"][0]]
    yv = bf16_val(y[0])
    for a, b in zip(yv, gg["y"][0]):
        assert abs(a - b) <= abs(b) * 2 ** -8


def test_gemm_bruteforce_tiny_nonsquare():
    g = synth.rng(2)
    M, N, K = 5, 7, 33
    a = g.integers(-128, 128, (M, K)).astype(np.int8)
    t = g.integers(-1, 2, (N, K)).astype(np.int8)
    s = (g.random(M) + 0.1).astype(np.float32)
    alpha = np.float32(0.0173)
    acc, y = oracle.gemm(a, s, t, alpha)
    for m in range(M):
        for n in range(N):
            ref = sum(int(a[m, k]) * int(t[n, k]) for k in range(K))
            assert acc[m, n] == ref
            exact = Fraction(ref) * Fraction(float(s[m])) * Fraction(float(alpha))
            yv = Fraction(float(bf16_val(y[m:m + 1, n])[0]))
            assert abs(yv - exact) <= abs(exact) * Fraction(1, 256)   # half a bf16 ulp
    # row selection returns the same rows
    acc2, _ = oracle.gemm(a, s, t, alpha, rows=[4, 0])
    assert np.array_equal(acc2, acc[[4, 0]])


def test_gemm_alpha_groups():
    g = synth.rng(12)
    a = g.integers(-8, 8, (3, 16)).astype(np.int8)
    t = g.integers(-1, 2, (6, 16)).astype(np.int8)
    s = np.ones(3, np.float32)
    _, y = oracle.gemm(a, s, t, np.array([1.0, 2.0], np.float32), alpha_group=3)
    acc, y1 = oracle.gemm(a, s, t, np.float32(1.0))
    assert np.array_equal(bf16_val(y[:, :3]), bf16_val(y1[:, :3]))
    assert np.array_equal(bf16_val(y[:, 3:]), 2 * bf16_val(y1[:, 3:]))


def test_gemm_end_to_end_dequant_matches_fp64():
    # y ~ (dequantized X) . (dequantized W)^T in fp64, the product the method defines
    x, w = synth.tiny_inputs(0)
    c, _, s = oracle.quant_int4(x)
    t, alpha = oracle.ternary_quantize(w)
    _, y = oracle.gemm(c, s, t, alpha)
    ref = (c.astype(np.float64) * s[:, None]) @ (t.astype(np.float64) * float(alpha)).T
    err = np.abs(bf16_val(y).astype(np.float64) - ref).max(axis=1) / np.linalg.norm(ref, axis=1)
    assert err.max() < 1e-2


# ----------------------------------------------------------------------------
# KV cache
# ----------------------------------------------------------------------------
def test_kv_hand_example():
    g = read_golden("kv_hand.txt")
    kv = bf16(g["x"]).reshape(1, 1, 8)
    codes, scale = oracle.kv_quant(kv, bits=3, bos_pos=-1)
    assert codes[0, 0].tolist() == [int(v) for v in g["codes3"][0]]
    assert abs(scale[0, 0] - g["scale3"][0][0]) < 1e-6
    assert oracle.pack_kv3(codes)[0, 0].tolist() == [int(v) for v in g["packed3"][0]]
    codes4, scale4 = oracle.kv_quant(kv, bits=3, bos_pos=0)       # BOS row at 4 bits
    assert codes4[0, 0].tolist() == [int(v) for v in g["codes4"][0]]
    assert abs(scale4[0, 0] - g["scale4"][0][0]) < 1e-6


def test_kv_ranges_and_roundtrip_bound():
    k, _ = synth.kv_inputs(0, positions=9, heads=3, head_dim=128)
    codes, scale = oracle.kv_quant(k, bits=3, bos_pos=0)
    x = bf16_val(k).astype(np.float64)
    for t in range(9):
        b = 4 if t == 0 else 3
        q = 2 ** (b - 1) - 1
        c = codes[t].astype(np.int64)
        assert c.min() >= 1 and c.max() <= 2 ** b - 1        # symmetric: code 0 unused
        deq = (c - 2 ** (b - 1)) * scale[t][:, None].astype(np.float64)
        gamma = np.abs(x[t]).max(axis=1)
        assert np.all(np.abs(deq - x[t]) <= (gamma / (2 * q))[:, None] * (1 + 1e-4))


# ----------------------------------------------------------------------------
# Storage layouts
# ----------------------------------------------------------------------------
def test_pack_layouts():
    assert oracle.pack_nibbles(np.array([1, -2], np.int8)).tolist() == [0xE1]
    assert oracle.pack_ternary2(np.array([1, -1, 0, 1], np.int8)).tolist() == [0x4D]
    # ternary as E2M1 (FP4 weight layout): +1 -> 0x2, -1 -> 0xA, 0 -> 0x0, element 2i low nibble
    assert oracle.pack_ternary_e2m1(np.array([1, -1, 0, 1], np.int8)).tolist() == [0xA2, 0x20]
    # the same codes are what the FP4 quantizer writes for +1, -1 and 0 (scale 2^0 when max|x| = 6)
    code4, twice, _, _ = oracle.quant_fp4(synth.f32_to_bf16_bits(np.array([[1.0, -1.0, 0.0, 6.0]], np.float32)))
    assert code4[0].tolist() == [0x2, 0xA, 0x0, 0x7]
    assert twice[0].tolist() == [2, -2, 0, 12]
    m = np.zeros((1, 40), np.uint8)
    m[0, [0, 31, 32, 39]] = 1
    assert oracle.pack_mask_bits(m).tolist() == [[0x80000001, 0x81]]


# ----------------------------------------------------------------------------
# Quantizer variants of the ablations (Fig. 5 / Fig. 6), as flags
# ----------------------------------------------------------------------------
def test_int4_absmax_hand_examples():
    # gamma = max|x| = 4: mult = 7/(4+eps) = 1.7499956 -> 0.175, -0.350, 6.99998,
    # 0.526 -> [0, 0, 7, 1] (the bf16 values of 0.1, -0.2, 0.3 are 0.10009766,
    # -0.20019531, 0.30078125); scale = 4/7
    codes, gamma, scale = oracle.quant_int4_absmax(bf16([[0.1, -0.2, 4.0, 0.3]]))
    assert codes[0].tolist() == [0, 0, 7, 1]
    assert gamma[0] == 4.0
    assert scale[0] == np.float32(np.float32(4.0) / np.float32(7.0))
    # gamma = 7: mult ~ 1 - 1.4e-6 -> the integers themselves
    codes, gamma, scale = oracle.quant_int4_absmax(bf16([[1.0, -2.0, 3.0, -7.0]]))
    assert codes[0].tolist() == [1, -2, 3, -7]
    assert scale[0] == 1.0


def test_int4_absmax_max_element_maps_to_7():
    # the largest magnitude always lands on +-7 (7*g/(g+eps) rounds to 7 for g >> eps)
    x = synth.gaussian_bf16(synth.rng(21), (6, 256))
    codes, gamma, _ = oracle.quant_int4_absmax(x)
    xf = bf16_val(x)
    for m in range(6):
        k = int(np.argmax(np.abs(xf[m])))
        assert abs(int(codes[m, k])) == 7
        assert gamma[m] == np.float32(np.abs(xf[m]).max())
    assert codes.min() >= -7 and codes.max() <= 7


def test_int4_absmax_brute_force_nearest_code():
    x = synth.gaussian_bf16(synth.rng(22), (4, 96), outlier_channels=(7,), outlier_scale=9.0)
    codes, gamma, _ = oracle.quant_int4_absmax(x)
    xf = bf16_val(x).astype(np.float32)
    for m in range(x.shape[0]):
        mult = np.float32(np.float32(7.0) / (np.float32(gamma[m]) + np.float32(EPS)))
        for k in range(x.shape[1]):
            v = float(np.float32(xf[m, k] * mult))
            best = min(range(-8, 8), key=lambda c: (abs(v - c), c % 2))
            assert codes[m, k] == best


def test_int4_absmean2_hand_example_and_relation():
    # mean|x| = 2.5 -> beta = 5; mult = sqrt7/(5+eps) = 0.52915 -> 0.529, -1.058,
    # 1.587, -2.117 -> [1, -1, 2, -2]; scale = 5/sqrt7
    codes, beta, scale = oracle.quant_int4_absmean2(bf16([[1.0, -2.0, 3.0, -4.0]]))
    assert codes[0].tolist() == [1, -1, 2, -2]
    assert beta[0] == 5.0
    assert scale[0] == np.float32(np.float32(5.0) / np.float32(math.sqrt(7)))
    # beta is twice the absmean beta of the same row, which is twice the absmean
    # beta of the halved row (halving bf16 values is exact)
    x = synth.gaussian_bf16(synth.rng(23), (5, 512))
    c2, b2, _ = oracle.quant_int4_absmean2(x, 0.0)
    _, b1, _ = oracle.quant_int4(x, 0.0)
    _, bh, _ = oracle.quant_int4(synth.f32_to_bf16_bits(bf16_val(x) / 2), 0.0)
    assert np.array_equal(b2, 2 * b1) and np.array_equal(b2, 4 * bh)
    # each code is the nearest INT4 value to x*sqrt7/(beta+eps), ties to even (brute force)
    xf = bf16_val(x).astype(np.float32)
    for m in range(2):
        mult = np.float32(np.float32(math.sqrt(7)) / (np.float32(b2[m]) + np.float32(0.0)))
        for k in range(64):
            v = float(np.float32(xf[m, k] * mult))
            assert c2[m, k] == min(range(-8, 8), key=lambda c: (abs(v - c), c % 2))


def test_fp4_e1m2_hand_examples():
    # max|x| = 5 = 1.25 * 2^2 -> p = 2; x/4 = 0.0752, -0.3008, 1.25, 0.0175 ->
    # nearest of {0,.25,...,1.75}: indices 0, 1 (negative), 5, 0
    code4, fv, p, scale = oracle.quant_fp4_e1m2(bf16([[0.3, -1.2, 5.0, 0.07]]))
    assert p[0] == 2 and scale[0] == 4.0
    assert code4[0].tolist() == [0, 8 | 1, 5, 0]
    assert fv[0].tolist() == [0, -1, 5, 0]
    # ties to the even encoding: 0.125 (between 0 and .25) -> 0, 0.375 -> .5,
    # -0.625 (between .5 and .75) -> -.5; max 1.75 -> p = 0
    code4, fv, p, _ = oracle.quant_fp4_e1m2(bf16([[0.125, 0.375, 1.75, -0.625]]))
    assert p[0] == 0
    assert code4[0].tolist() == [0, 2, 7, 8 | 2]
    assert fv[0].tolist() == [0, 2, 7, -2]


@pytest.mark.parametrize("gmax,p", [(1.75, 0), (1.765625, 1), (0.875, -1), (3.5, 1), (3.515625, 2),
                                    (1.0, 0), (1e-3, -10)])
def test_fp4_e1m2_scale_exponent_closed_form(gmax, p):
    row = bf16([[gmax, -gmax / 4, 0.0, gmax / 3]])
    g = float(bf16_val(row)[0, 0])
    _, _, pp, scale = oracle.quant_fp4_e1m2(row)
    assert pp[0] == p
    assert g <= 1.75 * 2.0 ** p and g > 1.75 * 2.0 ** (p - 1)
    assert scale[0] == np.float32(2.0 ** p)


def test_fp4_e1m2_exhaustive_bf16_is_rint_of_4x():
    # On the uniform 0.25 grid, nearest-with-ties-to-even-index is rint(4|x|):
    # every finite bf16 magnitude up to 1.75 at p = 0
    bits = np.arange(0, 0x8000, dtype=np.uint16)
    vals = bf16_val(bits)
    keep = np.isfinite(vals) & (vals <= 1.75)
    bits = bits[keep]
    for sign in (0, 0x8000):
        b = (bits | sign).astype(np.uint16)
        row = np.concatenate([b, bf16([1.75])]).reshape(1, -1)
        code4, fv, p, _ = oracle.quant_fp4_e1m2(row)
        assert p[0] == 0
        v = bf16_val(b).astype(np.float64)
        idx = np.rint(4 * np.abs(v)).astype(np.int64)
        neg = (v < 0) & (idx != 0)
        assert np.array_equal(fv[0, :-1].astype(np.int64), np.where(neg, -idx, idx))
        assert np.array_equal(code4[0, :-1].astype(np.int64), idx | np.where(neg, 8, 0))


# ----------------------------------------------------------------------------
# RMSNorm ahead of the 4-bit quantizer (§3.2 data flow; formula a reading)
# ----------------------------------------------------------------------------
def test_rmsnorm_hand_examples():
    g = read_golden("rmsnorm_hand.txt")
    for xs, gs, ys in zip(g["x"], g["g"], g["y"]):
        y, _ = oracle.rmsnorm(bf16([xs]), gamma=np.array(gs, np.float32), eps_norm=1e-8)
        assert bf16_val(y)[0].tolist() == ys


def test_rmsnorm_within_bf16_rounding_of_exact():
    # y against the exact x * g / sqrt(mean(x^2) + eps) in fp64: within half a bf16
    # ulp plus the few fp32 roundings before it (relative 2^-8 covers both)
    g = synth.rng(61)
    x = synth.student_t_bf16(g, (16, 1536))
    w = (1.0 + 0.25 * g.standard_normal(1536)).astype(np.float32)
    y, _ = oracle.rmsnorm(x, gamma=w, eps_norm=1e-6)
    xf = bf16_val(x).astype(np.float64)
    exact = xf * w.astype(np.float64) / np.sqrt((xf ** 2).mean(axis=1, keepdims=True) + 1e-6)
    err = np.abs(bf16_val(y).astype(np.float64) - exact)
    assert np.all(err <= 2.0 ** -8 * np.abs(exact) + 1e-30)


def test_rmsnorm_constant_power_of_two_rows():
    # x = c everywhere with c a power of two: mean(x^2) = c^2 exactly, sqrt exact,
    # r = 1/|c| exactly, so y = sign(c) * g
    w = np.array([1.5, -0.25, 3.0, 0.125] * 8, np.float32)
    for c in (0.5, -4.0, 2.0 ** -20, 1024.0):
        y, r = oracle.rmsnorm(bf16([[c] * 32]), gamma=w, eps_norm=1e-30)
        assert float(r[0]) == 1.0 / abs(c)
        assert bf16_val(y)[0].tolist() == (np.sign(c) * w).tolist()


def test_rmsnorm_zero_row_and_eps():
    y, r = oracle.rmsnorm(np.zeros((1, 8), np.uint16), eps_norm=0.25)
    assert not y.any() and float(r[0]) == 2.0           # 1/sqrt(0 + 0.25)
    with pytest.raises(ValueError):
        oracle.rmsnorm(np.zeros((1, 8), np.uint16), eps_norm=0.0)


def test_rmsnorm_quant_constant_row_codes():
    # after the norm a constant row is all g; with g = 1, beta = 1 and every code is
    # RoundClip(sqrt7 / (1 + eps)) = 3 (INT4); for FP4 the smallest p with 1 <= 6 * 2^p
    # is -2, so every value is 1 * 2^2 = 4, E2M1 code 0b110
    c, b, _ = oracle.rmsnorm_quant(bf16([[-6.0] * 64, [0.375] * 64]), quant="int4")
    assert c.tolist() == [[-3] * 64, [3] * 64] and b.tolist() == [1.0, 1.0]
    code4, _, p, _ = oracle.rmsnorm_quant(bf16([[0.375] * 64]), quant="fp4")
    assert set(code4[0].tolist()) == {0x6} and p[0] == -2


# ----------------------------------------------------------------------------
# INT4 absmean with a per-tensor scale (ablations; Eq. 6-7 read over all of X)
# ----------------------------------------------------------------------------
def test_int4_per_tensor_hand_example():
    g = read_golden("int4_per_tensor_hand.txt")
    c, beta, scale = oracle.quant_int4_per_tensor(bf16(g["x"]))
    assert c.tolist() == [[int(v) for v in row] for row in g["codes"]]
    assert float(beta) == g["beta"][0][0]
    assert np.all(scale == np.float32(beta) / np.float32(math.sqrt(7)))


def test_int4_per_tensor_single_row_is_per_token():
    # with one token the tensor mean is the token mean: the pinned per-token quantizer
    x = synth.gaussian_bf16(synth.rng(62), (1, 3200))
    c1, b1, s1 = oracle.quant_int4(x)
    c2, b2, s2 = oracle.quant_int4_per_tensor(x)
    assert np.array_equal(c1, c2) and float(b1[0]) == float(b2) and s1[0] == s2[0]


def test_int4_per_tensor_beta_exact_mean_brute_force():
    # beta is the exact rational mean of |x| rounded once to fp32 (checked with
    # Fractions), and permuting the rows changes nothing but the row order
    g = synth.rng(63)
    x = synth.student_t_bf16(g, (7, 96))
    x[0, :5] = bf16([1e-30, 3e30, -2.5e-38, 65504.0, -1e-3])
    exact = sum(Fraction(float(abs(v))) for v in bf16_val(x).ravel()) / x.size
    c, beta, _ = oracle.quant_int4_per_tensor(x)
    assert float(beta) == float(oracle.round_fraction_to_f32(exact))
    perm = g.permutation(7)
    c2, beta2, _ = oracle.quant_int4_per_tensor(x[perm])
    assert float(beta2) == float(beta) and np.array_equal(c2, c[perm])


def test_int4_per_tensor_constant_tensor():
    c, beta, _ = oracle.quant_int4_per_tensor(bf16([[-0.5] * 16] * 3))
    assert float(beta) == 0.5 and set(c.ravel().tolist()) == {-3}


def test_rmsnorm_mean_is_exact_and_rejects_wide_rows():
    # ms is the exact mean of the squares rounded once: checked with Fractions on rows
    # that defeat a plain fp64 sum (squares spanning ~80 bits); a row whose squares
    # span beyond 106 bits is outside the contract and rejected
    g = synth.rng(64)
    x = synth.gaussian_bf16(g, (4, 512))
    x[1, :3] = bf16([1e-6, 3e3, -7e-7])
    y, r = oracle.rmsnorm(x, eps_norm=1e-6)
    for i in range(4):
        sq = sum(Fraction(float(v)) ** 2 for v in bf16_val(x[i]))
        ms = oracle.round_fraction_to_f32(sq / 512)
        s = np.sqrt(np.float32(ms) + np.float32(1e-6), dtype=np.float32)
        assert float(r[i]) == float(np.float32(1.0) / s)
    wide = np.zeros((1, 8), np.uint16)
    wide[0, :2] = bf16([1e30, 1e-30])
    with pytest.raises(ValueError):
        oracle.rmsnorm(wide)


# ---------------------------------------------------------------------------
# Low-bit attention over the quantized cache (§3.4 "Low-Bit KV Cache Quantization")
# ---------------------------------------------------------------------------
def _attention_case(g, c):
    M, T, bits, bos = (int(v) for v in g[c + "_meta"][0])
    D = len(g[c + "_q"][0])
    q = np.array(g[c + "_q"], np.uint8).reshape(M, 1, D)
    k = np.array(g[c + "_k"], np.uint8).reshape(T, 1, D)
    v = np.array(g[c + "_v"], np.uint8).reshape(T, 1, D)
    qs = np.array(g[c + "_qs"][0], np.float32).reshape(M, 1)
    ks = np.array(g[c + "_ks"][0], np.float32).reshape(T, 1)
    vs = np.array(g[c + "_vs"][0], np.float32).reshape(T, 1)
    o = oracle.attention_lowbit(q, qs, k, ks, v, vs, kv_bits=bits, bos_pos=bos,
                                softmax_scale=np.float32(g[c + "_sm"][0][0]))
    return o[:, 0, :], np.array(g[c + "_o"])


def test_attention_hand_examples():
    g = read_golden("attention_hand.txt")
    for c in ("c1", "c2", "c3"):
        o, want = _attention_case(g, c)
        np.testing.assert_allclose(o, want, rtol=0, atol=1e-6, err_msg=c)


def _random_cache(g, T, H, D, bits):
    k = g.integers(0, 1 << bits, (T, H, D)).astype(np.uint8)
    v = g.integers(0, 1 << bits, (T, H, D)).astype(np.uint8)
    ks = g.uniform(0.05, 2.0, (T, H)).astype(np.float32)
    vs = g.uniform(0.05, 2.0, (T, H)).astype(np.float32)
    return k, ks, v, vs


def _dequant(codes, scale, offset):
    return (codes.astype(np.float64) - offset) * scale.astype(np.float64)[..., None]


def test_attention_single_position_is_v():
    # softmax over one position is 1: the output is that position's dequantized V exactly
    g = synth.rng(70)
    for bits in (3, 4):
        k, ks, v, vs = _random_cache(g, 1, 3, 16, bits)
        q = g.integers(0, 16, (1, 3, 16)).astype(np.uint8)
        qs = g.uniform(0.1, 1.0, (1, 3)).astype(np.float32)
        o = oracle.attention_lowbit(q, qs, k, ks, v, vs, kv_bits=bits, bos_pos=-1)
        assert np.array_equal(o[0], _dequant(v[0], vs[0], 1 << (bits - 1)))


def test_attention_zero_query_is_the_mean_of_allowed_values():
    # q_hat = 0 makes every score 0: uniform weights over the positions the query sees
    g = synth.rng(71)
    T, H, D, M = 9, 2, 16, 3
    k, ks, v, vs = _random_cache(g, T, H, D, 3)
    q = np.full((M, H, D), 8, np.uint8)
    qs = np.ones((M, H), np.float32)
    o = oracle.attention_lowbit(q, qs, k, ks, v, vs, kv_bits=3, bos_pos=2)
    vh = _dequant(v, vs, 4.0)
    vh[2] = _dequant(v[2], vs[2], 8.0)          # the BOS position is 4-bit
    for m in range(M):
        np.testing.assert_allclose(o[m], vh[:T - M + m + 1].mean(axis=0), rtol=1e-12, atol=1e-12)


def test_attention_dominant_score_selects_its_value():
    # one score above all others by far more than 745 (fp64 exp underflows to 0):
    # the output is exactly that position's value; also checks that no overflow occurs
    g = synth.rng(72)
    T, H, D = 6, 1, 8
    k = np.full((T, H, D), 4, np.uint8)
    k[4, 0, 0] = 7                               # k_hat_4 = 3 e_0 * scale, the others 0
    ks = np.full((T, H), 1000.0, np.float32)
    v = g.integers(0, 8, (T, H, D)).astype(np.uint8)
    vs = g.uniform(0.1, 2.0, (T, H)).astype(np.float32)
    q = np.full((1, H, D), 8, np.uint8)
    q[0, 0, 0] = 15                              # q_hat = 7 e_0
    o = oracle.attention_lowbit(q, np.ones((1, H), np.float32), k, ks, v, vs, kv_bits=3, bos_pos=-1,
                                softmax_scale=np.float32(1.0))
    assert np.array_equal(o[0, 0], _dequant(v[4, 0], vs[4, 0], 4.0))


def test_attention_causal_mask_and_last_query():
    # query m sees positions 0..T-M+m: values at later positions do not move it, and
    # the last of M queries equals a single query over the whole cache
    g = synth.rng(73)
    T, H, D, M = 12, 2, 16, 4
    k, ks, v, vs = _random_cache(g, T, H, D, 3)
    q = g.integers(0, 16, (M, H, D)).astype(np.uint8)
    qs = g.uniform(0.1, 1.0, (M, H)).astype(np.float32)
    o = oracle.attention_lowbit(q, qs, k, ks, v, vs, kv_bits=3, bos_pos=0)
    k2, v2 = k.copy(), v.copy()
    k2[T - M + 1:] = 7 - k2[T - M + 1:]
    v2[T - M + 1:] = 7 - v2[T - M + 1:]
    o2 = oracle.attention_lowbit(q, qs, k2, ks, v2, vs, kv_bits=3, bos_pos=0)
    assert np.array_equal(o[0], o2[0]) and not np.array_equal(o[M - 1], o2[M - 1])
    o1 = oracle.attention_lowbit(q[M - 1:], qs[M - 1:], k, ks, v, vs, kv_bits=3, bos_pos=0)
    assert np.array_equal(o1[0], o[M - 1])


def test_attention_is_a_convex_combination_and_order_free():
    # every output lies between the smallest and largest allowed value per channel,
    # and permuting the cache positions (one query sees all of them) changes nothing
    g = synth.rng(74)
    T, H, D = 40, 3, 32
    k, ks, v, vs = _random_cache(g, T, H, D, 4)
    q = g.integers(0, 16, (1, H, D)).astype(np.uint8)
    qs = g.uniform(0.1, 1.0, (1, H)).astype(np.float32)
    o = oracle.attention_lowbit(q, qs, k, ks, v, vs, kv_bits=4)
    vh = _dequant(v, vs, 8.0)
    assert np.all(o[0] >= vh.min(axis=0) - 1e-12) and np.all(o[0] <= vh.max(axis=0) + 1e-12)
    perm = g.permutation(T)
    op = oracle.attention_lowbit(q, qs, k[perm], ks[perm], v[perm], vs[perm], kv_bits=4)
    np.testing.assert_allclose(op, o, rtol=1e-12, atol=1e-12)


def test_attention_of_quantized_cache_approaches_full_precision():
    # with the cache quantized by the pinned kv_quant at 4 bits and a 4-bit query, the
    # output stays within the quantization error of full-precision attention on the
    # bf16 inputs (each dequantized value is off by at most half a step, gamma/(2*7))
    g = synth.rng(75)
    T, H, D = 64, 2, 32
    x = synth.gaussian_bf16(g, (3 * T, H, D))
    kc, ksc = oracle.kv_quant(x[:T], bits=4, bos_pos=-1)
    vc, vsc = oracle.kv_quant(x[T:2 * T], bits=4, bos_pos=-1)
    qc, qsc = oracle.kv_quant(x[2 * T:2 * T + 1], bits=4, bos_pos=-1)
    o = oracle.attention_lowbit(qc, qsc, kc, ksc, vc, vsc, kv_bits=4)
    xf = bf16_val(x).astype(np.float64)
    K, V, Q = xf[:T], xf[T:2 * T], xf[2 * T]
    for h in range(H):
        s = (K[:, h, :] @ Q[h]) / np.sqrt(D)
        p = np.exp(s - s.max())
        ref = (p @ V[:, h, :]) / p.sum()
        assert np.max(np.abs(o[0, h] - ref)) < 0.35    # loose: 4-bit Q and K move the weights too
        assert np.corrcoef(o[0, h], ref)[0, 1] > 0.9
