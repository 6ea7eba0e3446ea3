"""GPU parity at the full 7B-layer sizes the benchmark runs (M = 8 x 4096
tokens, hidden 4096, FFN 11008, 32 x 128 heads), through the C ABI in the same
launch configuration.  Where the oracle is fast the whole output is compared;
where it is slow (Top-K ranking, the matmul) a seeded sample of rows is compared
element by element and properties that hold at any size are checked on every
row."""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_bit_activation_b200 as tba
from gpu_util import BF16_ROW_TOL, bf16_rows_rel_err, empty, host, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

EPS = 1e-5
S = synth.L7B
M = S.tokens
D = S.hidden
F = S.ffn


def sample_rows(n, k, seed):
    g = synth.rng(seed)
    rows = np.sort(g.choice(n, size=k, replace=False))
    return np.unique(np.concatenate([[0, n - 1], rows]))


@pytest.fixture(scope="module")
def acts():
    x_attn, x_o, _ = synth.layer_activations(S, seed=S.tokens, tokens=M)
    return x_attn, x_o


def test_quant_int4_full_7b(acts):
    x = acts[0]
    xd = to_dev(x)
    codes = empty((M, D), torch.uint8)
    scale = empty((M,), torch.float32)
    tba.bitlinear_quant_a4(xd, codes, scale, tba.BL_QUANT_INT4, tba.BL_STORE_BYTES, EPS)
    tba.sync_status()
    c_ref, _, s_ref = oracle.quant_int4(x, EPS)
    assert np.array_equal(host(codes).view(np.int8), c_ref)
    assert np.array_equal(host(scale).view(np.uint32), s_ref.view(np.uint32))


def test_quant_fp4_packed_full_7b(acts):
    x = acts[0]
    xd = to_dev(x)
    codes = empty((M, D // 2), torch.uint8)
    scale = empty((M,), torch.float32)
    tba.bitlinear_quant_a4(xd, codes, scale, tba.BL_QUANT_FP4_E2M1, tba.BL_STORE_PACKED, EPS)
    tba.sync_status()
    code4, _, _, s_ref = oracle.quant_fp4(x)
    assert np.array_equal(host(codes), oracle.pack_nibbles(code4))
    assert np.array_equal(host(scale).view(np.uint32), s_ref.view(np.uint32))


def test_sparsify_full_7b(acts):
    x = acts[1]
    keep = synth.k_keep(D, S.topk_pct_o)
    xd = to_dev(x)
    codes = empty((M, D), torch.int8)
    scale = empty((M,), torch.float32)
    mask = empty((M, D // 32), torch.int32)
    tba.bitlinear_sparsify_a8(xd, keep, codes, scale, mask, EPS)
    tba.sync_status()
    c, s, mk = host(codes), host(scale), host(mask, np.uint32)
    # every row: exactly keep survivors, codes zero outside the mask
    pop = np.unpackbits(mk.view(np.uint8), axis=1).sum(axis=1)
    assert np.all(pop == keep)
    bits = np.unpackbits(mk.view(np.uint8), axis=1, bitorder="little").astype(bool)
    assert not np.any(c[~bits])
    rows = sample_rows(M, 96, 1)
    c_ref, m_ref, _, s_ref = oracle.sparsify_a8(x[rows], keep, EPS)
    assert np.array_equal(c[rows], c_ref)
    assert np.array_equal(mk[rows], oracle.pack_mask_bits(m_ref))
    assert np.array_equal(s[rows].view(np.uint32), s_ref.view(np.uint32))


def test_relu2_glu_full_7b():
    gate, up = synth.glu_inputs(M, F, seed=7, gate_shift=0.0)
    both = np.empty((M, 2 * F), np.uint16)
    both[:, :F] = up
    both[:, F:] = gate
    d = to_dev(both)
    del both
    keep = synth.k_keep(F, S.topk_pct_down)
    codes = empty((M, F), torch.int8)
    scale = empty((M,), torch.float32)
    mask = empty((M, (F + 31) // 32), torch.int32)
    tba.relu2_glu(d[:, F:], d[:, :F], keep, codes, scale, mask, EPS, M=M, F=F, ld=2 * F)
    tba.sync_status()
    c, s, mk = host(codes), host(scale), host(mask, np.uint32)
    pop = np.unpackbits(mk.view(np.uint8), axis=1).sum(axis=1)
    assert np.all(pop == keep)
    rows = sample_rows(M, 48, 2)
    c_ref, m_ref, _, s_ref = oracle.relu2_glu(gate[rows], up[rows], keep, EPS)
    assert np.array_equal(c[rows], c_ref)
    assert np.array_equal(mk[rows], oracle.pack_mask_bits(m_ref))
    assert np.array_equal(s[rows].view(np.uint32), s_ref.view(np.uint32))


def test_kv_quant3_full():
    T, H, Dh = synth.KV_SHAPE
    k, _ = synth.kv_inputs(5)
    kd = to_dev(k.reshape(T, H * Dh))
    codes = empty((T, H, Dh * 3 // 8), torch.uint8)
    scale = empty((T, H), torch.float32)
    bos = empty((H, Dh // 2), torch.uint8)
    tba.kv_quant3(kd, T, H, Dh, codes, scale, bos, bits=3, bos_pos=0, eps=EPS)
    tba.sync_status()
    cu, s_ref = oracle.kv_quant(k, bits=3, bos_pos=0, eps=EPS)
    assert np.array_equal(host(scale).view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(host(codes)[1:], oracle.pack_kv3(cu[1:]))
    assert np.array_equal(host(bos), oracle.pack_nibbles(cu[0]))


@pytest.fixture(scope="module")
def up_weights():
    return synth.latent_weights_f32(synth.rng(77), F, D)


@pytest.mark.parametrize("wfmt", [tba.BL_W_I8, tba.BL_W_T2], ids=["i8", "t2"])
def test_pack_ternary_full_7b_up(up_weights, wfmt):
    w = up_weights
    wd = to_dev(w)
    out = empty((F, D if wfmt == tba.BL_W_I8 else D // 4), torch.uint8)
    alpha = empty((1,), torch.float32)
    ws = empty((tba.workspace_size("pack_ternary") // 8,), torch.int64)
    tba.pack_ternary(wd, alpha, out, wfmt, ws, eps=EPS)
    tba.sync_status()
    t_ref, a_ref = oracle.ternary_quantize(w, EPS)
    assert host(alpha).view(np.uint32)[0] == np.float32(a_ref).view(np.uint32)
    if wfmt == tba.BL_W_I8:
        assert np.array_equal(host(out).view(np.int8), t_ref)
    else:
        assert np.array_equal(host(out), oracle.pack_ternary2(t_ref))


@pytest.mark.parametrize("name,N,K", [("qkv", 3 * D, D), ("down", D, F)])
def test_gemm_tc_full_7b(name, N, K):
    g = synth.rng(N + K)
    a = g.integers(-128, 128, (M, K), dtype=np.int16).astype(np.int8)
    t = g.integers(-1, 2, (N, K), dtype=np.int16).astype(np.int8)
    s = (g.random(M) * 0.01 + 1e-4).astype(np.float32)
    alpha = np.float32(0.0156)
    acc = empty((M, N), torch.int32)
    y = empty((M, N), torch.int16)
    tba.bitlinear_gemm(to_dev(a), to_dev(s), to_dev(t), to_dev(np.array([alpha])), M, N, K, y=y, acc=acc)
    tba.sync_status()
    rows = sample_rows(M, 40, 3)
    acc_h = host(acc)[rows]
    acc_ref, _ = oracle.gemm(a, s, t, alpha, rows=rows, want_y=False)
    assert np.array_equal(acc_h, acc_ref)
    exact = acc_ref.astype(np.float64) * s[rows, None].astype(np.float64) * float(alpha)
    assert bf16_rows_rel_err(host(y, np.uint16)[rows], exact) <= BF16_ROW_TOL


def test_gemm_fp4_mxf4_full_7b_qkv(acts):
    """The FP4 variant's QKV GEMM at full size: FP4 E2M1 activations x
    E2M1-coded ternary weights on kind::mxf4; sampled rows against the oracle."""
    x = acts[0]
    N, K = 3 * D, D
    w = synth.latent_weights_f32(synth.rng(91), N, K)
    t_ref, a_ref = oracle.ternary_quantize(w, EPS)
    codes = empty((M, K // 2), torch.uint8)
    scale = empty((M,), torch.float32)
    tba.bitlinear_quant_a4(to_dev(x), codes, scale, tba.BL_QUANT_FP4_E2M1, tba.BL_STORE_PACKED, EPS)
    wdev = empty((N, K // 2), torch.uint8)
    alpha = empty((1,), torch.float32)
    ws = empty((tba.workspace_size("pack_ternary") // 8,), torch.int64)
    tba.pack_ternary(to_dev(w), alpha, wdev, tba.BL_W_E2M1, ws, eps=EPS)
    acc = empty((M, N), torch.int32)
    y = empty((M, N), torch.int16)
    tba.bitlinear_gemm(codes, scale, wdev, alpha, M, N, K, y=y, acc=acc, afmt=tba.BL_A_E2M1, wfmt=tba.BL_W_E2M1)
    tba.sync_status()
    assert np.array_equal(host(wdev), oracle.pack_ternary_e2m1(t_ref))
    rows = sample_rows(M, 40, 4)
    code4, twice, _, s_ref = oracle.quant_fp4(x[rows])
    assert np.array_equal(host(codes)[rows], oracle.pack_nibbles(code4))
    acc_scale = (s_ref.astype(np.float64) / 2).astype(np.float32)
    acc_ref, _ = oracle.gemm(twice, acc_scale, t_ref, a_ref, want_y=False)
    assert np.array_equal(host(acc)[rows], acc_ref)
    exact = acc_ref.astype(np.float64) * acc_scale[:, None].astype(np.float64) * float(a_ref)
    assert bf16_rows_rel_err(host(y, np.uint16)[rows], exact) <= BF16_ROW_TOL


@pytest.mark.parametrize("m", [1, 8])
def test_decode_gemm_full_7b_qkv(up_weights, m):
    # 2-bit weights of a 7B-size matrix against m INT4-packed tokens
    w = up_weights
    t_ref, a_ref = oracle.ternary_quantize(w, EPS)
    x = synth.gaussian_bf16(synth.rng(m), (m, D))
    c, _, s = oracle.quant_int4(x, EPS)
    acc = empty((m, F), torch.int32)
    y = empty((m, F), torch.int16)
    tba.bitlinear_gemm(to_dev(oracle.pack_nibbles(c)), to_dev(s), to_dev(oracle.pack_ternary2(t_ref)),
                       to_dev(np.array([a_ref], np.float32)), m, F, D, y=y, acc=acc, afmt=tba.BL_A_I4,
                       wfmt=tba.BL_W_T2)
    tba.sync_status()
    acc_ref, _ = oracle.gemm(c, s, t_ref, a_ref, want_y=False)
    assert np.array_equal(host(acc), acc_ref)


@pytest.fixture(scope="module")
def decode_weights():
    """The four 7B-layer matrices packed to 2 bits on the GPU, with the
    oracle's codes and alphas (Up and Gate stacked, one alpha each)."""
    wts = synth.layer_weights(S, seed=11)
    out = {}
    for name in ("qkv", "o", "down"):
        t_ref, a_ref = oracle.ternary_quantize(wts[name], EPS)
        out[name] = (t_ref, np.array([a_ref], np.float32))
    t_up, a_up = oracle.ternary_quantize(wts["up"], EPS)
    t_gate, a_gate = oracle.ternary_quantize(wts["gate"], EPS)
    out["upgate"] = (np.concatenate([t_up, t_gate]), np.array([a_up, a_gate], np.float32))
    dev = {}
    ws = empty((tba.workspace_size("pack_ternary") // 8,), torch.int64)
    for name, (t_ref, a_ref) in out.items():
        n, k = t_ref.shape
        packed = empty((n, k // 4), torch.uint8)
        alpha = empty((a_ref.size,), torch.float32)
        srcs = [wts[name]] if name != "upgate" else [wts["up"], wts["gate"]]
        for i, w in enumerate(srcs):
            rows = slice(i * w.shape[0], (i + 1) * w.shape[0])
            tba.pack_ternary(to_dev(w), alpha[i:i + 1], packed[rows], tba.BL_W_T2, ws, eps=EPS)
            tba.sync_status()
        assert np.array_equal(host(alpha).view(np.uint32), a_ref.view(np.uint32)), name
        assert np.array_equal(host(packed), oracle.pack_ternary2(t_ref)), name
        dev[name] = (packed, alpha)
    return out, dev


@pytest.mark.parametrize("m", [1, 2, 4, 8, 16])
def test_decode_layer_7b(decode_weights, m):
    """One decode step of a 7B layer, stage by stage, as the decode benchmark
    runs it (packed INT4 / INT8 activations against 2-bit weights).  Each stage
    is checked against the oracle on the same input bytes the GPU stage read."""
    ref, dev = decode_weights
    x_attn, x_o, x_ffn = synth.layer_activations(S, seed=500 + m, tokens=m)
    keep_o, keep_d = synth.k_keep(D, S.topk_pct_o), synth.k_keep(F, S.topk_pct_down)

    def gemm_stage(a_dev, afmt, a_scale_dev, name, a_codes, a_scale, n, k, group=0):
        acc = empty((m, n), torch.int32)
        y = empty((m, n), torch.int16)
        packed, alpha = dev[name]
        tba.bitlinear_gemm(a_dev, a_scale_dev, packed, alpha, m, n, k, y=y, acc=acc, afmt=afmt,
                           wfmt=tba.BL_W_T2, alpha_group=group if group else n)
        tba.sync_status()
        t_ref, a_ref = ref[name]
        acc_ref, _ = oracle.gemm(a_codes, a_scale, t_ref, a_ref, alpha_group=group, want_y=False)
        assert np.array_equal(host(acc), acc_ref), name
        al = np.repeat(a_ref.astype(np.float64), group if group else n)[:n]
        exact = acc_ref.astype(np.float64) * a_scale[:, None].astype(np.float64) * al[None, :]
        assert bf16_rows_rel_err(host(y, np.uint16), exact) <= BF16_ROW_TOL, name
        return y

    def quant4(x):
        qa = empty((m, D // 2), torch.uint8)
        qs = empty((m,), torch.float32)
        tba.bitlinear_quant_a4(to_dev(x), qa, qs, tba.BL_QUANT_INT4, tba.BL_STORE_PACKED, EPS)
        tba.sync_status()
        c, _, s = oracle.quant_int4(x, EPS)
        assert np.array_equal(host(qa), oracle.pack_nibbles(c))
        assert np.array_equal(host(qs).view(np.uint32), s.view(np.uint32))
        return qa, qs, c, s

    qa, qs, c, s = quant4(x_attn)
    gemm_stage(qa, tba.BL_A_I4, qs, "qkv", c, s, 3 * D, D)

    o8 = empty((m, D), torch.int8)
    o8_s = empty((m,), torch.float32)
    tba.bitlinear_sparsify_a8(to_dev(x_o), keep_o, o8, o8_s, None, EPS)
    tba.sync_status()
    c_o, _, _, s_o = oracle.sparsify_a8(x_o, keep_o, EPS)
    assert np.array_equal(host(o8), c_o)
    assert np.array_equal(host(o8_s).view(np.uint32), s_o.view(np.uint32))
    gemm_stage(o8, tba.BL_A_I8, o8_s, "o", c_o, s_o, D, D)

    qa, qs, c, s = quant4(x_ffn)
    y_ug = gemm_stage(qa, tba.BL_A_I4, qs, "upgate", c, s, 2 * F, D, group=F)

    h8 = empty((m, F), torch.int8)
    h8_s = empty((m,), torch.float32)
    tba.relu2_glu(y_ug[:, F:], y_ug[:, :F], keep_d, h8, h8_s, None, EPS, M=m, F=F, ld=2 * F)
    tba.sync_status()
    ug = host(y_ug, np.uint16)
    c_h, _, _, s_h = oracle.relu2_glu(ug[:, F:], ug[:, :F], keep_d, EPS)
    assert np.array_equal(host(h8), c_h)
    assert np.array_equal(host(h8_s).view(np.uint32), s_h.view(np.uint32))
    gemm_stage(h8, tba.BL_A_I8, h8_s, "down", c_h, s_h, D, F)


def test_gemm_upgate_full_7b(acts):
    """The stacked Up|Gate GEMM as the benchmark runs it: N = 2F = 22016 rows
    [W_up; W_gate] with one alpha per tensor (alpha_group = F), INT4 byte codes
    of a Gaussian input, M = 32768; sampled rows against the oracle."""
    x = acts[0]
    wu = synth.latent_weights_f32(synth.rng(93), F, D)
    wg = synth.latent_weights_f32(synth.rng(94), F, D)
    t_up, a_up = oracle.ternary_quantize(wu, EPS)
    t_gate, a_gate = oracle.ternary_quantize(wg, EPS)
    w8 = empty((2 * F, D), torch.uint8)
    alpha = empty((2,), torch.float32)
    ws = empty((tba.workspace_size("pack_ternary") // 8,), torch.int64)
    tba.pack_ternary(to_dev(wu), alpha[0:1], w8[:F], tba.BL_W_I8, ws, eps=EPS)
    tba.pack_ternary(to_dev(wg), alpha[1:2], w8[F:], tba.BL_W_I8, ws, eps=EPS)
    codes = empty((M, D), torch.uint8)
    scale = empty((M,), torch.float32)
    tba.bitlinear_quant_a4(to_dev(x), codes, scale, tba.BL_QUANT_INT4, tba.BL_STORE_BYTES, EPS)
    y = empty((M, 2 * F), torch.int16)
    acc = empty((M, 2 * F), torch.int32)
    tba.bitlinear_gemm(codes, scale, w8, alpha, M, 2 * F, D, y=y, acc=acc, alpha_group=F)
    tba.sync_status()
    a_ref = np.array([a_up, a_gate], np.float32)
    assert np.array_equal(host(alpha).view(np.uint32), a_ref.view(np.uint32))
    rows = sample_rows(M, 24, 5)
    c_ref, _, s_ref = oracle.quant_int4(x[rows], EPS)
    assert np.array_equal(host(codes)[rows].view(np.int8), c_ref)
    t_ref = np.concatenate([t_up, t_gate])
    acc_ref, _ = oracle.gemm(c_ref, s_ref, t_ref, a_ref, alpha_group=F, want_y=False)
    assert np.array_equal(host(acc)[rows], acc_ref)
    al = np.repeat(a_ref.astype(np.float64), F)
    exact = acc_ref.astype(np.float64) * s_ref[:, None].astype(np.float64) * al[None, :]
    assert bf16_rows_rel_err(host(y, np.uint16)[rows], exact) <= BF16_ROW_TOL


def test_gemm_o_full_7b_topk_codes(acts):
    """The O GEMM as the benchmark runs it: the Top-K 50% INT8 codes of the
    heavy-tailed O input (from the GPU quantizer) x int8 ternary weights,
    M = 32768, N = K = 4096; sampled rows against the oracle."""
    x = acts[1]
    keep = synth.k_keep(D, S.topk_pct_o)
    w = synth.latent_weights_f32(synth.rng(95), D, D)
    t_ref, a_ref = oracle.ternary_quantize(w, EPS)
    w8 = empty((D, D), torch.uint8)
    alpha = empty((1,), torch.float32)
    ws = empty((tba.workspace_size("pack_ternary") // 8,), torch.int64)
    tba.pack_ternary(to_dev(w), alpha, w8, tba.BL_W_I8, ws, eps=EPS)
    c8 = empty((M, D), torch.int8)
    s8 = empty((M,), torch.float32)
    tba.bitlinear_sparsify_a8(to_dev(x), keep, c8, s8, None, EPS)
    y = empty((M, D), torch.int16)
    acc = empty((M, D), torch.int32)
    tba.bitlinear_gemm(c8, s8, w8, alpha, M, D, D, y=y, acc=acc)
    tba.sync_status()
    rows = sample_rows(M, 32, 6)
    c_ref, _, _, s_ref = oracle.sparsify_a8(x[rows], keep, EPS)
    assert np.array_equal(host(c8)[rows], c_ref)
    acc_ref, _ = oracle.gemm(c_ref, s_ref, t_ref, a_ref, want_y=False)
    assert np.array_equal(host(acc)[rows], acc_ref)
    exact = acc_ref.astype(np.float64) * s_ref[:, None].astype(np.float64) * float(a_ref)
    assert bf16_rows_rel_err(host(y, np.uint16)[rows], exact) <= BF16_ROW_TOL


@pytest.mark.parametrize("m", [17, 32, 64, 128, 256])
def test_decode_layer_7b_tensor_cores(decode_weights, m):
    """Decode of 17-256 tokens as the decode benchmark runs it: one-byte INT4 /
    Top-K INT8 codes against the 2-bit weights of all four 7B matrices, which
    takes the tcgen05 kernel with the weights widened into tensor memory.
    Every GPU stage reads the previous GPU stage's output; each product is
    checked on a seeded sample of token rows (all N) against the oracle."""
    ref, dev = decode_weights
    x_attn, x_o, x_ffn = synth.layer_activations(S, seed=900 + m, tokens=m)
    keep_o, keep_d = synth.k_keep(D, S.topk_pct_o), synth.k_keep(F, S.topk_pct_down)
    rows = np.arange(m) if m <= 32 else sample_rows(m, 14, m)

    def gemm_stage(a_dev, a_scale_dev, name, n, k, group=0):
        acc = empty((m, n), torch.int32)
        y = empty((m, n), torch.int16)
        packed, alpha = dev[name]
        tba.bitlinear_gemm(a_dev, a_scale_dev, packed, alpha, m, n, k, y=y, acc=acc, afmt=tba.BL_A_I8,
                           wfmt=tba.BL_W_T2, alpha_group=group if group else n)
        tba.sync_status()
        t_ref, a_ref = ref[name]
        a_codes = host(a_dev).view(np.int8)[rows]
        a_scale = host(a_scale_dev)[rows]
        acc_ref, _ = oracle.gemm(a_codes, a_scale, t_ref, a_ref, alpha_group=group, want_y=False)
        assert np.array_equal(host(acc)[rows], acc_ref), name
        al = np.repeat(a_ref.astype(np.float64), group if group else n)[:n]
        exact = acc_ref.astype(np.float64) * a_scale[:, None].astype(np.float64) * al[None, :]
        assert bf16_rows_rel_err(host(y, np.uint16)[rows], exact) <= BF16_ROW_TOL, name
        return y

    def quant4(x):
        qa = empty((m, D), torch.int8)
        qs = empty((m,), torch.float32)
        tba.bitlinear_quant_a4(to_dev(x), qa, qs, tba.BL_QUANT_INT4, tba.BL_STORE_BYTES, EPS)
        tba.sync_status()
        c, _, s = oracle.quant_int4(x, EPS)
        assert np.array_equal(host(qa), c)
        assert np.array_equal(host(qs).view(np.uint32), s.view(np.uint32))
        return qa, qs

    qa, qs = quant4(x_attn)
    gemm_stage(qa, qs, "qkv", 3 * D, D)
    o8 = empty((m, D), torch.int8)
    o8_s = empty((m,), torch.float32)
    tba.bitlinear_sparsify_a8(to_dev(x_o), keep_o, o8, o8_s, None, EPS)
    gemm_stage(o8, o8_s, "o", D, D)
    qf, qfs = quant4(x_ffn)
    y_ug = gemm_stage(qf, qfs, "upgate", 2 * F, D, group=F)
    h8 = empty((m, F), torch.int8)
    h8_s = empty((m,), torch.float32)
    tba.relu2_glu(y_ug[:, F:], y_ug[:, :F], keep_d, h8, h8_s, None, EPS, M=m, F=F, ld=2 * F)
    tba.sync_status()
    ug = host(y_ug, np.uint16)[rows]
    c_h, _, _, s_h = oracle.relu2_glu(np.ascontiguousarray(ug[:, F:]), np.ascontiguousarray(ug[:, :F]), keep_d, EPS)
    assert np.array_equal(host(h8)[rows], c_h)
    gemm_stage(h8, h8_s, "down", D, F)
