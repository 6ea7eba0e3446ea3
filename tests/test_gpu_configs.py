"""GPU parity of the whole BitLinear path at the 700M-layer and 3B-set shapes
(the 7B layer is covered at full size in test_gpu_fullsize.py, the tiny
config in test_gpu_gemm.py).  Every step runs on the GPU at the config's full
token count; the quantizers' codes and scales are compared in full, the Top-K
steps and the matmuls on a seeded sample of rows (the oracle's ranking and
matmul are slow), and the Top-K survivor count on every row.  The shapes carry
GEMM K tails that the 7B shapes do not (K = 1536, 3200, 8640 against 128-wide
K blocks) and other N (4608, 9600, 8192, 17280)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_bit_activation_b200 as tba
from gpu_util import BF16_ROW_TOL, bf16_rows_rel_err, empty, host, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

EPS = 1e-5


def sample_rows(n, k, seed):
    g = synth.rng(seed)
    return np.unique(np.concatenate([[0, n - 1], g.choice(n, size=k, replace=False)]))


def pack_i8(w):
    n, k = w.shape
    out = empty((n, k), torch.int8)
    alpha = empty((1,), torch.float32)
    ws = empty((tba.workspace_size("pack_ternary") // 8,), torch.int64)
    tba.pack_ternary(to_dev(w), alpha, out.view(torch.uint8), tba.BL_W_I8, ws, eps=EPS)
    tba.sync_status()
    t_ref, a_ref = oracle.ternary_quantize(w, EPS)
    assert host(alpha).view(np.uint32)[0] == np.float32(a_ref).view(np.uint32)
    assert np.array_equal(host(out), t_ref)
    return out, alpha, t_ref, np.float32(a_ref)


def check_gemm(a_codes, a_scale, t, alpha, y_gpu, rows, group=0):
    acc_ref, _ = oracle.gemm(a_codes, a_scale, t, alpha, alpha_group=group, rows=rows, want_y=False)
    al = np.atleast_1d(np.asarray(alpha, np.float64))
    n = t.shape[0]
    col_alpha = al[np.arange(n) // (group if group else n)]
    exact = acc_ref.astype(np.float64) * a_scale[rows, None].astype(np.float64) * col_alpha[None, :]
    assert bf16_rows_rel_err(y_gpu[rows], exact) <= BF16_ROW_TOL
    return acc_ref


@pytest.mark.parametrize("shape", [synth.L700M, synth.L3B], ids=["700M", "3B"])
def test_layer_path(shape):
    m, d, f = shape.tokens, shape.hidden, shape.ffn
    x_attn, x_o, x_ffn = synth.layer_activations(shape, seed=synth.SEEDS[shape.name], tokens=m)
    wts = synth.layer_weights(shape, seed=synth.SEEDS[shape.name] + 10)
    rows = sample_rows(m, 62, seed=m + d)

    # ternary weights (int8 layout, the prefill operand), codes in full
    w_qkv, a_qkv, t_qkv, al_qkv = pack_i8(wts["qkv"])
    w_o, a_o, t_o, al_o = pack_i8(wts["o"])
    w_up, a_up, t_up, al_up = pack_i8(wts["up"])
    w_gate, a_gate, t_gate, al_gate = pack_i8(wts["gate"])
    w_down, a_down, t_down, al_down = pack_i8(wts["down"])

    # INT4 quant -> QKV GEMM
    qa = empty((m, d), torch.int8)
    qs = empty((m,), torch.float32)
    tba.bitlinear_quant_a4(to_dev(x_attn), qa, qs, tba.BL_QUANT_INT4, tba.BL_STORE_BYTES, EPS)
    tba.sync_status()
    c_ref, _, s_ref = oracle.quant_int4(x_attn, EPS)
    assert np.array_equal(host(qa), c_ref)
    assert np.array_equal(host(qs).view(np.uint32), s_ref.view(np.uint32))
    y = empty((m, 3 * d), torch.int16)
    acc = empty((m, 3 * d), torch.int32)
    tba.bitlinear_gemm(qa, qs, w_qkv, a_qkv, m, 3 * d, d, y=y, acc=acc)
    tba.sync_status()
    acc_ref = check_gemm(c_ref, s_ref, t_qkv, al_qkv, host(y, np.uint16), rows)
    assert np.array_equal(host(acc)[rows], acc_ref)

    # Top-K 50% + INT8 -> O GEMM
    keep_o = synth.k_keep(d, shape.topk_pct_o)
    o8 = empty((m, d), torch.int8)
    o8_s = empty((m,), torch.float32)
    mask = empty((m, (d + 31) // 32), torch.int32)
    tba.bitlinear_sparsify_a8(to_dev(x_o), keep_o, o8, o8_s, mask, EPS)
    tba.sync_status()
    mask_h = host(mask).view(np.uint32)
    counts = np.unpackbits(mask_h.view(np.uint8), axis=1).sum(axis=1)
    assert np.all(counts == keep_o)
    c_o, mask_ref, _, s_o = oracle.sparsify_a8(x_o[rows], keep_o, EPS)
    assert np.array_equal(host(o8)[rows], c_o)
    assert np.array_equal(mask_h[rows], oracle.pack_mask_bits(mask_ref))
    assert np.array_equal(host(o8_s).view(np.uint32)[rows], s_o.view(np.uint32))
    y_o = empty((m, d), torch.int16)
    acc_o = empty((m, d), torch.int32)
    tba.bitlinear_gemm(o8, o8_s, w_o, a_o, m, d, d, y=y_o, acc=acc_o)
    tba.sync_status()
    o8_h, o8s_h = host(o8), host(o8_s)
    acc_ref = check_gemm(o8_h, o8s_h, t_o, al_o, host(y_o, np.uint16), rows)
    assert np.array_equal(host(acc_o)[rows], acc_ref)

    # INT4 quant -> Up|Gate GEMM (stacked, one alpha each) -> ReLU^2-GLU + Top-K -> Down GEMM
    tba.bitlinear_quant_a4(to_dev(x_ffn), qa, qs, tba.BL_QUANT_INT4, tba.BL_STORE_BYTES, EPS)
    tba.sync_status()
    c_f, _, s_f = oracle.quant_int4(x_ffn, EPS)
    assert np.array_equal(host(qa), c_f)
    w_ug = torch.cat([w_up, w_gate])
    al_ug = torch.cat([a_up, a_gate])
    y_ug = empty((m, 2 * f), torch.int16)
    acc_ug = empty((m, 2 * f), torch.int32)
    tba.bitlinear_gemm(qa, qs, w_ug, al_ug, m, 2 * f, d, y=y_ug, acc=acc_ug, alpha_group=f)
    tba.sync_status()
    t_ug = np.concatenate([t_up, t_gate])
    acc_ref = check_gemm(c_f, s_f, t_ug, np.array([al_up, al_gate], np.float32), host(y_ug, np.uint16), rows,
                         group=f)
    assert np.array_equal(host(acc_ug)[rows], acc_ref)
    keep_d = synth.k_keep(f, shape.topk_pct_down)
    h8 = empty((m, f), torch.int8)
    h8_s = empty((m,), torch.float32)
    tba.relu2_glu(y_ug[:, f:], y_ug[:, :f], keep_d, h8, h8_s, None, EPS, M=m, F=f, ld=2 * f)
    tba.sync_status()
    ug = host(y_ug, np.uint16)
    c_h, _, _, s_h = oracle.relu2_glu(ug[rows, f:], ug[rows, :f], keep_d, EPS)
    h8_h, h8s_h = host(h8), host(h8_s)
    assert np.array_equal(h8_h[rows], c_h)
    assert np.array_equal(h8s_h.view(np.uint32)[rows], s_h.view(np.uint32))
    y_d = empty((m, d), torch.int16)
    acc_d = empty((m, d), torch.int32)
    tba.bitlinear_gemm(h8, h8_s, w_down, a_down, m, d, f, y=y_d, acc=acc_d)
    tba.sync_status()
    acc_ref = check_gemm(h8_h, h8s_h, t_down, al_down, host(y_d, np.uint16), rows)
    assert np.array_equal(host(acc_d)[rows], acc_ref)
