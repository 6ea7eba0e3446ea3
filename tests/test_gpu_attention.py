"""GPU parity of attention_lowbit (softmax attention of 4-bit queries over the
3-/4-bit KV cache, §3.4 "Low-Bit KV Cache Quantization", Table 3) against the
fp64 oracle.

Tolerance, from the kernel's arithmetic: <q, k> is exact (integers); the
scores, exponentials and sums are fp32, each a few ulp, over at most a few
hundred terms per partial sum, so the pre-rounding error stays far below
2^-12 max_t |v_hat_t| of the (query, head); the output is then rounded once to
bf16 (half an ulp, 2^-9 relative).  Bound used per element:
|out - o| <= 2^-8 |o| + 2^-12 max_t |v_hat_t|."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_bit_activation_b200 as tba
from gpu_util import CANARY, canaried, empty, host, to_dev

pytestmark = pytest.mark.gpu
EPS = 1e-5


def quant_cache(x_bf16, bits, bos_pos):
    """kv_quant3 on the GPU: packed codes, scales and the BOS row."""
    T, H, D = x_bf16.shape
    codes = empty((T, H, D * bits // 8), torch.uint8)
    scale = empty((T, H), torch.float32)
    bos = empty((H, D // 2), torch.uint8)
    tba.kv_quant3(to_dev(x_bf16), T, H, D, codes, scale, bos_codes=bos, bits=bits, bos_pos=bos_pos, eps=EPS)
    return codes, scale, bos


def run_attention(q, qs, k, ks, kb, v, vs, vb, M, T, H, D, bits, bos_pos, sm, ldo=None):
    ldo = H * D if ldo is None else ldo
    out = empty((M, ldo), torch.int16)
    ws = empty((tba.workspace_size("attention_lowbit", M, H, D) // 4,), torch.float32)
    tba.attention_lowbit(q, qs, M, k, ks, v, vs, T, H, D, out, ws, k_bos=kb, v_bos=vb, kv_bits=bits,
                         bos_pos=bos_pos, softmax_scale=sm, ldo=ldo)
    tba.sync_status()
    return out


def check(out_bits, o_ref, v_codes_u, v_scale, bits, bos_pos, H, D):
    """Per (query, head): |out - o| <= 2^-8 |o| + 2^-12 max_t |v_hat_t|."""
    M = o_ref.shape[0]
    y = synth.bf16_bits_to_f32(np.ascontiguousarray(out_bits[:, :H * D]).view(np.uint16)).astype(np.float64)
    y = y.reshape(M, H, D)
    off = np.full(v_codes_u.shape[0], float(1 << (bits - 1)))
    if bits == 3 and 0 <= bos_pos < v_codes_u.shape[0]:
        off[bos_pos] = 8.0
    vh = np.abs((v_codes_u.astype(np.float64) - off[:, None, None]) * v_scale.astype(np.float64)[..., None])
    vmax = vh.max(axis=(0, 2))                       # [H]
    err = np.abs(y - o_ref)
    bound = 2.0 ** -8 * np.abs(o_ref) + 2.0 ** -12 * vmax[None, :, None]
    worst = float((err / bound).max())
    assert worst <= 1.0, f"error reaches {worst:.3f} of the bound"
    return worst


def pipeline_case(seed, T, H, D, M, bits, bos_pos, sm=None, q_sigma=1.0):
    """bf16 Q/K/V -> kv_quant3 on the GPU (Q at 4 bits) -> attention_lowbit, against
    oracle.kv_quant -> oracle.attention_lowbit on the same bf16 inputs."""
    k_bf, v_bf = synth.kv_inputs(seed, positions=T, heads=H, head_dim=D)
    q_bf = synth.gaussian_bf16(synth.rng(seed + 77), (M, H, D), sigma=q_sigma)
    sm = float(np.float32(1.0 / math.sqrt(D))) if sm is None else sm
    kc, ks, kb = quant_cache(k_bf, bits, bos_pos)
    vc, vs, vb = quant_cache(v_bf, bits, bos_pos)
    qc, qs, _ = quant_cache(q_bf, 4, -1)
    out = run_attention(qc, qs, kc, ks, kb, vc, vs, vb, M, T, H, D, bits, bos_pos, sm)
    kq, ksr = oracle.kv_quant(k_bf, bits=bits, bos_pos=bos_pos, eps=EPS)
    vq, vsr = oracle.kv_quant(v_bf, bits=bits, bos_pos=bos_pos, eps=EPS)
    qq, qsr = oracle.kv_quant(q_bf, bits=4, bos_pos=-1, eps=EPS)
    o = oracle.attention_lowbit(qq, qsr, kq, ksr, vq, vsr, kv_bits=bits, bos_pos=bos_pos,
                                softmax_scale=np.float32(sm))
    return check(host(out), o, vq, vsr, bits, bos_pos, H, D)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bits,bos_pos", [(3, 0), (3, 5), (3, -1), (4, -1)])
@pytest.mark.parametrize("T,H,M", [(1, 4, 1), (7, 4, 3), (100, 32, 1), (1000, 8, 2), (4133, 32, 3)])
def test_attention_pipeline_parity(D, bits, bos_pos, T, H, M):
    if bos_pos >= T:
        bos_pos = -1
    pipeline_case(11 + T + D, T, H, D, M, bits, bos_pos)


@pytest.mark.parametrize("bits,bos_pos", [(3, 0), (4, -1)])
@pytest.mark.parametrize("M", [1, 5])
def test_attention_700m_heads(bits, bos_pos, M):
    # the 700M shape: 12 heads of 128 (d = 1536), so head groups of 4 heads, three of them
    pipeline_case(53 + M, 2500, 12, 128, M, bits, bos_pos)


@pytest.mark.parametrize("bits", [3, 4])
def test_attention_peaked_scores(bits):
    # large softmax scale: a few positions dominate (scores spread over tens of units)
    pipeline_case(23, 2000, 16, 128, 2, bits, 0 if bits == 3 else -1, sm=2.0, q_sigma=2.0)


def test_attention_many_query_groups():
    # 16 queries of 32 heads: several query groups, each re-reading the cache
    pipeline_case(29, 3000, 32, 128, 16, 3, 0)


@pytest.mark.parametrize("bits", [3, 4])
def test_attention_random_codes_all_values(bits):
    # codes drawn uniformly over every value (extremes included), scales over two decades
    g = synth.rng(31 + bits)
    T, H, D, M, bos_pos = 300, 8, 128, 5, (7 if bits == 3 else -1)
    kq = g.integers(0, 1 << bits, (T, H, D)).astype(np.uint8)
    vq = g.integers(0, 1 << bits, (T, H, D)).astype(np.uint8)
    if bos_pos >= 0:
        kq[bos_pos] = g.integers(0, 16, (H, D))
        vq[bos_pos] = g.integers(0, 16, (H, D))
    qq = g.integers(0, 16, (M, H, D)).astype(np.uint8)
    ksr = g.uniform(0.01, 1.0, (T, H)).astype(np.float32)
    vsr = g.uniform(0.01, 1.0, (T, H)).astype(np.float32)
    qsr = g.uniform(0.01, 1.0, (M, H)).astype(np.float32)

    def pack(c):
        return oracle.pack_kv3(c) if bits == 3 else oracle.pack_nibbles(c)

    kp = pack(kq)
    vp = pack(vq)
    kb = vb = None
    if bos_pos >= 0:
        kp[bos_pos] = 0
        vp[bos_pos] = 0
        kb = to_dev(oracle.pack_nibbles(kq[bos_pos]))
        vb = to_dev(oracle.pack_nibbles(vq[bos_pos]))
    sm = 0.125
    out = run_attention(to_dev(oracle.pack_nibbles(qq)), to_dev(qsr), to_dev(kp), to_dev(ksr), kb, to_dev(vp),
                        to_dev(vsr), vb, M, T, H, D, bits, bos_pos, sm)
    o = oracle.attention_lowbit(qq, qsr, kq, ksr, vq, vsr, kv_bits=bits, bos_pos=bos_pos,
                                softmax_scale=np.float32(sm))
    check(host(out), o, vq, vsr, bits, bos_pos, H, D)


def test_attention_zero_query_is_the_mean():
    # all query codes 8 (q_hat = 0): every score is 0, so each output is the mean of
    # the values the query sees -- a closed form independent of the softmax
    g = synth.rng(37)
    T, H, D, M = 513, 4, 128, 2
    vq = g.integers(0, 8, (T, H, D)).astype(np.uint8)
    vsr = g.uniform(0.1, 1.0, (T, H)).astype(np.float32)
    kq = g.integers(0, 8, (T, H, D)).astype(np.uint8)
    ksr = np.ones((T, H), np.float32)
    qq = np.full((M, H, D), 8, np.uint8)
    out = run_attention(to_dev(oracle.pack_nibbles(qq)), to_dev(np.ones((M, H), np.float32)),
                        to_dev(oracle.pack_kv3(kq)), to_dev(ksr), None, to_dev(oracle.pack_kv3(vq)), to_dev(vsr),
                        None, M, T, H, D, 3, -1, 0.1)
    vh = (vq.astype(np.float64) - 4.0) * vsr.astype(np.float64)[..., None]
    o = np.stack([vh[:T - M + m + 1].mean(axis=0) for m in range(M)])
    check(host(out), o, vq, vsr, 3, -1, H, D)


def test_attention_full_decode_7b():
    # the 7B decode context: one query over a 32768-position cache of 32 heads of 128
    worst = pipeline_case(41, 32768, 32, 128, 1, 3, 0)
    assert worst <= 1.0


def test_attention_output_stride_untouched():
    # a row stride wider than H*D: the padding columns and the buffer margins keep their canary bytes
    T, H, D, M = 200, 4, 64, 3
    k_bf, v_bf = synth.kv_inputs(43, positions=T, heads=H, head_dim=D)
    q_bf = synth.gaussian_bf16(synth.rng(44), (M, H, D))
    kc, ks, kb = quant_cache(k_bf, 3, 0)
    vc, vs, vb = quant_cache(v_bf, 3, 0)
    qc, qs, _ = quant_cache(q_bf, 4, -1)
    ldo = H * D + 24
    out, buf = canaried((M, ldo), torch.int16)
    ws = empty((tba.workspace_size("attention_lowbit", M, H, D) // 4,), torch.float32)
    tba.attention_lowbit(qc, qs, M, kc, ks, vc, vs, T, H, D, out, ws, k_bos=kb, v_bos=vb, kv_bits=3, bos_pos=0,
                         softmax_scale=0.125, ldo=ldo)
    tba.sync_status()
    b = host(buf)
    pad = (b.size - M * ldo * 2) // 2
    assert (b[:pad] == CANARY).all() and (b[-pad:] == CANARY).all()
    rows = b[pad:pad + M * ldo * 2].reshape(M, ldo * 2)
    assert (rows[:, H * D * 2:] == CANARY).all()
    assert not (rows[:, :H * D * 2] == CANARY).all()
