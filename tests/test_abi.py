"""The C ABI library: loads, exports every symbol the public header declares,
and validates arguments on the host (these calls return before any CUDA work,
so they need no GPU)."""
import ctypes
import os
import re

import pytest

import ternary_bit_activation_b200 as tba
from ternary_bit_activation_b200 import build as tba_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    tba_build.build()
    return tba.lib()


def declared_symbols():
    hdr = open(os.path.join(ROOT, "include", "bitlinear.h")).read()
    return re.findall(r"BL_API\s+[\w\s\*]+?\b(\w+)\s*\(", hdr)


def test_header_declares_the_boundary():
    names = declared_symbols()
    for required in ("bitlinear_quant_a4", "bitlinear_sparsify_a8", "pack_ternary", "bitlinear_gemm",
                     "relu2_glu", "kv_quant3"):
        assert required in names
    assert sorted(names) == sorted(tba.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
    assert "sm_100a" in tba.version()


def test_status_strings(L):
    for code, name in enumerate(tba.STATUS_NAMES):
        assert tba.status_string(code) == name


def test_workspace_size(L):
    assert tba.workspace_size("pack_ternary", 0, 4096, 4096) == 2048
    assert tba.workspace_size("bitlinear_gemm", 128, 128, 128) == 0
    # quant_gemm run as two kernels: M x K int8 codes, then M fp32 scales, each 16-byte aligned
    assert tba.workspace_size("quant_gemm", 3, 64, 64) == 192 + 16
    assert tba.workspace_size("quant_gemm", 32768, 4096, 4096) == 32768 * 4096 + 4 * 32768


def test_quant_gemm_validation(L):
    g = L.bitlinear_quant_gemm
    ok = dict(x=A16, ldx=256, q=0, eps=1e-5, w=A16, wfmt=0, al=A16, grp=256, M=16, N=256, K=256, y=A16, ldy=256,
              acc=None, ws=A16, wsb=1 << 20)

    def call(**kw):
        d = dict(ok, **kw)
        return g(P(d["x"]), d["ldx"], d["q"], d["eps"], P(d["w"]), d["wfmt"], P(d["al"]), d["grp"], d["M"], d["N"],
                 d["K"], P(d["y"]), d["ldy"], P(d["acc"]), P(d["ws"]), d["wsb"], None)

    assert call(q=2) == 4
    assert call(wfmt=2) == 4           # E2M1 weights: use the separate calls
    assert call(eps=-1.0) == 4
    assert call(K=100) == 3
    assert call(K=16448) == 3          # the quantizer's row limit
    assert call(ldx=200) == 3          # ldx < K
    assert call(ldx=260) == 3          # ldx % 8
    assert call(M=0) == 0
    assert call(x=None) == 1
    assert call(y=None, acc=None) == 1
    assert call(x=MIS) == 2
    # 16 tokens run as quantizer + GEMM: the workspace is checked before any launch
    assert call(ws=None) == 1
    assert call(ws=MIS) == 2
    assert call(wsb=16 * 256) == 8


# fake device addresses: validation rejects before anything dereferences them
A16 = 0x10000
MIS = 0x10001
P = ctypes.c_void_p


def test_gemm_validation(L):
    g = L.bitlinear_gemm
    ok = dict(a=A16, afmt=0, s=A16, w=A16, wfmt=1, al=A16, grp=256, M=128, N=256, K=256, y=A16, ldy=256, acc=None)

    def call(**kw):
        d = dict(ok, **kw)
        return g(P(d["a"]), d["afmt"], P(d["s"]), P(d["w"]), d["wfmt"], P(d["al"]), d["grp"], d["M"], d["N"],
                 d["K"], P(d["y"]), d["ldy"], P(d["acc"]), None)

    assert call(K=100) == 3            # K % 64
    assert call(K=0) == 3
    assert call(N=0) == 3
    assert call(ldy=100) == 3          # ldy < N
    assert call(ldy=260) == 3          # ldy % 8
    assert call(afmt=7) == 4
    assert call(wfmt=9) == 4
    assert call(grp=0) == 4
    assert call(M=0) == 0              # empty: no-op
    assert call(a=None) == 1
    assert call(y=None, acc=None) == 1
    assert call(a=MIS) == 2
    assert call(w=MIS) == 2


def test_quant_validation(L):
    q = L.bitlinear_quant_a4
    assert q(P(A16), 4, 100, 100, 0, 0, 1e-5, P(A16), P(A16), None) == 3    # K % 8
    assert q(P(A16), 4, 64, 60, 0, 0, 1e-5, P(A16), P(A16), None) == 3      # ldx < K
    assert q(P(A16), 4, 32768, 32768, 0, 0, 1e-5, P(A16), P(A16), None) == 3  # K too large
    assert q(P(A16), 4, 64, 64, 5, 0, 1e-5, P(A16), P(A16), None) == 4
    assert q(P(A16), 4, 64, 64, 0, 3, 1e-5, P(A16), P(A16), None) == 4
    assert q(P(A16), 4, 64, 64, 0, 0, -1.0, P(A16), P(A16), None) == 4
    assert q(None, 4, 64, 64, 0, 0, 1e-5, P(A16), P(A16), None) == 1
    assert q(P(MIS), 4, 64, 64, 0, 0, 1e-5, P(A16), P(A16), None) == 2
    assert q(P(A16), 0, 64, 64, 0, 0, 1e-5, P(A16), P(A16), None) == 0


def test_rmsnorm_quant_and_per_tensor_validation(L):
    r = L.bitlinear_rmsnorm_quant_a4
    ok = dict(x=A16, M=4, K=64, ldx=64, g=None, en=1e-6, q=0, st=0, eps=1e-5, c=A16, s=A16)

    def call(**kw):
        d = dict(ok, **kw)
        return r(P(d["x"]), d["M"], d["K"], d["ldx"], P(d["g"]), d["en"], d["q"], d["st"], d["eps"], P(d["c"]),
                 P(d["s"]), None)

    assert call(en=0.0) == 4                 # eps_norm must be positive
    assert call(en=float("inf")) == 4
    assert call(K=100) == 3
    assert call(K=16392, ldx=16392) == 3
    assert call(q=9) == 4
    assert call(g=MIS) == 2                  # the weight is read 16 bytes at a time
    assert call(x=None) == 1
    assert call(M=0) == 0
    pt = L.bitlinear_quant_a4_per_tensor
    okp = dict(x=A16, M=4, K=64, ldx=64, st=0, eps=1e-5, c=A16, s=A16, b=A16, ws=A16, wsb=2048)

    def callp(**kw):
        d = dict(okp, **kw)
        return pt(P(d["x"]), d["M"], d["K"], d["ldx"], d["st"], d["eps"], P(d["c"]), P(d["s"]), P(d["b"]),
                  P(d["ws"]), d["wsb"], None)

    assert callp(wsb=1024) == 8
    assert callp(ws=None) == 1
    assert callp(b=None) == 1
    assert callp(M=1 << 20, K=4096, ldx=4096) == 3      # M * K >= 2^31
    assert callp(M=1 << 62, K=64) == 3                  # no overflowing product
    assert callp(st=7) == 4
    assert callp(M=0) == 0
    assert tba.workspace_size("quant_a4_per_tensor") == 2048


def test_topk_validation(L):
    s = L.bitlinear_sparsify_a8
    assert s(P(A16), 4, 64, 64, 0, 1e-5, P(A16), P(A16), None, None) == 4      # k_keep < 1
    assert s(P(A16), 4, 64, 64, 65, 1e-5, P(A16), P(A16), None, None) == 4     # k_keep > K
    assert s(P(A16), 4, 20000, 20000, 5, 1e-5, P(A16), P(A16), None, None) == 3
    assert s(P(A16), 4, 64, 64, 5, 1e-5, P(A16), P(A16), P(MIS), None) == 2
    r = L.relu2_glu
    assert r(P(A16), P(A16), 4, 64, 32, 5, 1e-5, P(A16), P(A16), None, None) == 3   # ld < F
    assert r(P(A16), None, 4, 64, 64, 5, 1e-5, P(A16), P(A16), None, None) == 1


def test_pack_and_kv_validation(L):
    pk = L.pack_ternary
    assert pk(P(A16), 8, 24, 24, 1e-5, 0, P(A16), 0, P(A16), P(A16), 2048, None) == 3   # K % 16
    assert pk(P(A16), 8, 64, 64, 1e-5, 0, P(A16), 0, P(A16), P(A16), 1024, None) == 8   # workspace too small
    assert pk(P(A16), 8, 64, 64, 1e-5, 0, P(A16), 0, P(A16), None, 0, None) == 1
    assert pk(P(A16), 8, 64, 64, 1e-5, 0, P(A16), 5, P(A16), P(A16), 2048, None) == 4
    pn = L.pack_ternary_noalloc
    assert pn(P(A16), 1 << 16, 1 << 15, 1 << 15, 1e-5, 0, P(A16), 0, P(A16), None) == 3   # N*K >= 2^31
    # a product N*K that wraps in 64 bits (2^62 * 64 = 2^68) must not slip past the limit
    assert pn(P(A16), 1 << 62, 64, 64, 1e-5, 0, P(A16), 0, P(A16), None) == 3
    assert pk(P(A16), 1 << 62, 64, 64, 1e-5, 0, P(A16), 0, P(A16), P(A16), 2048, None) == 3
    # the largest accepted N for K = 16 is 2^27 - 1; 2^27 reaches 2^31 elements
    assert pn(P(A16), 1 << 27, 16, 16, 1e-5, 0, P(A16), 0, P(A16), None) == 3
    assert pk(P(A16), 1 << 27, 16, 16, 1e-5, 0, P(A16), 0, P(A16), P(A16), 2048, None) == 3
    assert pn(P(A16), 8, 24, 24, 1e-5, 0, P(A16), 0, P(A16), None) == 3                   # K % 16
    assert pn(P(A16), 8, 64, 64, 1e-5, 0, None, 0, P(A16), None) == 1
    kv = L.kv_quant3
    assert kv(P(A16), 8, 4, 100, 400, 3, 0, 1e-5, P(A16), P(A16), P(A16), None) == 3     # D % 32
    assert kv(P(A16), 8, 4, 96, 384, 3, 0, 1e-5, P(A16), P(A16), P(A16), None) == 3      # D not a power of two
    assert kv(P(A16), 8, 4, 128, 512, 5, 0, 1e-5, P(A16), P(A16), P(A16), None) == 4     # bits
    assert kv(P(A16), 8, 4, 128, 512, 3, 0, 1e-5, P(A16), P(A16), None, None) == 1       # BOS buffer needed


def test_attention_validation(L):
    at = L.attention_lowbit
    ws = tba.workspace_size("attention_lowbit", 1, 32, 128)
    assert ws == 512 * 32 * 132 * 4
    ok = dict(q=A16, qs=A16, M=1, k=A16, ks=A16, kb=A16, v=A16, vs=A16, vb=A16, T=100, H=32, D=128, bits=3, bos=0,
              sm=0.088, out=A16, ldo=4096, ws=A16, wsb=ws)

    def call(**kw):
        d = dict(ok, **kw)
        return at(P(d["q"]), P(d["qs"]), d["M"], P(d["k"]), P(d["ks"]), P(d["kb"]), P(d["v"]), P(d["vs"]),
                  P(d["vb"]), d["T"], d["H"], d["D"], d["bits"], d["bos"], d["sm"], P(d["out"]), d["ldo"],
                  P(d["ws"]), d["wsb"], None)

    assert call(bits=2) == 4
    assert call(bos=-2) == 4
    assert call(sm=float("nan")) == 4
    assert call(D=32) == 3 and call(D=256) == 3
    assert call(H=128, ldo=128 * 128) == 3          # H * D / 32 > 256
    assert call(M=101) == 3                         # more queries than positions
    assert call(ldo=4095) == 3
    assert call(T=1 << 30) == 3
    assert call(M=0) == 0
    assert call(kb=None) == 1                       # a 3-bit cache with a BOS position needs its 4-bit row
    # ... a 4-bit cache does not, nor one without a BOS position: the call gets past the
    # null checks to the workspace check
    assert call(kb=None, vb=None, bits=4, wsb=ws - 1) == 8
    assert call(kb=None, vb=None, bos=-1, wsb=ws - 1) == 8
    assert call(k=MIS) == 2
    assert call(ws=MIS) == 2
    assert call(wsb=ws - 1) == 8
    assert call(ws=None) == 1


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(tba, "_lib", None)
    monkeypatch.setattr(tba, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError):
        tba.lib()
