"""pack_ternary_noalloc, the allocation-free variant of pack_ternary.

Some callers cannot allocate device memory while they run: an inference engine
that owns every byte of device memory and forbids allocation inside its execute
step, or a C host with no device allocator of its own.  For them the library
keeps pack_ternary's scratch (the exponent bins of the exact mean |W|) in a
2 KiB array of its own, so the call needs no workspace argument.  This test
checks, through the C ABI, that the variant gives exactly what pack_ternary
gives -- alpha and every packed byte -- on two calls in a row, so a second call
cannot see the first call's scratch.  It is collected last and also passes alone
in a fresh process (the first call on the device does the one-time address
lookup)."""
import numpy as np
import pytest
import torch

import synth
import ternary_bit_activation_b200 as tba

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda:0")


def _width(wfmt):
    return {tba.BL_W_T2: 4, tba.BL_W_E2M1: 2}.get(wfmt, 1)


def _with_workspace(wd, wfmt):
    N, K = wd.shape
    out = torch.empty((N, K // _width(wfmt)), dtype=torch.uint8, device=wd.device)
    alpha = torch.empty((1,), dtype=torch.float32, device=wd.device)
    ws = torch.empty((tba.workspace_size("pack_ternary") // 8,), dtype=torch.int64, device=wd.device)
    tba.pack_ternary(wd, alpha, out, wfmt=wfmt, workspace=ws)
    tba.sync_status()
    return out.cpu().numpy(), alpha.cpu().numpy()


def _no_alloc(wd, wfmt, alpha_in=None):
    """Outputs are allocated first; the call itself must leave torch's caching
    allocator exactly as it found it."""
    N, K = wd.shape
    out = torch.empty((N, K // _width(wfmt)), dtype=torch.uint8, device=wd.device)
    alpha = torch.empty((1,), dtype=torch.float32, device=wd.device)
    if alpha_in is not None:
        alpha.fill_(float(alpha_in))
    torch.cuda.synchronize()
    before = (torch.cuda.memory_allocated(), torch.cuda.memory_reserved())
    tba.pack_ternary_noalloc(wd, alpha, out, wfmt=wfmt, alpha_given=alpha_in is not None)
    tba.sync_status()
    assert (torch.cuda.memory_allocated(), torch.cuda.memory_reserved()) == before
    return out.cpu().numpy(), alpha.cpu().numpy()


def test_no_alloc_matches_workspace_variant_on_two_calls():
    assert torch.cuda.is_available()
    cases = [(synth.latent_weights_f32(synth.rng(41), 4608, 1536), tba.BL_W_T2),
             (synth.latent_weights_f32(synth.rng(42), 300, 3200) * np.float32(3.0), tba.BL_W_I8)]
    for w, wfmt in cases:                    # two calls in a row, different tensors
        wd = _dev(w)
        ref_codes, ref_alpha = _with_workspace(wd, wfmt)
        codes, alpha = _no_alloc(wd, wfmt)
        assert alpha.view(np.uint32)[0] == ref_alpha.view(np.uint32)[0]
        assert np.array_equal(codes, ref_codes)
    # the same tensor twice: the scratch is cleared at the start of each call
    wd = _dev(cases[0][0])
    first = _no_alloc(wd, tba.BL_W_I8)
    second = _no_alloc(wd, tba.BL_W_I8)
    assert first[1].view(np.uint32)[0] == second[1].view(np.uint32)[0]
    assert np.array_equal(first[0], second[0])


def test_no_alloc_e2m1_and_given_alpha_on_two_calls():
    """The E2M1 weight layout (the FP4 tensor-core operand), and alpha_given,
    which skips the static scratch altogether: both match pack_ternary."""
    w = synth.latent_weights_f32(synth.rng(43), 1000, 4096)
    wd = _dev(w)
    ref_codes, ref_alpha = _with_workspace(wd, tba.BL_W_E2M1)
    for _ in range(2):
        codes, alpha = _no_alloc(wd, tba.BL_W_E2M1)
        assert alpha.view(np.uint32)[0] == ref_alpha.view(np.uint32)[0]
        assert np.array_equal(codes, ref_codes)
    # a caller-given alpha: the codes follow it, the alpha is left as given
    given = np.float32(ref_alpha[0] * np.float32(1.5))
    ws_out = torch.empty((1000, 4096 // 4), dtype=torch.uint8, device="cuda:0")
    al = torch.full((1,), float(given), dtype=torch.float32, device="cuda:0")
    tba.pack_ternary(wd, al, ws_out, wfmt=tba.BL_W_T2, alpha_given=True)
    tba.sync_status()
    for _ in range(2):
        codes, alpha = _no_alloc(wd, tba.BL_W_T2, alpha_in=given)
        assert alpha.view(np.uint32)[0] == np.array([given], np.float32).view(np.uint32)[0]
        assert np.array_equal(codes, ws_out.cpu().numpy())
