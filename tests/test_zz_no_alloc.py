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


def _with_workspace(wd, wfmt):
    N, K = wd.shape
    out = torch.empty((N, K // 4 if wfmt == tba.BL_W_T2 else K), dtype=torch.uint8, device=wd.device)
    alpha = torch.empty((1,), dtype=torch.float32, device=wd.device)
    ws = torch.empty((tba.workspace_size("pack_ternary") // 8,), dtype=torch.int64, device=wd.device)
    tba.pack_ternary(wd, alpha, out, wfmt=wfmt, workspace=ws)
    tba.sync_status()
    return out.cpu().numpy(), alpha.cpu().numpy()


def _no_alloc(wd, wfmt):
    N, K = wd.shape
    out = torch.empty((N, K // 4 if wfmt == tba.BL_W_T2 else K), dtype=torch.uint8, device=wd.device)
    alpha = torch.empty((1,), dtype=torch.float32, device=wd.device)
    tba.pack_ternary_noalloc(wd, alpha, out, wfmt=wfmt)
    tba.sync_status()
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
