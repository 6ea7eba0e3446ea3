"""Failure handling on the GPU without a fault: a bounded wait that runs out
records BL_ERR_TIMEOUT in the device status word, the host reads and clears it,
and the same context then still computes the path correctly."""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_bit_activation_b200 as tba
from gpu_util import empty, host, to_dev

pytestmark = pytest.mark.gpu

EPS = 1e-5


def test_bounded_wait_timeout_is_reported_and_context_survives():
    tba.sync_status()
    t0 = time.monotonic()
    tba.selftest_timeout()
    with pytest.raises(tba.BitLinearError) as err:
        tba.sync_status()
    assert tba.STATUS_NAMES[err.value.status] == "BL_ERR_TIMEOUT"
    assert time.monotonic() - t0 >= 1.5          # the wait ran to its 2 s limit
    tba.sync_status()                            # read once, then cleared

    x = synth.gaussian_bf16(synth.rng(77), (5, 256))
    codes = empty((5, 256), torch.int8)
    scale = empty((5,), torch.float32)
    tba.bitlinear_quant_a4(to_dev(x), codes, scale, tba.BL_QUANT_INT4, tba.BL_STORE_BYTES, EPS)
    tba.sync_status()
    c_ref, _, s_ref = oracle.quant_int4(x, EPS)
    assert np.array_equal(host(codes), c_ref)
    assert np.array_equal(host(scale).view(np.uint32), s_ref.view(np.uint32))
