"""The canary helpers that the GPU out-of-bounds tests rely on, checked on the
CPU: the tensor lies exactly between the margins, it starts as canary bytes,
writes inside it leave the margins intact, and a write one byte outside either
end is detected."""
import numpy as np
import torch

from gpu_util import CANARY, CANARY_PAD, canaried, canary_bytes, canary_margins_intact

CPU = torch.device("cpu")


def test_tensor_sits_between_the_margins():
    for shape, dtype in [((37, 328), torch.int8), ((37,), torch.float32), ((37, 11), torch.int32),
                         ((3, 5, 24), torch.uint8), ((200, 304), torch.int16)]:
        t, buf = canaried(shape, dtype, CPU)
        assert tuple(t.shape) == shape and t.dtype == dtype
        nbytes = t.numel() * t.element_size()
        assert buf.numel() == 2 * CANARY_PAD + nbytes
        assert t.data_ptr() == buf.data_ptr() + CANARY_PAD and t.data_ptr() % 16 == 0
        assert np.all(canary_bytes(t) == CANARY)
        t.zero_()
        assert canary_margins_intact(t, buf)
        assert np.all(buf.numpy()[CANARY_PAD:CANARY_PAD + nbytes] == 0)


def test_writes_just_outside_are_detected():
    for off in (CANARY_PAD - 1, None):
        t, buf = canaried((37, 11), torch.int32, CPU)
        nbytes = t.numel() * t.element_size()
        buf[CANARY_PAD + nbytes if off is None else off] = 0
        assert not canary_margins_intact(t, buf)


def test_canary_bytes_rows():
    t, _ = canaried((4, 6), torch.int16, CPU)
    t[2, 5] = 0
    b = canary_bytes(t)
    assert b.shape == (4, 12)
    assert np.all(b[2, 10:] == 0) and np.all(b[:2] == CANARY) and np.all(b[3] == CANARY)
