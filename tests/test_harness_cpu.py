"""The GPU parity harness's canary-guarded outputs, checked on CPU tensors:
the view the library receives has the right shape, dtype, contiguity and
alignment, writes inside it pass, and a write one element past either end is
caught."""
import numpy as np
import pytest
import torch

from tests.gpu_cases import (CANARY_ACC, CANARY_BETA, CANARY_XQ, CANARY_Y, Guarded,
                             guarded_outputs, read_guarded)


@pytest.mark.parametrize("shape,dtype,canary", [((3, 130), torch.bfloat16, CANARY_Y),
                                                ((3, 130), torch.int32, CANARY_ACC),
                                                ((5, 256), torch.int8, CANARY_XQ),
                                                ((7,), torch.float32, CANARY_BETA),
                                                ((0, 64), torch.bfloat16, CANARY_Y)])
def test_guarded_view_and_canaries(shape, dtype, canary):
    g = Guarded(shape, dtype, "cpu", canary)
    t = g.t
    assert tuple(t.shape) == shape and t.dtype == dtype and t.is_contiguous()
    if t.numel():                                   # an empty tensor reports address 0
        assert t.data_ptr() % 16 == 0
        assert t.data_ptr() - g.raw.data_ptr() == Guarded.PAD_BYTES
    g.check()
    if t.numel():
        t.view(-1)[0] = 1
        t.view(-1)[-1] = 2
        g.check()                                   # writes inside the output pass
    for idx in (g.pad - 1, g.pad + g.n):            # one element before / past the end
        h = Guarded(shape, dtype, "cpu", canary)
        h.raw[idx] = 0
        with pytest.raises(AssertionError):
            h.check()


def test_canaries_are_not_results():
    # no correct output holds its canary: y and beta are NaN patterns, acc is
    # beyond 127 * 65536, x~ never reaches -128
    y = Guarded((1, 1), torch.bfloat16, "cpu", CANARY_Y).t
    beta = Guarded((1,), torch.float32, "cpu", CANARY_BETA).t
    assert torch.isnan(y.float()).all() and torch.isnan(beta).all()
    assert CANARY_ACC > 127 * 65536 and CANARY_XQ < -127


def test_read_guarded_returns_every_output():
    g = guarded_outputs(2, 48, 128, "cpu")
    g["y"].t.fill_(1.5)
    g["acc"].t.fill_(3)
    g["xq"].t.fill_(-4)
    g["beta"].t.fill_(0.25)
    out = read_guarded(g)
    assert out["y"].dtype == np.uint16 and np.all(out["y"] == 0x3FC0)     # bf16 1.5
    assert np.all(out["acc"] == 3) and np.all(out["xq"] == -4) and np.all(out["beta"] == 0.25)
    g["acc"].raw[-1] = 0
    with pytest.raises(AssertionError):
        read_guarded(g)
