"""The forward call's host-side contract (include/bitlinear.h) as a model, checked
against the library on random argument combinations.

Only combinations the model says are refused before any device work (or are
empty batches, which do nothing) are passed to the library; the placeholder
pointers are never handed to a kernel."""
import ctypes

import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

import ternary_weight_w1_b200 as bl

FAKE = 1 << 20                  # 16-byte aligned, never dereferenced
INT_MAX = 2 ** 31 - 1
REACHES_DEVICE = "device"


def gemv_fits(M, K):
    return M <= 16 and M * K <= 196608


def model(M, K, N, xdt, path, x, packed, y, acc, xq, beta):
    """Status the forward returns before touching the device, or
    REACHES_DEVICE. Checks in the order the header lists them."""
    if M < 0 or N < 1 or K < 1:
        return bl.BITLINEAR_ERR_ARG
    if M > 0 and (x is None or packed is None or y is None):
        return bl.BITLINEAR_ERR_ARG
    if xdt not in (bl.BITLINEAR_BF16, bl.BITLINEAR_FP32):
        return bl.BITLINEAR_ERR_DTYPE
    if (K % 128 or K > 65536 or N > INT_MAX // 2 or M > INT_MAX // 2 or M * K > 2 ** 40):
        return bl.BITLINEAR_ERR_SHAPE

    def misaligned(p, a):
        return p is not None and p % a != 0
    if (misaligned(x, 16) or misaligned(packed, 16) or misaligned(y, 16) or misaligned(xq, 16)
            or misaligned(acc, 4) or misaligned(beta, 4)):
        return bl.BITLINEAR_ERR_ALIGN
    if path not in (bl.PATH_AUTO, bl.PATH_GEMV, bl.PATH_TC):
        return bl.BITLINEAR_ERR_ARG
    if M == 0:
        return bl.BITLINEAR_OK
    if path == bl.PATH_GEMV and not gemv_fits(M, K):
        return bl.BITLINEAR_ERR_SHAPE
    return REACHES_DEVICE


ptr16 = st.sampled_from([None, FAKE, FAKE + 8, FAKE + 1])
ptr4 = st.sampled_from([None, FAKE, FAKE + 2, FAKE + 4])


@settings(max_examples=600, deadline=None)
@given(M=st.sampled_from([-1, 0, 1, 3, 6, 7, 12, 16, 17, 4096, INT_MAX // 2 + 1]),
       K=st.sampled_from([-128, 0, 64, 128, 200, 256, 12288, 16384, 65536, 65664, 1 << 20]),
       N=st.sampled_from([-1, 0, 1, 64, 6912, INT_MAX // 2, INT_MAX // 2 + 1]),
       xdt=st.sampled_from([-1, 0, 1, 2]),
       path=st.sampled_from([-1, 0, 1, 2, 3]),
       x=ptr16, packed=ptr16, y=ptr16, xq=ptr16, acc=ptr4, beta=ptr4)
def test_forward_host_contract(M, K, N, xdt, path, x, packed, y, xq, acc, beta):
    expected = model(M, K, N, xdt, path, x, packed, y, acc, xq, beta)
    if expected == REACHES_DEVICE:
        return                  # a valid call: it would launch, so it is not made here
    rc = bl.lib().bitlinear_forward_ex(x, xdt, M, K, packed, 1.0, N, y, None, 0, None, acc,
                                       xq, beta, path)
    assert rc == expected, (rc, expected)


@pytest.mark.parametrize("M,K,N,path", [(1, 256, 64, 1), (16, 12160, 64, 1), (6, 32768, 64, 0),
                                        (7, 256, 64, 0), (2048, 6912, 2560, 2)])
def test_model_marks_valid_calls(M, K, N, path):
    # a check of the model itself: these valid calls reach the device
    assert model(M, K, N, 0, path, FAKE, FAKE, FAKE, None, None, None) == REACHES_DEVICE
    size_max = ctypes.c_size_t(-1).value
    assert bl.bitlinear_workspace_bytes(M, N, K, path) != size_max
