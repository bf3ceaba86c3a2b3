"""bitlinear_forward_noalloc: the tensor-core forward for callers that cannot
allocate device memory (a plugin handed only its input and output pointers,
a serving loop that forbids allocation after start-up). Its scratch is a
fixed 16 MiB array inside the library instead of a caller workspace.

Checked through the C ABI against the existing entry point
(bitlinear_forward_ex on the tensor-core path with a caller workspace), with
the tolerance of the other parity tests, on two calls in a row: the second
call reuses the array the first one left behind. This file is collected
last so that a run stopping at the first failure has already run every
other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

import oracle
import ternary_weight_w1_b200 as bl
from tests.gpu_cases import Case, check_y, tensor_to_bf16_bits

pytestmark = pytest.mark.gpu


def call_noalloc(x, packed, gamma, N, y):
    import torch
    M, K = x.shape
    return bl.lib().bitlinear_forward_noalloc(
        x.data_ptr(), bl.BITLINEAR_BF16, M, K, packed.data_ptr(), ctypes.c_float(gamma), N,
        y.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_path_twice():
    import torch
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    # two different problems, back to back, sharing the static scratch
    cases = [Case(300, 1280, 700, w_seed=21, x_seed=22), Case(130, 2560, 513, w_seed=23, x_seed=24)]
    for c in cases:
        x, packed = c.x_tensor(), c.packed_tensor()
        y_ref = torch.empty((c.M, c.N), dtype=torch.bfloat16, device="cuda")
        bl.bitlinear_forward(x, packed, c.gamma, c.N, y=y_ref, path=bl.PATH_TC)
        y = torch.full((c.M, c.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert call_noalloc(x, packed, c.gamma, c.N, y) == bl.BITLINEAR_OK
        torch.cuda.synchronize()
        got, ref = tensor_to_bf16_bits(y), tensor_to_bf16_bits(y_ref)
        check_y(got, ref)                        # the parity tolerance (rel 1e-2)
        np.testing.assert_array_equal(got, ref)  # same kernels: identical bits
        assert check_y(got, c.oracle_full()[1]) == 1.0   # and the oracle's bits
    assert bl.bitlinear_get_fault() == (bl.BITLINEAR_OK, 0)


def test_noalloc_fills_the_scratch_exactly_and_rejects_beyond_it():
    """M = 2424 tokens of K = 6912 fill the 16 MiB array to its last bytes
    (x~, beta and the row sums of x~); on seeded nonzero data the result must
    equal the workspace path's and the oracle's bit for bit. One more token
    is refused before any device work."""
    import torch
    c = Case(2424, 6912, 80, w_seed=25, x_seed=26)
    x, packed = c.x_tensor(), c.packed_tensor()
    y_ref = torch.empty((c.M, c.N), dtype=torch.bfloat16, device="cuda")
    bl.bitlinear_forward(x, packed, c.gamma, c.N, y=y_ref, path=bl.PATH_TC)
    y = torch.full((c.M, c.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert call_noalloc(x, packed, c.gamma, c.N, y) == bl.BITLINEAR_OK
    torch.cuda.synchronize()
    got, ref = tensor_to_bf16_bits(y), tensor_to_bf16_bits(y_ref)
    check_y(got, ref)
    np.testing.assert_array_equal(got, ref)
    # the oracle's bits for the whole problem (integer products on all host cores)
    assert check_y(got, c.oracle_full(oracle.Oracle(oracle.load_omp()))[1]) == 1.0
    assert bl.bitlinear_get_fault() == (bl.BITLINEAR_OK, 0)

    x1 = torch.zeros((2425, 6912), dtype=torch.bfloat16, device="cuda")
    y1 = torch.empty((2425, 80), dtype=torch.bfloat16, device="cuda")
    assert call_noalloc(x1, packed, c.gamma, 80, y1) == bl.BITLINEAR_ERR_SCRATCH_LIMIT
