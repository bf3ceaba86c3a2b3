"""Parity of bitlinear_forward_rmsnorm with the oracle: the tokens are
RMS-normalised (the nn.RMSNorm member of the BitLinear listing in "BitNet
b1.58 2B4T Guide: Scaling Native 1-Bit LLMs") inside the quantisation pass of
either path, then contracted and rescaled as in bitlinear_forward.

Comparison. The device adds the squares of a token in another order than the
oracle (both in double). Its fp32 mean can then differ in the last bit when
the two double sums straddle an fp32 rounding boundary, which moves every
normalised value by at most an ulp. So:
  * beta is compared within 2 ulps and x~ exactly, except that an element
    whose oracle value n * 127 / beta lies within TIE_BAND of a half-integer
    may take either neighbour;
  * acc and y are compared exactly against the oracle applied to the kernel's
    own x~ and beta (the integer product and the rescale have one answer).
In practice every element matches: the double sums differ by far less than an
fp32 rounding step, so the two means round alike except in about one row in
10^8.
"""
import numpy as np
import pytest

import workloads
import ternary_weight_w1_b200 as bl
from tests.gpu_cases import NormCase

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bl.lib()
    return torch


# -------------------------------------------------------------- GEMV path

@pytest.mark.parametrize("M", [1, 3, 6, 16])
@pytest.mark.parametrize("K,N", [(256, 200), (2560, 640), (6912, 37)])
def test_gemv_rmsnorm_parity(cuda, M, K, N):
    c = NormCase(M, K, N, g_seed=K + M, w_seed=K + N + 1, x_seed=M + 11 * K)
    c.check_norm_full(c.run(path=bl.PATH_GEMV))


def test_gemv_rmsnorm_long_rows(cuda):
    # 65536 channels: past the prologue's register cache, so the re-read
    # passes normalise as well
    c = NormCase(2, 65536, 48, g_seed=3, w_seed=4, x_seed=5)
    c.check_norm_full(c.run(path=bl.PATH_GEMV))


def test_gemv_rmsnorm_fp32_input(cuda):
    c = NormCase(4, 256, 256, w_seed=0, x_seed=0, x_dtype="fp32", outliers=False)
    c.check_norm_full(c.run(path=bl.PATH_GEMV))


# ------------------------------------------------------ tensor-core path

@pytest.mark.parametrize("M,K,N", [(7, 256, 136), (64, 2560, 640), (200, 6912, 300),
                                   (33, 1280, 2000)])
def test_tc_rmsnorm_parity(cuda, M, K, N):
    c = NormCase(M, K, N, g_seed=M + K, w_seed=N + 3, x_seed=M * 5 + K)
    c.check_norm_full(c.run(path=bl.PATH_TC))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_tc_rmsnorm_long_rows(cuda, dtype):
    # eight warps per row and rows past the register cache
    c = NormCase(3, 65536, 40, g_seed=8, w_seed=9, x_seed=10, x_dtype=dtype)
    c.check_norm_full(c.run(path=bl.PATH_TC))


@pytest.mark.parametrize("M,K,dtype", [(1030, 2560, "bf16"), (1027, 1280, "fp32")])
def test_tc_rmsnorm_staged_rows(cuda, M, K, dtype):
    # from 1024 tokens the quantiser stages whole rows in shared memory (eight
    # per block, a ragged last block)
    c = NormCase(M, K, 48, g_seed=M, w_seed=K + 1, x_seed=M + K, x_dtype=dtype)
    c.check_norm_full(c.run(path=bl.PATH_TC))


# ------------------------------------------------------------- edge cases

@pytest.mark.parametrize("path", [bl.PATH_GEMV, bl.PATH_TC])
def test_rmsnorm_special_rows(cuda, path):
    K = 512
    x = workloads.activations_f32(4, K, seed=21)
    x[0, :] = 0.0                   # zero token: normalises to zero, y = 0
    x[1, :] = -2.5                  # constant token
    x[2, :] *= np.float32(1e-4)     # so small that eps shifts r
    c = NormCase(4, K, 96, g_seed=22, w_seed=23, x=x)
    got = c.run(path=path)
    c.check_norm_full(got)
    assert np.all(got["xq"][0] == 0) and np.all(got["y"][0] == 0)
    assert got["beta"][0] == np.float32(1e-5)


@pytest.mark.parametrize("path", [bl.PATH_GEMV, bl.PATH_TC])
def test_rmsnorm_unit_gains_and_other_eps(cuda, path):
    K = 1024
    c = NormCase(5, K, 130, gain=np.ones(K, dtype=np.float32), eps=1e-6, w_seed=31, x_seed=32)
    c.check_norm_full(c.run(path=path))


def test_rmsnorm_paths_agree(cuda):
    c = NormCase(16, 2560, 700, g_seed=41, w_seed=42, x_seed=43)
    a = c.run(path=bl.PATH_GEMV)
    b = c.run(path=bl.PATH_TC)
    c.check_norm_full(a)
    c.check_norm_full(b)


# ------------------------------------------------- full-size workloads

def test_rmsnorm_decode_2b(cuda):
    for p in workloads.decode_gemv_2b().problems:
        c = NormCase(p.M, p.K, p.N, g_seed=p.w_seed + 50, w_seed=p.w_seed, x_seed=p.x_seed)
        c.check_norm_full(c.run())


def test_rmsnorm_prefill_2b(cuda):
    for p in workloads.prefill_2b().problems:
        c = NormCase(p.M, p.K, p.N, g_seed=p.w_seed + 50, w_seed=p.w_seed, x_seed=p.x_seed)
        c.check_norm_sampled(c.run(), count=30000)
