"""Parity of the CUDA library (through its C ABI) with the CPU oracle.

Small and mid sizes that span several tiles and ragged tails are compared
element by element. The full-size workloads run in the launch configuration
the benchmark uses (the automatic path) and are compared in full (x~, beta,
every acc and y element, with the OpenMP build of the oracle for the integer
products), except the M = 4096 large shapes: those on the full activation
stage and on sampled outputs of the product.
"""
import numpy as np
import pytest

import oracle
import workloads
import ternary_weight_w1_b200 as bl
from tests.gpu_cases import Case, bf16_bits_to_tensor, check_y, tensor_to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bl.lib()
    return torch


# ------------------------------------------------------- quantisation kernel

# From 1024 tokens the rows are staged in shared memory, 4 to 8 per block:
# (2048, 6912) eight per block; (1027, 2560, fp32) eight, the last block three;
# (1100, 8192) seven, the last block one; (1030, 7168, fp32) four.
@pytest.mark.parametrize("M,K,dtype", [(4, 256, "fp32"), (1, 2560, "bf16"), (1, 6912, "bf16"),
                                       (37, 1280, "bf16"), (300, 2560, "fp32"),
                                       (2048, 6912, "bf16"), (1027, 2560, "fp32"),
                                       (1100, 8192, "bf16"), (1030, 7168, "fp32"),
                                       (3, 28672, "bf16"), (5, 65536, "fp32")])
def test_quant_act(cuda, M, K, dtype):
    xf = workloads.activations_f32(M, K, seed=M * 31 + K)
    xf[0, :] = 0.0                                           # an all-zero token
    if M > 2:
        xf[1, :] = -0.375                                    # a constant token
    c = Case(M, K, 16, x=xf, x_dtype=dtype)
    xq, beta = bl.bitlinear_quant_act(c.x_tensor())
    cuda.cuda.synchronize()
    np.testing.assert_array_equal(beta.cpu().numpy(), c.beta)
    np.testing.assert_array_equal(xq.cpu().numpy(), c.xq)


# -------------------------------------------------------------- GEMV path

@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 11, 16])
@pytest.mark.parametrize("K,N", [(256, 256), (1280, 300), (2560, 640), (6912, 37), (128, 5)])
def test_gemv_parity(cuda, M, K, N):
    c = Case(M, K, N, w_seed=K + N, x_seed=M + 7 * K)
    got = c.run(path=bl.PATH_GEMV)
    exact = c.check_full(got)
    assert exact == 1.0


def test_gemv_fp32_input(cuda):
    c = Case(4, 256, 256, w_seed=0, x_seed=0, x_dtype="fp32", outliers=False)
    assert c.check_full(c.run(path=bl.PATH_GEMV)) == 1.0


# ------------------------------------------------------ tensor-core path

@pytest.mark.parametrize("M", [1, 100, 128, 129, 300])
@pytest.mark.parametrize("K,N", [(256, 256), (1280, 333), (2560, 600), (128, 513)])
def test_tc_parity(cuda, M, K, N):
    c = Case(M, K, N, w_seed=3 * K + N, x_seed=M + 5 * K)
    got = c.run(path=bl.PATH_TC)
    exact = c.check_full(got)
    assert exact == 1.0


@pytest.mark.parametrize("M,K,N", [(40, 6912, 8192), (17, 2560, 19000), (64, 8320, 4600)])
def test_tc_deep_stages(cuda, M, K, N):
    """Token tiles of 32 and 64 with at least 8 k-blocks of 256 per CTA take
    512-k stages; K = 6912 and 8320 leave part of the last stage outside the
    tensors (zero-filled), N a ragged last weight tile. Full comparison."""
    c = Case(M, K, N, w_seed=7 * K + N, x_seed=M + 3 * K)
    got = c.run(path=bl.PATH_TC)
    assert c.check_full(got, _omp_oracle()) == 1.0


@pytest.mark.parametrize("M", [20, 50, 200, 300])
def test_tc_token_tiles_shared_k(cuda, M):
    # token tiles of 32, 64, 128 and 192 rows; only a few tiles with 54
    # k-blocks each, so the k-range of every tile is shared by many CTAs
    # whose int32 partial sums are combined by the tile's first CTA
    c = Case(M, 6912, 300, w_seed=M, x_seed=M + 1)
    assert c.check_full(c.run(path=bl.PATH_TC)) == 1.0


def test_tc_tiles_split_between_two_ctas(cuda):
    # 160 tiles of 10 k-blocks over the CTAs: most tiles are split in two
    c = Case(1000, 1280, 2560, w_seed=21, x_seed=22)
    assert c.check_full(c.run(path=bl.PATH_TC)) == 1.0


@pytest.mark.parametrize("path,M", [(bl.PATH_GEMV, 1), (bl.PATH_GEMV, 3), (bl.PATH_TC, 3),
                                    (bl.PATH_TC, 40)])
def test_maximum_k_and_single_output_row(cuda, path, M):
    # K = 65536 (the largest K the forward calls accept) and N = 1 (one row
    # block holding 15 padding rows), on both paths
    for K, N in [(65536, 130), (2560, 1)]:
        if path == bl.PATH_GEMV and M * K > 196608:
            continue
        c = Case(M, K, N, w_seed=K + N + M, x_seed=M + K)
        assert c.check_full(c.run(path=path)) == 1.0


def test_gemv_tall_matrix_next_to_large_x(cuda):
    # x~ of 16 x 12160 bytes leaves little shared memory beside it, so the
    # weights stream in small stages; 1499 row blocks (the last one ragged)
    # spread over the CTAs, some holding one block more than others
    c = Case(16, 12160, 23970, w_seed=61, x_seed=62)
    assert c.check_sampled(c.run(path=bl.PATH_GEMV), count=20000) == 1.0


@pytest.mark.parametrize("K,N,dtype", [(8320, 700, "bf16"), (16384, 333, "bf16"),
                                       (28672, 1000, "bf16"), (32768, 130, "bf16"),
                                       (16384, 300, "fp32"), (33024, 77, "bf16")])
def test_gemv_long_rows_single_token(cuda, K, N, dtype):
    # one bf16 token of 8192 < K <= 32768 takes the kernel that stages the
    # row in shared memory for its prologue (x~ then overwrites the staged
    # row); fp32 tokens and K = 33024 take the register-cached prologue with
    # reloads
    c = Case(1, K, N, w_seed=K + N, x_seed=K - N, x_dtype=dtype)
    assert c.check_full(c.run(path=bl.PATH_GEMV)) == 1.0


def test_tc_many_tiles_per_cta(cuda):
    # more tiles than SMs: every CTA loops over several tiles and both TMEM
    # accumulator buffers are reused
    c = Case(1024, 512, 8192, w_seed=11, x_seed=12)
    got = c.run(path=bl.PATH_TC)
    assert c.check_sampled(got, count=50000) == 1.0


def test_tc_fp32_input(cuda):
    c = Case(200, 256, 256, w_seed=0, x_seed=0, x_dtype="fp32", outliers=False)
    assert c.check_full(c.run(path=bl.PATH_TC)) == 1.0


# ------------------------------------------------------------- edge cases

@pytest.mark.parametrize("path", [bl.PATH_GEMV, bl.PATH_TC])
def test_zero_activations_and_weights(cuda, path):
    x = np.zeros((3, 256), dtype=np.float32)
    c = Case(3, 256, 64, x=x)
    got = c.run(path=path)
    c.check_full(got)
    assert np.all(got["y"] == 0) and np.all(got["beta"] == np.float32(1e-5))
    W = np.zeros((64, 256), dtype=np.float32)
    c2 = Case(3, 256, 64, W=W)
    got2 = c2.run(path=path)
    c2.check_full(got2)
    assert np.all(got2["acc"] == 0)


@pytest.mark.parametrize("path", [bl.PATH_GEMV, bl.PATH_TC])
def test_identity_weights(cuda, path):
    K = 256
    c = Case(2, K, K, W=np.eye(K, dtype=np.float32))
    got = c.run(path=path)
    c.check_full(got)
    np.testing.assert_array_equal(got["acc"], c.xq.astype(np.int32))


def test_empty_batch_is_a_noop(cuda):
    torch = cuda
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros((64, 64), dtype=torch.uint8, device="cuda")
    y = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    bl.bitlinear_forward(x, packed, 1.0, 64, y=y)
    torch.cuda.synchronize()


def test_deterministic(cuda):
    c = Case(300, 1280, 700, w_seed=5, x_seed=6)
    a = c.run(path=bl.PATH_TC)
    b = c.run(path=bl.PATH_TC)
    np.testing.assert_array_equal(a["y"], b["y"])
    g1 = c.run(path=bl.PATH_AUTO, debug=False)
    np.testing.assert_array_equal(a["y"], g1["y"])


def test_paths_agree_at_m16(cuda):
    c = Case(16, 2560, 1000, w_seed=8, x_seed=9)
    a = c.run(path=bl.PATH_GEMV)
    b = c.run(path=bl.PATH_TC)
    np.testing.assert_array_equal(a["acc"], b["acc"])
    np.testing.assert_array_equal(a["y"], b["y"])


# ------------------------------------------------- full-size workloads

def _problem_case(p):
    return Case(p.M, p.K, p.N, w_seed=p.w_seed, x_seed=p.x_seed, x_dtype=p.x_dtype,
                outliers=p.outliers)


def test_tiny_workload(cuda):
    for p in workloads.tiny().problems:
        c = _problem_case(p)
        assert c.check_full(c.run()) == 1.0


def test_decode_gemv_2b(cuda):
    for p in workloads.decode_gemv_2b().problems:
        c = _problem_case(p)
        assert c.check_full(c.run()) == 1.0


def _omp_oracle():
    """The OpenMP build of the oracle (integer products over all host cores),
    for comparing whole full-size problems."""
    return oracle.Oracle(oracle.load_omp())


@pytest.mark.parametrize("B", [1, 8, 64])
def test_layer_set_2b(cuda, B):
    wl = workloads.layer_set_2b(B)
    first = wl.problems[:7]           # layer 0: every projection shape
    last = wl.problems[-7:]           # layer 29
    orc = _omp_oracle()
    for p in first + last:
        c = _problem_case(p)
        assert c.check_full(c.run(), orc) == 1.0


def test_prefill_2b(cuda):
    """The M = 2048 prefill step in full: x~, beta, every acc element and every
    output of both projections (all token tiles, weight tiles and stream-K
    segments of the launches)."""
    orc = _omp_oracle()
    for p in workloads.prefill_2b().problems:
        c = _problem_case(p)
        assert c.check_full(c.run(), orc) == 1.0


@pytest.mark.parametrize("M", [1, 16, 256, 4096])
def test_large_sweep(cuda, M):
    """In full up to M = 256; at M = 4096 (1.9 T multiply-adds, minutes of
    host time) on sampled outputs, two full rows and two full columns."""
    orc = _omp_oracle()
    for p in workloads.large_sweep(M).problems:
        c = _problem_case(p)
        got = c.run()
        if M <= 256:
            assert c.check_full(got, orc) == 1.0
        else:
            assert c.check_sampled(got, count=20000) == 1.0


# ------------------------------------------------- failure detection

@pytest.mark.parametrize("path,M,K,N", [(bl.PATH_TC, 256, 512, 512),
                                         (bl.PATH_GEMV, 1, 2560, 700),
                                         (bl.PATH_GEMV, 3, 6912, 300)])
def test_bounded_wait_reports_timeout_and_context_survives(cuda, path, M, K, N):
    """One wait made to run out (GEMV: the first weight stage is never loaded;
    tensor cores: the MMA issuer waits on a barrier nobody arrives at): the
    fault word reports it, y is left untouched (no partial results), the word
    is cleared by reading it, and the context still computes correct
    results."""
    torch = cuda
    c = Case(M, K, N, w_seed=1, x_seed=1)
    x = c.x_tensor()
    packed = c.packed_tensor()
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    canary = tensor_to_bf16_bits(y)
    assert bl.bitlinear_get_fault() == (bl.BITLINEAR_OK, 0)
    rc = bl.bitlinear_forward_inject_timeout(x, packed, c.gamma, c.N, timeout_us=2000, y=y,
                                             path=path)
    assert rc == bl.BITLINEAR_OK
    status, word = bl.bitlinear_get_fault()
    assert status == bl.BITLINEAR_ERR_TIMEOUT and word == 1
    np.testing.assert_array_equal(tensor_to_bf16_bits(y), canary)
    # the word is cleared, and the context still runs correct work
    assert bl.bitlinear_get_fault() == (bl.BITLINEAR_OK, 0)
    assert c.check_full(c.run(path=path)) == 1.0
    assert bl.bitlinear_get_fault() == (bl.BITLINEAR_OK, 0)
