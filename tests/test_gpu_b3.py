"""bitlinear_forward_b3: the GEMV on base-3 packed weights (five codes per
byte, decoded through a table in shared memory) against the CPU oracle, bit
for bit: x~, beta, the int32 product and y. The weights are ternarised by the
oracle with the packer's gamma, as for the 2-bit layout."""
import numpy as np
import pytest

import ternary_weight_w1_b200 as bl
from tests.gpu_cases import Case, guarded_outputs, read_guarded

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bl.lib()
    return torch


def run_b3(c):
    import torch
    packed, gamma = bl.bitlinear_pack_weights_b3(c.W)
    assert gamma == c.gamma                         # the same gamma as the 2-bit packer
    x = c.x_tensor()
    g = guarded_outputs(c.M, c.N, c.K, x.device)
    bl.bitlinear_forward_b3(x, torch.from_numpy(packed).cuda(), gamma, c.N, y=g["y"].t,
                            acc=g["acc"].t, xq=g["xq"].t, beta=g["beta"].t)
    torch.cuda.synchronize()
    return read_guarded(g)


@pytest.mark.parametrize("M,K,N", [(1, 2560, 6912), (1, 6912, 2560), (3, 384, 500),
                                   (16, 1280, 333), (2, 128, 16), (6, 8192, 700),
                                   (1, 28672, 300), (5, 2560, 17)])
def test_b3_matches_oracle(M, K, N):
    # K = 6912, 384, 8192, 28672, 128 are not multiples of 160: padded groups
    c = Case(M, K, N, w_seed=K + N + M, x_seed=3 * M + K)
    assert c.check_full(run_b3(c)) == 1.0


def test_b3_fp32_tokens_and_zero_rows():
    x = np.random.default_rng(9).standard_normal((4, 640)).astype(np.float32)
    x[2] = 0.0                                      # beta clamps to 1e-5, y is zero
    c = Case(4, 640, 96, x=x, x_dtype="fp32")
    got = run_b3(c)
    assert c.check_full(got) == 1.0
    assert np.all(got["acc"][2] == 0)


def test_b3_equals_2bit_path():
    c = Case(2, 2560, 1000, w_seed=4, x_seed=5)
    got = run_b3(c)
    ref = c.run(path=bl.PATH_GEMV)
    np.testing.assert_array_equal(got["y"], ref["y"])
    np.testing.assert_array_equal(got["acc"], ref["acc"])
    assert bl.bitlinear_get_fault() == (bl.BITLINEAR_OK, 0)


def test_b3_grouped_decode_pair_and_mixed():
    """bitlinear_forward_grouped_b3: the decode step's two projections and a
    mixed group in one launch each, every problem bit-exact against the
    oracle and equal to its single base-3 call."""
    import torch
    groups = [[Case(1, 2560, 6912, w_seed=21, x_seed=22), Case(1, 6912, 2560, w_seed=23, x_seed=24)],
              [Case(3, 384, 500, w_seed=25, x_seed=26), Case(1, 8192, 96, w_seed=27, x_seed=28),
               Case(6, 640, 33, w_seed=29, x_seed=30)]]
    for cases in groups:
        probs = []
        for c in cases:
            packed, gamma = bl.bitlinear_pack_weights_b3(c.W)
            probs.append((c.x_tensor(), torch.from_numpy(packed).cuda(), gamma, c.N, None))
        ys = bl.bitlinear_forward_grouped_b3(probs)
        torch.cuda.synchronize()
        for c, y, pr in zip(cases, ys, probs):
            got = y.view(torch.int16).cpu().numpy().view(np.uint16)
            np.testing.assert_array_equal(got, c.oracle_full()[1])
            single = run_b3(c)["y"]
            np.testing.assert_array_equal(got, single)
    assert bl.bitlinear_get_fault() == (bl.BITLINEAR_OK, 0)
