"""bitlinear_forward_grouped: several independent BitLinear matmuls in one
GEMV launch must give, problem by problem, exactly what the oracle gives and
what separate bitlinear_forward calls give."""
import numpy as np
import pytest

import workloads
import ternary_weight_w1_b200 as bl
from tests.gpu_cases import Case, check_y, tensor_to_bf16_bits

pytestmark = pytest.mark.gpu


def run_group(cases, xs=None):
    import torch
    probs = []
    for i, c in enumerate(cases):
        x = c.x_tensor() if xs is None else xs[i]
        probs.append((x, c.packed_tensor(), c.gamma, c.N, None))
    outs = bl.bitlinear_forward_grouped(probs)
    torch.cuda.synchronize()
    return [tensor_to_bf16_bits(y) for y in outs], probs


def test_grouped_mixed_shapes():
    cases = [Case(1, 2560, 6912, w_seed=1, x_seed=101), Case(1, 6912, 2560, w_seed=2, x_seed=102),
             Case(3, 1280, 300, w_seed=3, x_seed=103), Case(2, 256, 640, w_seed=4, x_seed=104),
             Case(16, 384, 17, w_seed=5, x_seed=105)]
    ys, _ = run_group(cases)
    for c, y in zip(cases, ys):
        _, y_ref = c.oracle_full()
        assert check_y(y, y_ref) == 1.0
        single = c.run(path=bl.PATH_GEMV, debug=False)["y"]
        np.testing.assert_array_equal(y, single)


def test_grouped_decode_step_2b():
    cases = [Case(p.M, p.K, p.N, w_seed=p.w_seed, x_seed=p.x_seed)
             for p in workloads.decode_gemv_2b(1).problems]
    ys, _ = run_group(cases)
    for c, y in zip(cases, ys):
        assert check_y(y, c.oracle_full()[1]) == 1.0


def test_grouped_qkv_share_x():
    # q, k, v of one decoder layer read the same token
    p_q, p_k, p_v = workloads.layer_set_2b(4, layers=1).problems[:3]
    cases = [Case(p.M, p.K, p.N, w_seed=p.w_seed, x_seed=p_q.x_seed) for p in (p_q, p_k, p_v)]
    x = cases[0].x_tensor()
    ys, _ = run_group(cases, xs=[x, x, x])
    for c, y in zip(cases, ys):
        assert check_y(y, c.oracle_full()[1]) == 1.0


def test_grouped_eight_problems_fp32():
    cases = [Case(1 + i % 4, 256 * (1 + i % 3), 96 + 40 * i, w_seed=20 + i, x_seed=40 + i,
                  x_dtype="fp32") for i in range(8)]
    ys, _ = run_group(cases)
    for c, y in zip(cases, ys):
        assert check_y(y, c.oracle_full()[1]) == 1.0
