"""bitlinear_forward_grouped: several independent BitLinear matmuls in one
GEMV launch must give, problem by problem, exactly what the oracle gives and
what separate bitlinear_forward calls give."""
import numpy as np
import pytest

import workloads
import ternary_weight_w1_b200 as bl
from tests.gpu_cases import CANARY_Y, Case, Guarded, check_y, tensor_to_bf16_bits

pytestmark = pytest.mark.gpu


def _guarded_problems(cases, xs):
    """(problems with canary-guarded outputs, the guards)."""
    import torch
    probs, guards = [], []
    for i, c in enumerate(cases):
        x = c.x_tensor() if xs is None else xs[i]
        g = Guarded((c.M, c.N), torch.bfloat16, x.device, CANARY_Y)
        guards.append(g)
        probs.append((x, c.packed_tensor(), c.gamma, c.N, g.t))
    return probs, guards


def _read(guards):
    for i, g in enumerate(guards):
        g.check(f"problem {i}'s y")
    return [tensor_to_bf16_bits(g.t) for g in guards]


def run_group(cases, xs=None):
    import torch
    probs, guards = _guarded_problems(cases, xs)
    bl.bitlinear_forward_grouped(probs)
    torch.cuda.synchronize()
    return _read(guards), probs


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


# ---------------------------------------------- grouped tensor-core path

def run_group_ws(cases, xs=None):
    import torch
    probs, guards = _guarded_problems(cases, xs)
    need = bl.bitlinear_workspace_bytes_grouped(probs)
    ws = torch.empty((max(need, 1),), dtype=torch.uint8, device="cuda")
    bl.bitlinear_forward_grouped(probs, workspace=ws)
    torch.cuda.synchronize()
    return _read(guards)


def test_grouped_tc_mixed_shapes_match_single_calls():
    # batch 8 of four 2B shapes: one quantisation launch and one GEMM launch;
    # every problem equals the oracle and its own bitlinear_forward call
    cases = [Case(8, 2560, 2560, w_seed=61, x_seed=71), Case(8, 2560, 640, w_seed=62, x_seed=72),
             Case(8, 2560, 6912, w_seed=63, x_seed=73), Case(8, 6912, 2560, w_seed=64, x_seed=74)]
    ys = run_group_ws(cases)
    for c, y in zip(cases, ys):
        assert check_y(y, c.oracle_full()[1]) == 1.0
        single = c.run(path=bl.PATH_TC, debug=False)["y"]
        np.testing.assert_array_equal(y, single)


def test_grouped_tc_layer_b64():
    # the seven projections of one decoder layer at batch 64 (token tile 64)
    cases = [Case(p.M, p.K, p.N, w_seed=p.w_seed, x_seed=p.x_seed)
             for p in workloads.layer_set_2b(64, layers=1).problems]
    ys = run_group_ws(cases)
    for c, y in zip(cases, ys):
        assert check_y(y, c.oracle_full()[1]) == 1.0


def test_grouped_tc_mixed_batches_fp32():
    # one problem above the GEMV threshold sends the whole group to the
    # tensor-core path, M = 1 and ragged shapes included; largest M sets the tile
    cases = [Case(1, 256, 300, w_seed=81, x_seed=91, x_dtype="fp32"),
             Case(40, 1280, 333, w_seed=82, x_seed=92, x_dtype="fp32"),
             Case(150, 384, 129, w_seed=83, x_seed=93, x_dtype="fp32")]
    ys = run_group_ws(cases)
    for c, y in zip(cases, ys):
        assert check_y(y, c.oracle_full()[1]) == 1.0


def test_grouped_ws_small_batches_use_gemv():
    cases = [Case(1, 2560, 6912, w_seed=1, x_seed=101), Case(4, 6912, 2560, w_seed=2, x_seed=102)]
    ys = run_group_ws(cases)
    for c, y in zip(cases, ys):
        assert check_y(y, c.oracle_full()[1]) == 1.0


# ------------------------------------------- grouped, RMS-normalised tokens

def run_group_norm(cases, gains, eps=bl.RMSNORM_EPS):
    import torch
    probs, guards = _guarded_problems(cases, None)
    need = bl.bitlinear_workspace_bytes_grouped(probs)
    ws = torch.empty((max(need, 1),), dtype=torch.uint8, device="cuda")
    g_dev = [torch.from_numpy(g).cuda() for g in gains]
    bl.bitlinear_forward_grouped_rmsnorm(probs, g_dev, eps=eps, workspace=ws)
    torch.cuda.synchronize()
    return _read(guards)


@pytest.mark.parametrize("B", [1, 8, 64])
def test_grouped_rmsnorm_layer_matches_oracle(B):
    """The seven projections of a decoder layer, each normalising its tokens
    with its own gains (GEMV launch at B = 1, grouped quantisation and GEMM
    at B = 8 and 64), against the oracle's RMSNorm + forward. The device adds
    each token's squares in another order, so an x~ on a rounding tie may go
    either way (the bar of the other normalised forms): y within the parity
    tolerance and bit-identical almost everywhere, and the same against the
    single-problem normalising call (whose quantiser may combine a long row's
    partial sums in another order)."""
    probs = workloads.layer_set_2b(B, layers=1).problems
    cases = [Case(p.M, p.K, p.N, w_seed=p.w_seed, x_seed=p.x_seed) for p in probs]
    gains = [workloads.norm_gains(p.K, p.w_seed + 7) for p in probs]
    ys = run_group_norm(cases, gains)
    import torch
    for c, g, y in zip(cases, gains, ys):
        ref = c.orc.forward(c.x_bits, c.W, gamma=c.gamma, norm_gain=g)
        assert check_y(y, ref["y"]) >= 0.99
        single = torch.empty((c.M, c.N), dtype=torch.bfloat16, device="cuda")
        bl.bitlinear_forward_rmsnorm(c.x_tensor(), c.packed_tensor(), c.gamma, c.N,
                                     torch.from_numpy(g).cuda(), y=single)
        torch.cuda.synchronize()
        assert check_y(y, tensor_to_bf16_bits(single)) >= 0.99


# ------------------------------------------- host buffers in and out

def _host_call_check(cases, contiguous, pinned, repeats=1, pinned_y=None):
    """Runs bitlinear_forward_grouped_host on the cases' tokens (host memory,
    problem after problem) and compares the host outputs with the oracle bit
    for bit; the device staging buffers lie back to back (one copy each way)
    or in separate allocations (one copy per problem). Pinned host memory
    takes the kernel-staged tokens and the direct output path (when every
    problem's output part is 16-byte aligned), pageable memory the copies."""
    if pinned_y is None:
        pinned_y = pinned
    import torch
    dt = torch.bfloat16 if cases[0].x_dtype == "bf16" else torch.float32
    xk = [c.M * c.K for c in cases]
    yn = [c.M * c.N for c in cases]
    if contiguous:
        xs = [t.view(c.M, c.K) for t, c in zip(torch.split(torch.empty(sum(xk), dtype=dt,
                                                                      device="cuda"), xk), cases)]
        ys = [t.view(c.M, c.N) for t, c in
              zip(torch.split(torch.empty(sum(yn), dtype=torch.bfloat16, device="cuda"), yn),
                  cases)]
    else:
        xs = [torch.empty((c.M, c.K), dtype=dt, device="cuda") for c in cases]
        ys = [torch.empty((c.M, c.N), dtype=torch.bfloat16, device="cuda") for c in cases]
    call = bl.GroupedHostCall([(x, c.packed_tensor(), c.gamma, c.N, y)
                               for x, c, y in zip(xs, cases, ys)])
    host_x = torch.cat([c.x_tensor().reshape(-1).cpu() for c in cases])
    host_y = torch.full((sum(yn),), CANARY_Y, dtype=torch.int16).view(torch.bfloat16)
    if pinned:
        host_x = host_x.pin_memory()
    if pinned_y:
        host_y = host_y.pin_memory()
    for _ in range(repeats):
        call(host_x, host_y)
        torch.cuda.synchronize()
    got = host_y.view(torch.int16).numpy().view(np.uint16)
    assert not np.any(got == CANARY_Y), "an output element was not written"
    off = 0
    for c, n in zip(cases, yn):
        assert check_y(got[off:off + n].reshape(c.M, c.N), c.oracle_full()[1]) == 1.0
        off += n
    assert bl.bitlinear_get_fault() == (bl.BITLINEAR_OK, 0)


def test_grouped_host_decode_step_2b_pinned():
    cases = [Case(p.M, p.K, p.N, w_seed=p.w_seed, x_seed=p.x_seed)
             for p in workloads.decode_gemv_2b(1).problems]
    _host_call_check(cases, contiguous=True, pinned=True, repeats=3)


def test_grouped_host_mixed_fp32_separate_buffers_pageable():
    cases = [Case(1 + i % 3, 256 * (1 + i % 3), 80 + 48 * i, w_seed=60 + i, x_seed=70 + i,
                  x_dtype="fp32") for i in range(5)]
    _host_call_check(cases, contiguous=False, pinned=False)


def test_grouped_host_pinned_tokens_pageable_outputs():
    cases = [Case(p.M, p.K, p.N, w_seed=p.w_seed, x_seed=p.x_seed)
             for p in workloads.decode_gemv_2b(1).problems]
    _host_call_check(cases, contiguous=True, pinned=True, pinned_y=False, repeats=2)


def test_grouped_host_pinned_unaligned_output_parts():
    """N = 17 and 40: the second problem's outputs start 34 bytes into y_host,
    so the outputs go through the device buffers and a copy back."""
    cases = [Case(1, 512, 17, w_seed=81, x_seed=91), Case(2, 384, 40, w_seed=82, x_seed=92)]
    _host_call_check(cases, contiguous=False, pinned=True, repeats=2)
