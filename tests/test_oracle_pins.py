"""The CPU oracle against its pins (hand examples, brute force, library
routines, closed forms and invariants); see tests/pins.py."""
import pytest

import oracle
from tests import pins


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_forward_normalises_before_quantising(orc):
    """forward(norm_gain=g) quantises the RMS-normalised tokens, both for fp32
    inputs and for bf16 bit patterns (widened first); without a gain the
    tokens go to the quantiser as they are."""
    import numpy as np
    r = np.random.Generator(np.random.PCG64(84))
    x = (r.standard_normal((3, 256)) * 4.0).astype(np.float32)
    W = (r.standard_normal((40, 256)) * 0.02).astype(np.float32)
    g = r.uniform(0.5, 1.5, size=256).astype(np.float32)
    res = orc.forward(x, W, norm_gain=g)
    xq, beta = orc.quant_act(orc.rmsnorm(x, g))
    np.testing.assert_array_equal(res["xq"], xq)
    np.testing.assert_array_equal(res["beta"], beta)
    np.testing.assert_array_equal(res["y"], orc.rescale_bf16(orc.matmul_i32(xq, res["Wq"]),
                                                            beta, res["gamma"]))
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    res16 = orc.forward(bits, W, norm_gain=g)
    np.testing.assert_array_equal(res16["xq"], orc.quant_act(orc.rmsnorm(orc.bf16_to_f32(bits), g))[0])
    np.testing.assert_array_equal(orc.forward(x, W)["xq"], orc.quant_act(x)[0])


def test_openmp_build_gives_the_same_products(orc):
    """The all-core copy of the oracle (the same source built with -fopenmp,
    timed only by the benchmark's CPU baseline) computes the same integer
    products as the single-threaded build: each output is the same plain sum,
    only the outputs are shared between threads."""
    import numpy as np
    omp = oracle.Oracle(oracle.load_omp())
    r = np.random.Generator(np.random.PCG64(85))
    xq = r.integers(-127, 128, size=(5, 1280)).astype(np.int8)
    Wq = r.integers(-1, 2, size=(333, 1280)).astype(np.int8)
    np.testing.assert_array_equal(omp.matmul_i32(xq, Wq), orc.matmul_i32(xq, Wq))
    ms = r.integers(0, 5, 999)
    ns = r.integers(0, 333, 999)
    np.testing.assert_array_equal(omp.matmul_i32_pairs(xq, Wq, ms, ns),
                                  orc.matmul_i32_pairs(xq, Wq, ms, ns))
