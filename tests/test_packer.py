"""The library's host packer (bitlinear_pack_weights) against the oracle:
the packed bytes equal the oracle's layout of the oracle's ternary weights,
bit for bit, and gamma agrees with the oracle's (double-accumulated) mean."""
import numpy as np
import pytest

import oracle
import workloads
import ternary_weight_w1_b200 as bl
from tests import pins


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


def check_pack(orc, W):
    packed, gamma = bl.bitlinear_pack_weights(W)
    g_or = orc.absmean_gamma(W)
    assert abs(np.float32(gamma) - g_or) <= np.spacing(g_or), (gamma, g_or)
    Wq = orc.ternarize(W, np.float32(gamma))
    np.testing.assert_array_equal(packed, orc.pack_codes(Wq))
    return packed, gamma, Wq


def test_hand_example(orc):
    g = pins.load_golden("hand_example.txt")
    W = np.zeros((2, 16), dtype=np.float32)
    W[:, :4] = np.array(g["W"], dtype=np.float32)
    packed, gamma, Wq = check_pack(orc, W)
    # 4 weights + 12 zeros: mean over 32 entries is 0.144 / 32
    assert abs(gamma - 0.144 / 32) < 1e-8
    np.testing.assert_array_equal(pins.decode_packed_spec(packed, 16), Wq)


def test_golden_words(orc):
    for name, wq, by in pins.load_pack_cases():
        # a latent whose ternarisation is wq: +-1 map to +-1, 0 to 0 (gamma = mean |W|,
        # and |W| / gamma >= 1 for the nonzeros, 0 for the zeros)
        W = np.array([wq], dtype=np.float32)
        packed, gamma = bl.bitlinear_pack_weights(W)
        assert packed.tolist() == [by], name


@pytest.mark.parametrize("N,K,seed", [(256, 256, 0), (7, 16, 1), (33, 1280, 2),
                                      (640, 2560, 3), (2560, 6912, 2)])
def test_random_latents(orc, N, K, seed):
    check_pack(orc, workloads.latent_weights(N, K, seed))


def test_zero_and_tiny_matrices(orc):
    packed, gamma, Wq = check_pack(orc, np.zeros((3, 32), dtype=np.float32))
    assert gamma == np.float32(1e-5) and np.all(Wq == 0)
    assert np.all(packed == 0x55)
    check_pack(orc, np.full((2, 16), 3e-7, dtype=np.float32))


def test_rejects_bad_shapes():
    with pytest.raises(bl.BitLinearError):
        bl.bitlinear_pack_weights(np.zeros((2, 20), dtype=np.float32))
    L = bl.lib()
    g = np.zeros(1, dtype=np.float32)
    out = np.zeros(64, dtype=np.uint8)
    W = np.zeros((4, 16), dtype=np.float32)
    assert L.bitlinear_pack_weights(None, 4, 16, out.ctypes.data, g.ctypes.data) == bl.BITLINEAR_ERR_ARG
    assert L.bitlinear_pack_weights(W.ctypes.data, 0, 16, out.ctypes.data, g.ctypes.data) == bl.BITLINEAR_ERR_ARG
    assert L.bitlinear_pack_weights(W.ctypes.data, 4, 8, out.ctypes.data, g.ctypes.data) == bl.BITLINEAR_ERR_SHAPE
