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
    W = np.zeros((2, 128), dtype=np.float32)
    W[:, :4] = np.array(g["W"], dtype=np.float32)
    packed, gamma, Wq = check_pack(orc, W)
    # 4 weights + 124 zeros per row: the mean over 256 entries is 0.144 / 256
    assert abs(gamma - 0.144 / 256) < 1e-9
    np.testing.assert_array_equal(pins.decode_packed_spec(packed, 2, 128), Wq)


def test_golden_bytes(orc):
    for name, N, K, ws, by, size in pins.load_pack_cases():
        # latents whose ternarisation is the golden pattern: +-1 entries
        # among zeros have |W| / mean|W| >= 1 whenever zeros dominate
        W = np.zeros((N, K), dtype=np.float32)
        for r, k, v in ws:
            W[r, k] = v
        packed, gamma = bl.bitlinear_pack_weights(W)
        want = np.full(size, 0x55, dtype=np.uint8)
        for off, val in by.items():
            want[off] = val
        np.testing.assert_array_equal(packed, want, err_msg=name)


@pytest.mark.parametrize("N,K,seed", [(256, 256, 0), (7, 128, 1), (33, 1280, 2),
                                      (640, 2560, 3), (2560, 6912, 2), (1001, 384, 4)])
def test_random_latents(orc, N, K, seed):
    check_pack(orc, workloads.latent_weights(N, K, seed))


def test_zero_and_tiny_matrices(orc):
    packed, gamma, Wq = check_pack(orc, np.zeros((3, 128), dtype=np.float32))
    assert gamma == np.float32(1e-5) and np.all(Wq == 0)
    assert np.all(packed == 0x55)
    check_pack(orc, np.full((2, 128), 3e-7, dtype=np.float32))


def test_rejects_bad_shapes():
    with pytest.raises(bl.BitLinearError):
        bl.bitlinear_pack_weights(np.zeros((2, 64), dtype=np.float32))
    L = bl.lib()
    g = np.zeros(1, dtype=np.float32)
    out = np.zeros(16 * 32, dtype=np.uint8)
    W = np.zeros((4, 128), dtype=np.float32)
    assert L.bitlinear_pack_weights(None, 4, 128, out.ctypes.data, g.ctypes.data) == bl.BITLINEAR_ERR_ARG
    assert L.bitlinear_pack_weights(W.ctypes.data, 0, 128, out.ctypes.data, g.ctypes.data) == bl.BITLINEAR_ERR_ARG
    assert L.bitlinear_pack_weights(W.ctypes.data, 4, 64, out.ctypes.data, g.ctypes.data) == bl.BITLINEAR_ERR_SHAPE


# ------------------------------------------------------------- base-3 layout

def check_pack_b3(orc, W):
    """The base-3 packer: the same gamma as the 2-bit packer, and bytes equal
    to the oracle's base-3 layout of the oracle's ternary weights."""
    packed, gamma = bl.bitlinear_pack_weights_b3(W)
    _, gamma2 = bl.bitlinear_pack_weights(W)
    assert gamma == gamma2
    Wq = orc.ternarize(W, np.float32(gamma))
    np.testing.assert_array_equal(packed, orc.pack_codes_b3(Wq))
    N, K = W.shape
    assert packed.size == bl.bitlinear_packed_bytes_b3(N, K)
    assert packed.size == (N + 15) // 16 * 16 * ((K + 159) // 160 * 160) // 5
    return packed, Wq


def test_b3_golden_bytes():
    for name, N, K, ws, by, size in pins.load_pack_cases("pack_b3_bytes.txt"):
        W = np.zeros((N, K), dtype=np.float32)
        for r, k, v in ws:
            W[r, k] = v
        packed, _ = bl.bitlinear_pack_weights_b3(W)
        want = np.full(size, 121, dtype=np.uint8)
        for off, val in by.items():
            want[off] = val
        np.testing.assert_array_equal(packed, want, err_msg=name)


@pytest.mark.parametrize("N,K,seed", [(256, 256, 0), (7, 128, 1), (33, 1280, 2),
                                      (640, 2560, 3), (2560, 6912, 2), (1001, 384, 4)])
def test_b3_random_latents(orc, N, K, seed):
    packed, Wq = check_pack_b3(orc, workloads.latent_weights(N, K, seed))
    if N * K <= 64 * 1024:
        np.testing.assert_array_equal(pins.decode_packed_b3_spec(packed, N, K), Wq)


def test_b3_sizes_and_bad_shapes():
    # 1.6 bits per weight once K is a multiple of 160
    assert bl.bitlinear_packed_bytes_b3(16, 2560) * 5 == 16 * 2560
    assert bl.bitlinear_packed_bytes_b3(16, 6912) == 16 * 7040 // 5
    assert bl.bitlinear_packed_bytes_b3(0, 128) == 0
    assert bl.bitlinear_packed_bytes_b3(4, 100) == 0
    with pytest.raises(bl.BitLinearError):
        bl.bitlinear_pack_weights_b3(np.zeros((2, 64), dtype=np.float32))
    L = bl.lib()
    g = np.zeros(1, dtype=np.float32)
    out = np.zeros(16 * 32, dtype=np.uint8)
    W = np.zeros((4, 128), dtype=np.float32)
    assert L.bitlinear_pack_weights_b3(None, 4, 128, out.ctypes.data, g.ctypes.data) == bl.BITLINEAR_ERR_ARG
    assert L.bitlinear_pack_weights_b3(W.ctypes.data, 4, 64, out.ctypes.data, g.ctypes.data) == bl.BITLINEAR_ERR_SHAPE
