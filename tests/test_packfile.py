"""Packed-weight files (bitlinear_save_packed / bitlinear_read_packed_header /
bitlinear_load_packed): host-only, no GPU.

The header layout is checked by parsing the raw bytes here with struct, and
the payload hash by an FNV-1a implementation written from its published
definition and checked against the FNV test vectors."""
import ctypes
import os
import struct

import numpy as np
import pytest

import workloads
import ternary_weight_w1_b200 as bl

HEADER = struct.Struct("<8sIIqqfIQQQ")        # 64 bytes


def fnv1a64(data: bytes) -> int:
    h = 0xCBF29CE484222325
    for c in data:
        h = ((h ^ c) * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def test_fnv1a64_matches_published_vectors():
    assert HEADER.size == 64
    assert fnv1a64(b"") == 0xCBF29CE484222325
    assert fnv1a64(b"a") == 0xAF63DC4C8601EC8C
    assert fnv1a64(b"foobar") == 0x85944171F73967E8


@pytest.fixture
def packed_case():
    N, K = 300, 384                                  # ragged row blocks
    packed, gamma = bl.bitlinear_pack_weights(workloads.latent_weights(N, K, 17))
    return packed, N, K, gamma


def test_round_trip_and_header_layout(tmp_path, packed_case):
    packed, N, K, gamma = packed_case
    path = tmp_path / "w.blp"
    bl.bitlinear_save_packed(path, packed, N, K, gamma)
    assert not os.path.exists(str(path) + ".tmp")
    raw = path.read_bytes()
    assert len(raw) == 64 + packed.size
    magic, ver, layout, n, k, g, r0, nbytes, h, r1 = HEADER.unpack(raw[:64])
    assert (magic, ver, layout, n, k, r0, nbytes, r1) == (b"BITLIN58", 1, 1, N, K, 0,
                                                          packed.size, 0)
    assert np.float32(g) == np.float32(gamma)
    assert raw[64:] == packed.tobytes()
    assert h == fnv1a64(packed.tobytes())

    assert bl.bitlinear_read_packed_header(path) == (N, K, float(np.float32(gamma)))
    got, n2, k2, g2 = bl.bitlinear_load_packed(path)
    np.testing.assert_array_equal(got, packed)
    assert (n2, k2) == (N, K) and np.float32(g2) == np.float32(gamma)


def _rewrite(path, raw: bytes):
    with open(path, "wb") as f:
        f.write(raw)


@pytest.mark.parametrize("damage", ["payload_bit", "truncated", "trailing", "magic", "version",
                                    "layout", "size_field", "gamma_zero", "shape", "short_header"])
def test_damaged_files_are_refused(tmp_path, packed_case, damage):
    packed, N, K, gamma = packed_case
    path = tmp_path / "w.blp"
    bl.bitlinear_save_packed(path, packed, N, K, gamma)
    raw = bytearray(path.read_bytes())
    f = list(HEADER.unpack(bytes(raw[:64])))
    if damage == "payload_bit":
        raw[64 + 1000] ^= 0x04
    elif damage == "truncated":
        raw = raw[:-1]
    elif damage == "trailing":
        raw += b"\0"
    elif damage == "short_header":
        raw = raw[:40]
    else:
        if damage == "magic":
            f[0] = b"BITLIN57"
        elif damage == "version":
            f[1] = 2
        elif damage == "layout":
            f[2] = 7
        elif damage == "size_field":
            f[7] = packed.size - 512
        elif damage == "gamma_zero":
            f[5] = 0.0
        elif damage == "shape":
            f[4] = K + 64                            # not a multiple of 128
        raw[:64] = HEADER.pack(*f)
    _rewrite(path, bytes(raw))
    with pytest.raises(bl.BitLinearError) as e:
        bl.bitlinear_load_packed(path)
    assert e.value.status == bl.BITLINEAR_ERR_FORMAT


def test_io_errors(tmp_path, packed_case):
    packed, N, K, gamma = packed_case
    with pytest.raises(bl.BitLinearError) as e:
        bl.bitlinear_load_packed(tmp_path / "missing.blp")
    assert e.value.status == bl.BITLINEAR_ERR_IO
    target = tmp_path / "no_such_dir" / "w.blp"
    with pytest.raises(bl.BitLinearError) as e:
        bl.bitlinear_save_packed(target, packed, N, K, gamma)
    assert e.value.status == bl.BITLINEAR_ERR_IO
    assert not os.path.exists(str(target) + ".tmp")


def test_argument_errors(tmp_path, packed_case):
    packed, N, K, gamma = packed_case
    L = bl.lib()
    p = os.fsencode(tmp_path / "w.blp")
    buf = packed.ctypes.data
    assert L.bitlinear_save_packed(None, buf, N, K, gamma) == bl.BITLINEAR_ERR_ARG
    assert L.bitlinear_save_packed(p, None, N, K, gamma) == bl.BITLINEAR_ERR_ARG
    assert L.bitlinear_save_packed(p, buf, N, 200, gamma) == bl.BITLINEAR_ERR_SHAPE
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        assert L.bitlinear_save_packed(p, buf, N, K, bad) == bl.BITLINEAR_ERR_ARG
    assert not os.path.exists(tmp_path / "w.blp")
    bl.bitlinear_save_packed(tmp_path / "w.blp", packed, N, K, gamma)
    n, k, g = ctypes.c_int64(-5), ctypes.c_int64(-5), ctypes.c_float(-5.0)
    small = np.empty(packed.size - 1, dtype=np.uint8)
    rc = L.bitlinear_load_packed(p, small.ctypes.data, small.size, ctypes.addressof(n),
                                 ctypes.addressof(k), ctypes.addressof(g))
    assert rc == bl.BITLINEAR_ERR_ARG
    assert (n.value, k.value, g.value) == (-5, -5, -5.0)       # outputs untouched
    assert L.bitlinear_read_packed_header(p, None, ctypes.addressof(k),
                                          ctypes.addressof(g)) == bl.BITLINEAR_ERR_ARG


def test_packed_bytes_refuses_overflowing_sizes():
    assert bl.bitlinear_packed_bytes(1 << 62, 1 << 20) == 0
    assert bl.bitlinear_packed_bytes((1 << 63) - 1, 128) == 0
    assert bl.bitlinear_packed_bytes(16, 128) == 512
