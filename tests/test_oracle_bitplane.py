"""Pins of the oracle's bit-plane format (its reading R11: a "nonzero" plane
n = (w != 0) and a "sign" plane s = (w < 0), about 2 bits per weight -- Bonsai
page, "后面还有没有优化空间", first direction), against numpy and closed
forms rather than the oracle itself."""
import itertools
import math

import numpy as np
import pytest

import oracle
from ternary_weight_decode_b200 import synth


@pytest.mark.parametrize("K", [1, 7, 8, 9, 100, 128, 641])
def test_canonical_planes_equal_numpy_packbits(K):
    w = synth.trits(21, 4, 11, K)
    b = oracle.pack_bitplane(w)
    P = math.ceil(K / 8)
    assert b.shape == (11, 2 * P) == (11, oracle.bitplane_row_bytes(K))
    np.testing.assert_array_equal(b[:, :P], np.packbits(w != 0, axis=1, bitorder="little"))
    np.testing.assert_array_equal(b[:, P:], np.packbits(w < 0, axis=1, bitorder="little"))
    np.testing.assert_array_equal(oracle.unpack_bitplane(b, K), w)


def test_every_pattern_of_six_round_trips():
    pats = np.array(list(itertools.product((-1, 0, 1), repeat=6)), np.int8)  # 729 rows
    b = oracle.pack_bitplane(pats)
    np.testing.assert_array_equal(oracle.unpack_bitplane(b, 6), pats)
    stride = 16
    d = oracle.pack_device(oracle.FMT_BITPLANE, pats, stride)
    np.testing.assert_array_equal(oracle.unpack_device(oracle.FMT_BITPLANE, d, 6), pats)


def test_invalid_sign_without_nonzero_and_padding_rejected():
    w = np.zeros((1, 12), np.int8)
    b = oracle.pack_bitplane(w)
    bad = b.copy()
    bad[0, 2 + 0] |= 4  # sign bit of k = 2 with its nonzero bit clear
    with pytest.raises(oracle.OracleError):
        oracle.unpack_bitplane(bad, 12)
    bad = b.copy()
    bad[0, 1] |= 0x80  # nonzero bit of k = 15, past K
    with pytest.raises(oracle.OracleError):
        oracle.unpack_bitplane(bad, 12)


def test_device_layout_positions_by_probe():
    """Bit 8j + i of pair p holds K = 32p + 4i + j: so (word >> i) & 0x01010101
    lines its four bytes up with the activation word at K = 32p + 4i."""
    K = 77
    fmt = oracle.FMT_BITPLANE
    used = oracle.device_row_bytes(fmt, K)
    assert used == 8 * math.ceil(K / 32)
    stride = 32
    base = oracle.pack_device(fmt, np.zeros((1, K), np.int8), stride)
    assert not base.any()
    for k in range(K):
        for v in (1, -1):
            w = np.zeros((1, K), np.int8)
            w[0, k] = v
            row = oracle.pack_device(fmt, w, stride)[0].view(np.uint32)
            p, i, j = k // 32, (k % 32) // 4, k % 4
            want = np.zeros_like(row)
            want[2 * p] = 1 << (8 * j + i)
            if v < 0:
                want[2 * p + 1] = 1 << (8 * j + i)
            np.testing.assert_array_equal(row, want)


def test_two_bits_per_weight_and_the_pages_figure():
    """Same bytes as the 2-bit format: 2 bits per trit, 27e9 x 2 / 8 = 6.75e9
    bytes for a 27B model (page pwwt.cn/news/5175886, section 1.1)."""
    for K in (5120, 17408):
        assert 8 * oracle.bitplane_row_bytes(K) / K == 2.0
        assert oracle.device_row_bytes(oracle.FMT_BITPLANE, K) == oracle.twobit_row_bytes(K)
    assert 27e9 * 8 * oracle.bitplane_row_bytes(5120) / 5120 / 8 == 6.75e9


def test_matches_the_trit_values():
    """n and s planes restore -1/0/+1: t = 1 + n - 2 n s (the digit of the
    other formats), checked on every trit of a seeded matrix."""
    w = synth.trits(22, 0, 7, 640)
    d = oracle.pack_device(oracle.FMT_BITPLANE, w, 160).view(np.uint32).reshape(7, -1)
    for k in range(640):
        p, i, j = k // 32, (k % 32) // 4, k % 4
        nb = (d[:, 2 * p] >> (8 * j + i)) & 1
        sb = (d[:, 2 * p + 1] >> (8 * j + i)) & 1
        np.testing.assert_array_equal(1 + nb.astype(int) - 2 * (nb & sb).astype(int), w[:, k] + 1)
