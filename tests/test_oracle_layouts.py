"""Pins of the oracle's bit layouts (hand-worked positions, bijection,
round trips, and the tensor-memory operand semantics the octet layouts are
built for). No GPU needed."""

import os

import numpy as np
import pytest

import oracle
from oracle import LAYOUT_CANONICAL, LAYOUT_OCTET_K, LAYOUT_OCTET_V

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
NAMES = {"canonical": LAYOUT_CANONICAL, "octetk": LAYOUT_OCTET_K, "octetv": LAYOUT_OCTET_V}


def _rows():
    out = []
    with open(os.path.join(GOLDEN, "layout_positions.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                name, bits, d, i, j, byte, bit = line.split()
                out.append((NAMES[name], int(bits), int(d), int(i), int(j), int(byte), int(bit)))
    return out


def test_hand_worked_positions():
    rows = _rows()
    assert len(rows) >= 32
    for layout, bits, d, i, j, byte, bit in rows:
        n = i + 1
        got = oracle.bit_position(layout, i, j, n, d, bits)
        assert (int(got[0]), int(got[1])) == (byte, bit), (layout, i, j)
        # a lone code of 1 sets exactly that bit
        codes = np.zeros((1, 1, n, d), dtype=np.int64)
        codes[0, 0, i, j] = 1
        packed = oracle.pack_codes(codes, layout, bits)[0, 0]
        nz = np.flatnonzero(packed)
        assert list(nz) == [byte] and packed[byte] == (1 << bit)


@pytest.mark.parametrize("layout,bits,n", [(LAYOUT_CANONICAL, 1, 37), (LAYOUT_CANONICAL, 2, 5),
                                           (LAYOUT_CANONICAL, 4, 9), (LAYOUT_CANONICAL, 8, 3),
                                           (LAYOUT_OCTET_K, 1, 300), (LAYOUT_OCTET_V, 1, 300),
                                           (LAYOUT_OCTET_K, 2, 301), (LAYOUT_OCTET_V, 2, 301),
                                           (LAYOUT_OCTET_K, 4, 99), (LAYOUT_OCTET_V, 4, 99),
                                           (LAYOUT_OCTET_K, 8, 45), (LAYOUT_OCTET_V, 8, 45)])
def test_positions_are_a_bijection_onto_the_row(layout, bits, n):
    d = 128
    ii, jj = np.meshgrid(np.arange(n), np.arange(d), indexing="ij")
    byte, bit = oracle.bit_position(layout, ii, jj, n, d, bits)
    flat = (byte * 8 + bit).ravel()
    assert len(np.unique(flat)) == n * d
    nbytes = oracle.codes_nbytes(layout, n, d, bits)
    assert flat.min() >= 0 and flat.max() < nbytes * 8
    # padding bits of the octet layouts are exactly the unused tail
    assert nbytes * 8 == oracle.padded_tokens(layout, n, bits) * d * bits


@pytest.mark.parametrize("layout,bits,n", [(LAYOUT_CANONICAL, 1, 77), (LAYOUT_CANONICAL, 2, 33),
                                           (LAYOUT_CANONICAL, 8, 11), (LAYOUT_OCTET_K, 1, 257),
                                           (LAYOUT_OCTET_V, 1, 513), (LAYOUT_OCTET_K, 2, 130),
                                           (LAYOUT_OCTET_V, 4, 200), (LAYOUT_OCTET_K, 8, 33),
                                           (LAYOUT_OCTET_V, 8, 70)])
def test_pack_unpack_round_trip(layout, bits, n):
    rng = np.random.default_rng(n)
    codes = rng.integers(0, 1 << bits, size=(2, 3, n, 128))
    packed = oracle.pack_codes(codes, layout, bits)
    assert packed.shape == (2, 3, oracle.codes_nbytes(layout, n, 128, bits))
    assert np.array_equal(oracle.unpack_codes(packed, layout, n, 128, bits), codes)


def test_canonical_matches_little_endian_u32_words():
    """channel j at bit (j*b mod 32) of u32 word floor(j*b/32), little-endian."""
    rng = np.random.default_rng(1)
    for bits in (1, 2, 4, 8):
        codes = rng.integers(0, 1 << bits, size=(1, 1, 3, 128))
        words = oracle.pack_codes(codes, LAYOUT_CANONICAL, bits)[0, 0].view("<u4").reshape(3, -1)
        for i in range(3):
            for j in range(128):
                w = int(words[i, (j * bits) // 32])
                assert (w >> ((j * bits) % 32)) & ((1 << bits) - 1) == codes[0, 0, i, j]


def test_octet_k_rows_are_tensor_memory_a_rows():
    """K side: tensor-memory lane m of a 1024-token tile holds token octet m
    (128 bytes). In the MMA for bit k and 32-channel chunk c, A element
    (row m, K index kk) is bit k of byte 32c + kk of that lane, i.e. the code of
    token 8m + k, channel 32c + kk -- read from the 32-bit word 8c + kk // 4 of
    the lane at byte kk % 4."""
    for tile in range(2):
        for m in range(128):
            for c in range(4):
                for kk in range(32):
                    word, byte = 8 * c + kk // 4, kk % 4
                    for k in (0, 3, 7):
                        token, channel = 1024 * tile + 8 * m + k, 32 * c + kk
                        got = oracle.bit_position(LAYOUT_OCTET_K, token, channel, 2048, 128, 1)
                        want = ((1024 * tile) // 8 * 128 + m * 128 + 4 * word + byte, k)
                        assert (int(got[0]), int(got[1])) == want


def test_octet_v_rows_are_tensor_memory_a_rows():
    """V side: lane j of a 256-token tile holds channel j's 32 bytes; in the
    MMA for bit k, A element (row j, K index kk) is bit k of byte kk, i.e. the
    code of token 8 kk + k -- word kk // 4 of the lane, byte kk % 4."""
    for tile in range(2):
        for j in range(128):
            for kk in range(32):
                for k in range(8):
                    token = 256 * tile + 8 * kk + k
                    got = oracle.bit_position(LAYOUT_OCTET_V, token, j, 512, 128, 1)
                    want = (4096 * tile + 32 * j + 4 * (kk // 4) + kk % 4, k)
                    assert (int(got[0]), int(got[1])) == want


def test_octet_sub_positions_are_tensor_operand_values():
    """b bits: masking sub-position k of every byte ((2^b - 1) << k b) gives the
    8-bit operand "code of token P m + k times 2^(k b)" for byte group m, and
    (2^b - 1) << k b never exceeds 255."""
    for bits in (2, 4, 8):
        p = 8 // bits
        rng = np.random.default_rng(bits)
        n = 4 * p
        codes = rng.integers(0, 1 << bits, size=(1, 1, n, 128))
        packed = oracle.pack_codes(codes, LAYOUT_OCTET_K, bits)[0, 0].reshape(-1, 128)
        for m in range(n // p):
            for k in range(p):
                mask = ((1 << bits) - 1) << (k * bits)
                assert mask <= 255
                assert np.array_equal(packed[m] & mask, codes[0, 0, p * m + k] << (k * bits))


def test_layout_arguments_are_checked():
    with pytest.raises(ValueError):
        oracle.codes_nbytes(LAYOUT_OCTET_K, 10, 128, 3)
    with pytest.raises(ValueError):
        oracle.codes_nbytes(LAYOUT_OCTET_V, 10, 64, 1)
    with pytest.raises(ValueError):
        oracle.codes_nbytes(7, 10, 128, 1)
