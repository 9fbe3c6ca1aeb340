"""Pins of the oracle's bit layouts (hand-worked positions, bijection,
round trips, and the tensor-core fragment semantics the fragment layouts are
built for). No GPU needed."""

import os

import numpy as np
import pytest

import oracle
from oracle import LAYOUT_CANONICAL, LAYOUT_FRAG_K, LAYOUT_FRAG_V

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
NAMES = {"canonical": LAYOUT_CANONICAL, "fragk": LAYOUT_FRAG_K, "fragv": LAYOUT_FRAG_V}


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
    assert len(rows) >= 25
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
                                           (LAYOUT_FRAG_K, 1, 300), (LAYOUT_FRAG_V, 1, 300)])
def test_positions_are_a_bijection_onto_the_row(layout, bits, n):
    d = 128
    ii, jj = np.meshgrid(np.arange(n), np.arange(d), indexing="ij")
    byte, bit = oracle.bit_position(layout, ii, jj, n, d, bits)
    flat = (byte * 8 + bit).ravel()
    assert len(np.unique(flat)) == n * d
    nbytes = oracle.codes_nbytes(layout, n, d, bits)
    assert flat.min() >= 0 and flat.max() < nbytes * 8
    # padding bits of the fragment layouts are exactly the unused tail
    assert nbytes * 8 == oracle.padded_tokens(layout, n) * d * bits


@pytest.mark.parametrize("layout,bits,n", [(LAYOUT_CANONICAL, 1, 77), (LAYOUT_CANONICAL, 2, 33),
                                           (LAYOUT_CANONICAL, 8, 11), (LAYOUT_FRAG_K, 1, 257),
                                           (LAYOUT_FRAG_V, 1, 513)])
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


def _mma_a_element(lane, reg, byte):
    """(row, col) of an m16n8k32 8-bit A-fragment element (PTX fragment table)."""
    g, t = lane >> 2, lane & 3
    return g + 8 * (reg & 1), 4 * t + byte + 16 * (reg >> 1)


def _mma_b_element(lane, reg, byte):
    """(k_row, col) of an m16n8k32 8-bit B-fragment element (PTX fragment table)."""
    g, t = lane >> 2, lane & 3
    return 4 * t + byte + 16 * reg, g


def test_frag_k_is_the_a_fragment_of_bit_sliced_token_octets():
    """Lane L's 16 bytes of chunk c are its four A registers for the MMA that
    covers channels 32c..32c+31; masking bit k of every byte selects, in MMA
    row r, token 8r + k of the 128-token tile."""
    for c in range(4):
        for lane in range(32):
            for reg in range(4):
                for byte in range(4):
                    row, col = _mma_a_element(lane, reg, byte)
                    for k in range(8):
                        token, channel = 8 * row + k, 32 * c + col
                        got = oracle.bit_position(LAYOUT_FRAG_K, token, channel, 128, 128, 1)
                        want = (c * 512 + lane * 16 + reg * 4 + byte, k)
                        assert (int(got[0]), int(got[1])) == want


def test_frag_v_is_the_b_fragment_of_channel_token_octets():
    """Request q's 16 bytes of lane L hold the two B registers of channel tiles
    2q and 2q+1; bit k of byte i in register r is token 8(4t+i+16r) + k of
    the 256-token tile, channel 8*tile + g."""
    for q in range(8):
        for e in range(2):
            for lane in range(32):
                for reg in range(2):
                    for byte in range(4):
                        krow, col = _mma_b_element(lane, reg, byte)
                        for k in range(8):
                            token, channel = 8 * krow + k, 8 * (2 * q + e) + col
                            got = oracle.bit_position(LAYOUT_FRAG_V, token, channel, 256, 128, 1)
                            want = (q * 512 + lane * 16 + (2 * e + reg) * 4 + byte, k)
                            assert (int(got[0]), int(got[1])) == want


def test_layout_arguments_are_checked():
    with pytest.raises(ValueError):
        oracle.codes_nbytes(LAYOUT_FRAG_K, 10, 128, 2)
    with pytest.raises(ValueError):
        oracle.codes_nbytes(LAYOUT_FRAG_V, 10, 64, 1)
    with pytest.raises(ValueError):
        oracle.codes_nbytes(7, 10, 128, 1)
