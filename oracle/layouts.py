"""Bit layouts of the packed code cache, written from their documented formulas.

TEST INFRASTRUCTURE ONLY (see the package docstring). The article stores only
the b-bit integers (Method 2); how they are packed is this library's choice,
documented in ``include/calibq.h``. Three layouts exist; for each, this module
maps every (token i, channel j) of one (batch, head) row to a (byte, bit)
position and packs / unpacks with that map, one bit at a time.

* canonical (any b, d*b a multiple of 32): token-major. Token i occupies
  d*b/8 consecutive bytes; channel j's code sits at bits [j*b, j*b + b) of the
  token's little-endian bit string, i.e. byte (j*b) // 8, bits (j*b) % 8 ...

* octet-K (b in {1, 2, 4, 8}, d = 128): one byte per (P = 8/b consecutive
  tokens, channel). Token i, channel j:
      byte = (i // P) * 128 + j,   bit = (i % P) * b.
  Row bytes = ceil(n / P) * 128. (b = 1: byte (i >> 3) * 128 + j, bit i & 7.)

* octet-V (b in {1, 2, 4, 8}, d = 128): the same bytes transposed per tile of
  32 P tokens. Token i, channel j:
      byte = (i // (32 P)) * 4096 + j * 32 + (i % (32 P)) // P,   bit = (i % P) * b.
  Row bytes = ceil(n / (32 P)) * 4096. (b = 1: 256-token tiles.)

Tokens past n in the last byte group / tile are padding and hold code 0.
"""

from __future__ import annotations

import numpy as np

LAYOUT_CANONICAL = 0
LAYOUT_OCTET_K = 1
LAYOUT_OCTET_V = 2

def _per_byte(bits: int) -> int:
    """Tokens sharing one byte of an octet layout."""
    return 8 // bits


def _tile(layout: int, bits: int) -> int:
    """Tokens of one padding unit: a byte group (octet-K) or a tile (octet-V)."""
    return _per_byte(bits) * (32 if layout == LAYOUT_OCTET_V else 1)


def _check(layout: int, d: int, bits: int):
    if layout == LAYOUT_CANONICAL:
        if (d * bits) % 32:
            raise ValueError("canonical layout needs d*bits to be a multiple of 32")
    elif layout in (LAYOUT_OCTET_K, LAYOUT_OCTET_V):
        if bits not in (1, 2, 4, 8) or d != 128:
            raise ValueError("octet layouts are defined for bits in {1, 2, 4, 8}, d=128")
    else:
        raise ValueError(f"unknown layout {layout}")


def padded_tokens(layout: int, n: int, bits: int = 1) -> int:
    """Tokens stored per row: n, or n rounded up to the layout's padding unit."""
    if layout == LAYOUT_CANONICAL:
        return n
    t = _tile(layout, bits)
    return -(-n // t) * t


def codes_nbytes(layout: int, n: int, d: int, bits: int) -> int:
    """Bytes of one (batch, head) row of packed codes."""
    _check(layout, d, bits)
    return padded_tokens(layout, n, bits) * d * bits // 8


def bit_position(layout: int, i, j, n: int, d: int, bits: int):
    """(byte, bit) of the lowest code bit of token i, channel j within a row.

    i, j may be integer arrays (broadcast together).
    """
    _check(layout, d, bits)
    i = np.asarray(i, dtype=np.int64)
    j = np.asarray(j, dtype=np.int64)
    if layout == LAYOUT_CANONICAL:
        row = d * bits // 8
        pos = j * bits
        return i * row + pos // 8, pos % 8
    p = _per_byte(bits)
    if layout == LAYOUT_OCTET_K:
        return (i // p) * 128 + j, (i % p) * bits
    # LAYOUT_OCTET_V
    tile = 32 * p
    return (i // tile) * 4096 + j * 32 + (i % tile) // p, (i % p) * bits


def pack_codes(codes, layout: int, bits: int) -> np.ndarray:
    """Pack int codes ``[B, H, n, d]`` into uint8 ``[B, H, row_bytes]``."""
    codes = np.asarray(codes, dtype=np.int64)
    B, H, n, d = codes.shape
    if codes.size and (codes.min() < 0 or codes.max() > (1 << bits) - 1):
        raise ValueError("code out of range")
    nbytes = codes_nbytes(layout, n, d, bits)
    ii, jj = np.meshgrid(np.arange(n), np.arange(d), indexing="ij")
    byte, bit = bit_position(layout, ii, jj, n, d, bits)
    # Every (token, channel) owns distinct bits, so OR-ing the shifted codes
    # into their bytes is the same as adding them; bincount does the adding.
    rows = np.arange(B * H, dtype=np.int64)[:, None] * nbytes
    index = (rows + byte.ravel()[None, :]).ravel()
    weight = (codes.reshape(B * H, n * d) << bit.ravel()[None, :]).ravel()
    flat = np.bincount(index, weights=weight.astype(np.float64), minlength=B * H * nbytes)
    if flat.size and flat.max() > 255:
        raise AssertionError("two codes were mapped onto the same bits")
    return flat.astype(np.uint8).reshape(B, H, nbytes)


def unpack_codes(packed, layout: int, n: int, d: int, bits: int) -> np.ndarray:
    """Inverse of ``pack_codes``: uint8 ``[B, H, row_bytes]`` -> int64 ``[B, H, n, d]``."""
    packed = np.asarray(packed, dtype=np.uint8)
    B, H, nbytes = packed.shape
    if nbytes != codes_nbytes(layout, n, d, bits):
        raise ValueError("packed row size does not match the layout")
    ii, jj = np.meshgrid(np.arange(n), np.arange(d), indexing="ij")
    byte, bit = bit_position(layout, ii, jj, n, d, bits)
    vals = packed[:, :, byte].astype(np.int64)  # [B, H, n, d]
    return (vals >> bit) & ((1 << bits) - 1)
