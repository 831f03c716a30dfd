"""Hand-built packed blocks for the pins.

These encoders place fields where the format descriptions put them (see the
oracle's header for the sources and readings).  The Q2_K code packing uses
the expression printed in the ds4 quantizer walk-through: byte j/4 + l of qs
holds codes L[j+l], L[j+l+32], L[j+l+64], L[j+l+96] at shifts 0, 2, 4, 6 for
j in {0, 128}, l in 0..31.
"""
import numpy as np


def f16_bits(v: float) -> int:
    return int(np.array(v, dtype=np.float16).view(np.uint16))


def q2k_block(codes, scale_nib, min_nib, d: float, dmin: float) -> np.ndarray:
    """codes: 256 ints in 0..3; scale_nib/min_nib: 16 ints in 0..15."""
    L = np.asarray(codes, dtype=np.int64)
    blk = np.zeros(84, dtype=np.uint8)
    for j in (0, 128):
        for l in range(32):
            blk[16 + j // 4 + l] = (L[j + l] | (L[j + l + 32] << 2) | (L[j + l + 64] << 4) | (L[j + l + 96] << 6))
    for s in range(16):
        blk[s] = (int(scale_nib[s]) & 0xF) | ((int(min_nib[s]) & 0xF) << 4)
    b = f16_bits(d)
    blk[80], blk[81] = b & 0xFF, b >> 8
    b = f16_bits(dmin)
    blk[82], blk[83] = b & 0xFF, b >> 8
    return blk


def iq2xxs_block(d: float, groups) -> np.ndarray:
    """groups: 8 tuples (indices[4], masks7[4], scale_nibble)."""
    blk = np.zeros(66, dtype=np.uint8)
    b = f16_bits(d)
    blk[0], blk[1] = b & 0xFF, b >> 8
    for g, (indices, masks, s) in enumerate(groups):
        base = 2 + 8 * g
        for j in range(4):
            blk[base + j] = indices[j]
        S = 0
        for j in range(4):
            S |= (int(masks[j]) & 0x7F) << (7 * j)
        S |= (int(s) & 0xF) << 28
        for i in range(4):
            blk[base + 4 + i] = (S >> (8 * i)) & 0xFF
    return blk


def q80_block(d: float, q) -> np.ndarray:
    blk = np.zeros(34, dtype=np.uint8)
    b = f16_bits(d)
    blk[0], blk[1] = b & 0xFF, b >> 8
    blk[2:] = np.asarray(q, dtype=np.int8).view(np.uint8)
    return blk


def constant_iq2_rows(rows: int, cols: int, d: float, s: int, index: int = 0) -> np.ndarray:
    """Every element = d * (0.5 + s)/4 * grid[index][l], no negative signs."""
    blk = iq2xxs_block(d, [([index] * 4, [0] * 4, s)] * 8)
    return np.tile(blk, (rows, cols // 256))


def constant_q2k_rows(rows: int, cols: int, q: int, sc: int, mn: int, d: float, dmin: float) -> np.ndarray:
    blk = q2k_block([q] * 256, [sc] * 16, [mn] * 16, d, dmin)
    return np.tile(blk, (rows, cols // 256))


def constant_q80_rows(rows: int, cols: int, d: float, q: int) -> np.ndarray:
    blk = q80_block(d, [q] * 32)
    return np.tile(blk, (rows, cols // 32))
