"""Pins of the oracle's block encoders (Q8_0, Q2_K, Q4_K) and its binary32 ->
binary16 rounding, each against something other than the encoder's own
formula: every binary16 code, numpy's conversion, blocks built so that the
encoder must return them byte for byte, brute-force nearest codes through the
(separately pinned) decoders, and closed-form special cases.

Sources: [QUANT] section 3 (the Q2_K writer: a scale and a min per 16-element
sub-block, 2-bit codes, the printed packing expression, d at byte 80, dmin
at 82) and [FLOW] "Dwarf Star の量子化の工夫" (Q8_0: one symmetric scale per
32 elements)."""
import numpy as np
import pytest

import oracle

K8, KQ = oracle.KIND_Q80, oracle.KIND_Q2K


# ----------------------------------------------------------------- binary16

def test_every_finite_f16_code_round_trips():
    for c in range(0x10000):
        if (c & 0x7C00) == 0x7C00:  # inf / nan
            continue
        assert oracle.f32_to_f16(np.float32(oracle.f16(c))) == c, hex(c)


def test_f32_to_f16_matches_numpy_on_random_floats():
    rng = np.random.default_rng(11)
    n = 100_000
    # all exponents from deep subnormal f16 to past the overflow threshold
    mant = rng.integers(0, 1 << 23, n, dtype=np.uint32)
    expo = rng.integers(127 - 30, 127 + 17, n, dtype=np.uint32)
    sign = rng.integers(0, 2, n, dtype=np.uint32) << 31
    f = (sign | (expo << 23) | mant).view(np.float32)
    with np.errstate(over="ignore"):
        ref = f.astype(np.float16).view(np.uint16)
    got = np.array([oracle.f32_to_f16(v) for v in f], dtype=np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(f[i]), hex(got[i]), hex(ref[i])) for i in bad[:5]]


def test_f32_to_f16_ties_and_limits():
    assert oracle.f32_to_f16(1.0 + 2.0 ** -11) == 0x3C00      # tie between 0x3c00 and 0x3c01: even
    assert oracle.f32_to_f16(1.0 + 3 * 2.0 ** -11) == 0x3C02  # tie between 0x3c01 and 0x3c02: even
    assert oracle.f32_to_f16(2.0 ** -25) == 0x0000            # half the smallest subnormal: even (zero)
    assert oracle.f32_to_f16(3 * 2.0 ** -25) == 0x0002
    assert oracle.f32_to_f16(2.0 ** -14 - 2.0 ** -25) == 0x0400  # rounds up into the normal range
    assert oracle.f32_to_f16(65504.0) == 0x7BFF
    assert oracle.f32_to_f16(np.nextafter(np.float32(65520.0), np.float32(0))) == 0x7BFF
    assert oracle.f32_to_f16(65520.0) == 0x7C00
    assert oracle.f32_to_f16(-np.inf) == 0xFC00
    assert oracle.f32_to_f16(-0.0) == 0x8000
    assert (oracle.f32_to_f16(np.nan) & 0x7C00) == 0x7C00 and (oracle.f32_to_f16(np.nan) & 0x3FF)


# --------------------------------------------------------------------- Q8_0

def _q80_block(dh: int, q: np.ndarray) -> np.ndarray:
    return np.concatenate([np.array([dh & 0xFF, dh >> 8], np.uint8), q.astype(np.int8).view(np.uint8)])


def test_q80_exact_blocks_come_back_byte_for_byte():
    """Values d*q with max |q| = 127: max|x|/127 is d exactly, so the encoder
    must return the same d and codes."""
    rng = np.random.default_rng(1)
    for trial in range(200):
        dh = int(rng.integers(0x0400, 0x7800))  # normal f16 scales
        q = rng.integers(-127, 128, 32)
        q[rng.integers(0, 32)] = 127 if trial % 2 else -127
        blk = _q80_block(dh, q)
        x = oracle.decode_row(K8, blk, 32).astype(np.float32)
        assert np.array_equal(x.astype(np.float64), oracle.decode_row(K8, blk, 32))  # exact in fp32
        assert np.array_equal(oracle.quantize(K8, x)[0], blk), trial


def test_q80_codes_are_nearest_and_span_127():
    rng = np.random.default_rng(2)
    cand = np.arange(-127, 128, dtype=np.float64)
    for scale in (1e-3, 0.02, 1.0, 300.0):
        x = (rng.standard_normal((20, 32)) * scale).astype(np.float32)
        blocks = oracle.quantize(K8, x)
        for b in range(20):
            d = oracle.f16(int(blocks[b, 0]) | int(blocks[b, 1]) << 8)
            q = blocks[b, 2:].view(np.int8).astype(np.float64)
            assert np.abs(q).max() == 127
            dist = np.abs(x[b][:, None].astype(np.float64) - d * cand[None, :])
            mine = np.abs(x[b].astype(np.float64) - d * q)
            assert np.all(mine <= dist.min(axis=1) * (1 + 1e-6) + 1e-300)


def test_q80_zero_and_nonfinite_blocks():
    assert not oracle.quantize(K8, np.zeros(32, np.float32)).any()
    x = np.zeros(64, np.float32)
    x[40] = np.inf
    with pytest.raises(ValueError):
        oracle.quantize(K8, x)


# --------------------------------------------------------------------- Q2_K

def _q2k_block(dh: int, mh: int, sc: np.ndarray, m: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """A block assembled from its fields with the printed packing expression
    (code of element j+l+32i at byte j/4 + l, shift 2i, j in {0, 128})."""
    blk = np.zeros(84, np.uint8)
    blk[:16] = sc | (m << 4)
    for j in (0, 128):
        for l in range(32):
            v = 0
            for i in range(4):
                v |= int(codes[j + l + 32 * i]) << (2 * i)
            blk[16 + j // 4 + l] = v
    blk[80], blk[81], blk[82], blk[83] = dh & 0xFF, dh >> 8, mh & 0xFF, mh >> 8
    return blk


def _short_f16(rng, lo_exp: int, hi_exp: int) -> int:
    """A binary16 scale with at most 3 significant bits (so every product and
    sum the encoder forms with it is exact in binary32)."""
    e = int(rng.integers(lo_exp, hi_exp))
    frac = int(rng.integers(0, 4)) << 8
    return ((e + 15) << 10) | frac


def test_q2k_exact_blocks_come_back_byte_for_byte():
    """Blocks whose every sub-block with a non-zero scale holds codes 0 and 3,
    with scale nibble 15 and min nibble 15 (or no mins) present: the range of
    each sub-block is exactly [-dmin*m, d*sc*3 - dmin*m], so the encoder must
    recover d, dmin, every nibble and every code."""
    rng = np.random.default_rng(3)
    for trial in range(300):
        dh = _short_f16(rng, -10, 4)
        with_min = trial % 3 != 0
        mh = _short_f16(rng, -10, 4) if with_min else 0
        sc = rng.integers(0, 16, 16)
        m = rng.integers(0, 16, 16) if with_min else np.zeros(16, np.int64)
        sc[rng.integers(0, 16)] = 15
        if with_min:
            m[rng.integers(0, 16)] = 15
        codes = rng.integers(0, 4, 256)
        for j in range(16):
            if sc[j] == 0:
                codes[16 * j:16 * j + 16] = 0
            else:
                p0, p3 = rng.choice(16, 2, replace=False)
                codes[16 * j + p0], codes[16 * j + p3] = 0, 3
        blk = _q2k_block(dh, mh, sc, m, codes)
        x64 = oracle.decode_row(KQ, blk, 256)
        x = x64.astype(np.float32)
        assert np.array_equal(x.astype(np.float64), x64)  # exact in fp32
        got = oracle.quantize(KQ, x)[0]
        assert np.array_equal(got, blk), (trial, np.nonzero(got != blk)[0][:8])


def _with_code(blk: np.ndarray, e: int, q: int) -> np.ndarray:
    b = blk.copy()
    byte, shift = 16 + 32 * (e // 128) + e % 32, 2 * ((e % 128) // 32)
    b[byte] = (int(b[byte]) & ~(3 << shift) & 0xFF) | (q << shift)
    return b


def test_q2k_codes_are_the_nearest_of_the_four():
    """Each element's code gives the decoded value nearest to the input among
    the block's four values for that sub-block (checked through the decoder,
    with the code replaced by each alternative)."""
    rng = np.random.default_rng(4)
    for scale, shift in ((1.0, 0.0), (0.05, 0.03), (10.0, -4.0)):
        x = (rng.standard_normal(256) * scale + shift).astype(np.float32)
        blk = oracle.quantize(KQ, x)[0]
        for e in range(0, 256, 3):
            vals = [oracle.q2k_elem(_with_code(blk, e, q), e) for q in range(4)]
            dist = np.abs(np.array(vals) - float(x[e]))
            assert dist[oracle.q2k_elem(blk, e) == np.array(vals)].min() <= dist.min() * (1 + 1e-5) + 1e-12, e


def test_q2k_widest_sub_block_takes_the_top_nibbles():
    rng = np.random.default_rng(5)
    for _ in range(50):
        x = (rng.standard_normal(256) * rng.uniform(0.01, 10)).astype(np.float32)
        blk = oracle.quantize(KQ, x)[0]
        assert (blk[:16] & 15).max() == 15  # the largest range/3 is d*15
        assert (blk[:16] >> 4).max() == 15  # some value is negative: the largest min is dmin*15


def test_q2k_error_on_gaussian_data():
    """Four levels over each 16-sample range: relative RMS error near the
    uniform-quantiser step/sqrt(12) ~ 0.34 (range ~3.5 sigma, step = range/3)."""
    rng = np.random.default_rng(6)
    x = rng.standard_normal(256 * 64).astype(np.float32)
    blocks = oracle.quantize(KQ, x)
    y = np.concatenate([oracle.decode_row(KQ, b, 256) for b in blocks])
    rel = np.sqrt(np.mean((x - y) ** 2)) / np.std(x)
    assert 0.2 < rel < 0.4, rel


def test_q2k_closed_forms():
    assert not oracle.quantize(KQ, np.zeros(256, np.float32)).any()
    for c in (0.75, 3.0e-3, 123.0):
        # constant c > 0: range [0, c], every code 3 at scale nibble 15, no min
        y = oracle.decode_row(KQ, oracle.quantize(KQ, np.full(256, c, np.float32))[0], 256)
        assert np.allclose(y, c, rtol=2.0 ** -10)
        # constant -c: no spread, all at the min: -dmin * 15
        blk = oracle.quantize(KQ, np.full(256, -c, np.float32))[0]
        assert np.all(blk[:16] & 15 == 0) and np.all(blk[:16] >> 4 == 15)
        assert np.allclose(oracle.decode_row(KQ, blk, 256), -c, rtol=2.0 ** -10)
    x = np.zeros(512, np.float32)
    x[300] = np.nan
    with pytest.raises(ValueError):
        oracle.quantize(KQ, x)


# --------------------------------------------------------------------- Q4_K

K4 = oracle.KIND_Q4K


def _q4k_block(dh: int, mh: int, sc, mn, codes) -> np.ndarray:
    from tests.test_oracle_q4k import _pack
    return _pack(dh, mh, sc, mn, codes)


def test_q4k_exact_blocks_come_back_byte_for_byte():
    """Sub-blocks with a non-zero scale hold codes 0 and 15, scale 63 and (when
    there are mins) min 63 occur, and d, dmin have 3 significant bits within
    a few binades of each other: every step the encoder takes is exact, so it
    must return the block it was given."""
    rng = np.random.default_rng(13)
    for trial in range(300):
        dh = _short_f16(rng, -8, -4)
        with_min = trial % 3 != 0
        mh = _short_f16(rng, -8, -4) if with_min else 0
        sc = rng.integers(0, 64, 8)
        m = rng.integers(0, 64, 8) if with_min else np.zeros(8, np.int64)
        sc[rng.integers(0, 8)] = 63
        if with_min:
            m[rng.integers(0, 8)] = 63
        codes = rng.integers(0, 16, 256)
        for j in range(8):
            if sc[j] == 0:
                codes[32 * j:32 * j + 32] = 0
            else:
                p0, p15 = rng.choice(32, 2, replace=False)
                codes[32 * j + p0], codes[32 * j + p15] = 0, 15
        blk = _q4k_block(dh, mh, sc, m, codes)
        x64 = oracle.decode_row(K4, blk, 256)
        x = x64.astype(np.float32)
        assert np.array_equal(x.astype(np.float64), x64)  # exact in fp32
        got = oracle.quantize(K4, x)[0]
        assert np.array_equal(got, blk), (trial, np.nonzero(got != blk)[0][:8])


def _with_q4k_code(blk: np.ndarray, e: int, q: int) -> np.ndarray:
    b = blk.copy()
    byte, shift = 16 + 32 * (e // 64) + e % 32, 4 * ((e % 64) // 32)
    b[byte] = (int(b[byte]) & ~(15 << shift) & 0xFF) | (q << shift)
    return b


def test_q4k_codes_are_the_nearest_of_the_sixteen():
    rng = np.random.default_rng(14)
    for scale, shift in ((1.0, 0.0), (0.05, 0.03), (10.0, -4.0)):
        x = (rng.standard_normal(256) * scale + shift).astype(np.float32)
        blk = oracle.quantize(K4, x)[0]
        for e in range(0, 256, 5):
            vals = np.array([oracle.q4k_elem(_with_q4k_code(blk, e, q), e) for q in range(16)])
            dist = np.abs(vals - float(x[e]))
            assert dist[oracle.q4k_elem(blk, e) == vals].min() <= dist.min() * (1 + 1e-5) + 1e-12, e


def test_q4k_widest_sub_block_takes_the_top_values_and_error_level():
    rng = np.random.default_rng(15)
    x = rng.standard_normal(256 * 64).astype(np.float32)
    blocks = oracle.quantize(K4, x)
    for blk in blocks[:50]:
        sc = [oracle.q4k_elem(_with_q4k_code(blk, 32 * j, 1), 32 * j) - oracle.q4k_elem(_with_q4k_code(blk, 32 * j, 0),
                                                                                      32 * j) for j in range(8)]
        d = oracle.f16(int(blk[0]) | int(blk[1]) << 8)
        assert round(max(sc) / d) == 63  # the widest range/15 is d*63
    y = np.concatenate([oracle.decode_row(K4, b, 256) for b in blocks])
    rel = np.sqrt(np.mean((x - y) ** 2)) / np.std(x)
    assert 0.05 < rel < 0.11, rel  # 16 levels over ~4.1 sigma: step/sqrt(12) ~ 0.079


def test_q4k_closed_forms():
    assert not oracle.quantize(K4, np.zeros(256, np.float32)).any()
    # constants whose base c/945 (codes 15 at scale 63) is a normal binary16,
    # so the only rounding is d's 11 significant bits
    for c in (0.75, 0.1, 123.0):
        y = oracle.decode_row(K4, oracle.quantize(K4, np.full(256, c, np.float32))[0], 256)
        assert np.allclose(y, c, rtol=2.0 ** -10)
        y = oracle.decode_row(K4, oracle.quantize(K4, np.full(256, -c, np.float32))[0], 256)
        assert np.allclose(y, -c, rtol=2.0 ** -10)
    x = np.zeros(512, np.float32)
    x[300] = np.inf
    with pytest.raises(ValueError):
        oracle.quantize(K4, x)
