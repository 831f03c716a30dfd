"""Parity of the device block encoders (moe_quantize, through the C ABI:
Q8_0, Q2_K, Q4_K) with the oracle's encoders: every output byte equal (the codes are integer
decisions taken in binary32 on both sides), on random data over many scales,
blocks built to round-trip exactly, extreme magnitudes, block counts that
leave a ragged last CTA, a full 2048 x 4096 matrix, and blocks holding
non-finite values (written as zeros and counted)."""
import numpy as np
import pytest

import oracle
from tests.test_oracle_q4k import _pack as _q4k_block
from tests.test_oracle_quant import _q2k_block, _short_f16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


@pytest.fixture(scope="module")
def moe():
    from bit_moe_expert_sqrtsoftplus_b200 import build
    build.build()
    import bit_moe_expert_sqrtsoftplus_b200 as m
    return m


def _fmt(moe, kind):
    return {oracle.KIND_Q80: moe.MOE_QUANT_Q8_0, oracle.KIND_Q2K: moe.MOE_QUANT_Q2_K,
            oracle.KIND_Q4K: moe.MOE_QUANT_Q4_K}[kind]


KINDS = [oracle.KIND_Q80, oracle.KIND_Q2K, oracle.KIND_Q4K]


def _device(moe, kind, x: np.ndarray):
    out, bad = moe.quantize(_fmt(moe, kind), torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda())
    torch.cuda.synchronize()
    return out.cpu().numpy(), int(bad.item())


def _random_values(rng, n):
    """Gaussian blocks at scales from 1e-6 to 1e4, with offsets, plus a few
    all-positive, all-negative, zero and constant stretches."""
    x = rng.standard_normal(n)
    per = 256
    for b in range(n // per):
        s = 10.0 ** rng.uniform(-6, 4)
        kind = b % 7
        seg = slice(b * per, (b + 1) * per)
        if kind == 0:
            x[seg] = np.abs(x[seg]) * s
        elif kind == 1:
            x[seg] = -np.abs(x[seg]) * s
        elif kind == 2:
            x[seg] = 0.0
        elif kind == 3:
            x[seg] = s
        else:
            x[seg] = x[seg] * s + rng.uniform(-2, 2) * s
    return x.astype(np.float32)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("nblocks_q2k", [1, 37, 1000])
def test_random_blocks_bit_exact(moe, kind, nblocks_q2k):
    rng = np.random.default_rng(nblocks_q2k * 10 + kind)
    x = _random_values(rng, 256 * nblocks_q2k)
    got, bad = _device(moe, kind, x)
    ref = oracle.quantize(kind, x)
    assert bad == 0
    diff = np.nonzero((got != ref).any(axis=1))[0]
    assert diff.size == 0, (diff[:5], got[diff[0]] if diff.size else None, ref[diff[0]] if diff.size else None)


def test_constructed_q2k_blocks_round_trip(moe):
    rng = np.random.default_rng(21)
    blocks, xs = [], []
    for trial in range(64):
        dh = _short_f16(rng, -10, 4)
        mh = _short_f16(rng, -10, 4) if trial % 3 else 0
        sc = rng.integers(0, 16, 16)
        m = rng.integers(0, 16, 16) if mh else np.zeros(16, np.int64)
        sc[rng.integers(0, 16)] = 15
        if mh:
            m[rng.integers(0, 16)] = 15
        codes = rng.integers(0, 4, 256)
        for j in range(16):
            if sc[j] == 0:
                codes[16 * j:16 * j + 16] = 0
            else:
                p0, p3 = rng.choice(16, 2, replace=False)
                codes[16 * j + p0], codes[16 * j + p3] = 0, 3
        blk = _q2k_block(dh, mh, sc, m, codes)
        blocks.append(blk)
        xs.append(oracle.decode_row(oracle.KIND_Q2K, blk, 256).astype(np.float32))
    got, _ = _device(moe, oracle.KIND_Q2K, np.concatenate(xs))
    assert np.array_equal(got, np.stack(blocks))


def test_constructed_q4k_blocks_round_trip(moe):
    rng = np.random.default_rng(25)
    blocks, xs = [], []
    for trial in range(64):
        dh = _short_f16(rng, -8, -4)
        mh = _short_f16(rng, -8, -4) if trial % 3 else 0
        sc = rng.integers(0, 64, 8)
        m = rng.integers(0, 64, 8) if mh else np.zeros(8, np.int64)
        sc[rng.integers(0, 8)] = 63
        if mh:
            m[rng.integers(0, 8)] = 63
        codes = rng.integers(0, 16, 256)
        for j in range(8):
            if sc[j] == 0:
                codes[32 * j:32 * j + 32] = 0
            else:
                p0, p15 = rng.choice(32, 2, replace=False)
                codes[32 * j + p0], codes[32 * j + p15] = 0, 15
        blk = _q4k_block(dh, mh, sc, m, codes)
        blocks.append(blk)
        xs.append(oracle.decode_row(oracle.KIND_Q4K, blk, 256).astype(np.float32))
    got, _ = _device(moe, oracle.KIND_Q4K, np.concatenate(xs))
    assert np.array_equal(got, np.stack(blocks))


def test_extreme_magnitudes_bit_exact(moe):
    """Scales that overflow binary16 (infinite d) or underflow it (zero d),
    and subnormal d, on both encoders."""
    rng = np.random.default_rng(22)
    parts = [rng.standard_normal(256) * s for s in (1e7, 3e5, 1e-9, 3e-6, 6e-8, 1.0)]
    x = np.concatenate(parts).astype(np.float32)
    for kind in KINDS:
        got, bad = _device(moe, kind, x)
        assert bad == 0
        assert np.array_equal(got, oracle.quantize(kind, x)), kind


def test_full_matrix_bit_exact(moe):
    """A 2048 x 4096 matrix (the shape of one routed gate or up projection)."""
    rng = np.random.default_rng(23)
    x = (rng.standard_normal((2048, 4096)) * 0.02).astype(np.float32)
    for kind in KINDS:
        got, _ = _device(moe, kind, x)
        assert np.array_equal(got, oracle.quantize(kind, x)), kind


def test_nonfinite_blocks_are_zeroed_and_counted(moe):
    rng = np.random.default_rng(24)
    x = rng.standard_normal(256 * 12).astype(np.float32)
    x[5] = np.nan              # Q2_K block 0, Q8_0 block 0
    x[256 * 3 + 200] = np.inf  # Q2_K block 3, Q8_0 block 30
    x[256 * 7 + 1] = -np.inf   # Q2_K block 7, Q8_0 block 56
    for kind, per, hit in ((oracle.KIND_Q80, 32, [0, 30, 56]), (oracle.KIND_Q2K, 256, [0, 3, 7]),
                           (oracle.KIND_Q4K, 256, [0, 3, 7])):
        got, bad = _device(moe, kind, x)
        assert bad == len(hit)
        assert not got[hit].any()
        keep = [b for b in range(x.size // per) if b not in hit]
        ref = np.stack([oracle.quantize(kind, x[b * per:(b + 1) * per])[0] for b in keep])
        assert np.array_equal(got[keep], ref), kind
