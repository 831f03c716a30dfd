"""The seeded input generator: determinism, distributions, thread-count
invariance and the f16 rounding it uses for block scales."""
import numpy as np
import pytest

import synth


def test_f16_rounding_matches_numpy_round_to_nearest_even():
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.uniform(-70000, 70000, 2000), rng.uniform(-1e-4, 1e-4, 2000),
                           rng.uniform(0.001, 0.02, 2000), [0.0, -0.0, 65504.0, 65519.9, 65520.0, 6e-8, 3e-8,
                                                             2.9802322e-08, 5.96e-8, 1e-9]]).astype(np.float32)
    lib = synth._hostlib()
    got = np.array([lib.synth_f16_of(float(v)) for v in vals], dtype=np.uint16)
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


def test_routed_fill_is_deterministic_and_thread_invariant():
    a = synth.routed(7, 3, synth.T_GATE, synth.KIND_IQ2XXS, 2, 3, 64, 512)
    lib = synth._hostlib()
    b = np.empty_like(a)
    lib.synth_fill_routed(7, 3, synth.T_GATE, synth.KIND_IQ2XXS, 2, 3, 64, 512, b.ctypes.data, 1)
    assert np.array_equal(a, b)
    # a sub-range equals the same experts taken from a wider fill
    c = synth.routed(7, 3, synth.T_GATE, synth.KIND_IQ2XXS, 0, 6, 64, 512)
    assert np.array_equal(c[2:5], a)
    # another layer or tensor gives other bytes
    d = synth.routed(7, 4, synth.T_GATE, synth.KIND_IQ2XXS, 2, 3, 64, 512)
    assert not np.array_equal(a, d)


def test_block_field_distributions():
    W = synth.routed(1, 0, synth.T_GATE, synth.KIND_IQ2XXS, 0, 1, 256, 4096)[0].reshape(-1, 66)
    d = W[:, 0:2].copy().view(np.float16).astype(np.float64).ravel()
    assert d.min() >= 0.005 - 1e-5 and d.max() <= 0.02 + 1e-5
    idx = W[:, 2:].reshape(-1, 8, 8)[:, :, :4].ravel()
    assert idx.min() == 0 and idx.max() == 255
    S = W[:, 2:].reshape(-1, 8, 8)[:, :, 4:].copy().view("<u4").ravel()
    s = S >> 28
    assert set(np.unique(s).tolist()) == set(range(16))
    Q = synth.routed(1, 0, synth.T_DOWN, synth.KIND_Q2K, 0, 1, 256, 2048)[0].reshape(-1, 84)
    for off in (80, 82):
        v = Q[:, off:off + 2].copy().view(np.float16).astype(np.float64).ravel()
        assert v.min() >= 0.001 - 1e-5 and v.max() <= 0.01 + 1e-5
    S8 = synth.shared(1, 0, synth.T_SH_UP, 64, 4096).reshape(-1, 34)
    q = S8[:, 2:].copy().view(np.int8)
    assert q.min() == -127 and q.max() == 127
    assert np.all(S8[:, 0:2].copy().view(np.float16) == np.float16(0.0005))


def test_q4k_block_fields():
    """Q4_K blocks: f16 d and dmin in [0.0001, 0.001], raw scale/min and code
    bytes (every byte value occurs), deterministic and thread-invariant."""
    W = synth.routed(2, 40, synth.T_DOWN, synth.KIND_Q4K, 0, 1, 512, 2048)[0].reshape(-1, 144)
    for off in (0, 2):
        v = W[:, off:off + 2].copy().view(np.float16).astype(np.float64).ravel()
        assert v.min() >= 0.0001 - 1e-7 and v.max() <= 0.001 + 1e-6
    for lo, hi in ((4, 16), (16, 144)):
        assert np.unique(W[:, lo:hi]).size == 256
    lib = synth._hostlib()
    a = synth.routed(2, 40, synth.T_GATE, synth.KIND_Q4K, 3, 2, 64, 512)
    b = np.empty_like(a)
    lib.synth_fill_routed(2, 40, synth.T_GATE, synth.KIND_Q4K, 3, 2, 64, 512, b.ctypes.data, 1)
    assert np.array_equal(a, b)
    assert np.array_equal(synth.routed(2, 40, synth.T_GATE, synth.KIND_Q4K, 0, 5, 64, 512)[3:5], a)


def test_grid_bias_and_hash_table():
    g = synth.grid(0)
    assert g.shape == (256, 8) and set(np.unique(g).tolist()) == {8, 25, 43}
    b = synth.bias(0, 0, 256, False)
    assert b.min() >= -0.1 and b.max() < 0.1
    bs = synth.bias(0, 0, 256, True)
    assert np.array_equal(bs[0::8], b[0::8] + np.float32(0.5))
    assert np.array_equal(np.delete(bs, np.s_[0::8]), np.delete(b, np.s_[0::8]))
    tab = synth.tid2eid(0, 1, 5000, 256, 6)
    assert tab.min() >= 0 and tab.max() < 256
    assert all(len(set(r)) == 6 for r in tab.tolist())


def test_gaussian_inputs_are_seeded():
    a = synth.activations(3, 4, 256)
    assert np.array_equal(a, synth.activations(3, 4, 256))
    assert a.dtype == np.float32 and abs(float(a.std()) - 1) < 0.1
    w = synth.router_weight(3, 5, 16, 256)
    assert w.dtype == np.float16 and abs(float(w.astype(np.float64).std()) - 0.02) < 0.002


@pytest.mark.gpu
def test_device_fill_is_byte_identical_to_host_fill():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    for kind, tensor, rows, cols in ((synth.KIND_IQ2XXS, synth.T_GATE, 64, 4096),
                                     (synth.KIND_Q2K, synth.T_DOWN, 64, 2048),
                                     (synth.KIND_Q80, synth.T_SH_UP, 64, 4096)):
        host = synth.routed(3, 5, tensor, kind, 7, 2, rows, cols)
        dev = torch.empty(host.shape, dtype=torch.uint8, device="cuda")
        synth.device_routed(dev, 3, 5, tensor, kind, 7, 2, rows, cols)
        torch.cuda.synchronize()
        assert np.array_equal(dev.cpu().numpy(), host)
