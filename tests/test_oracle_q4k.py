"""Pins of the oracle's Q4_K decoder (the routed-expert format of the q2-q4
build's upgraded layers) and of the layer with Q4_K experts.

Sources: [QUANT] section 3 type table (q4_K: 256 values in 144 bytes);
[FLOW] format paragraph (K-quants are affine with a scale and a min per
sub-block) and the bit-width table after "パラメータはどこにあるか: 層別の内訳"
(Q4_K about 4.5 bpw, about 3.6 GB per routed layer; raising one layer from q2
to Q4_K costs about 1.8 GB).  The byte layout is a reading (the public GGUF
block; see oracle.c), so the hand-built blocks below pin the decoder to that
reading, not to real files."""
import numpy as np

import oracle

K4 = oracle.KIND_Q4K


def test_page_figures():
    assert oracle._BB[K4] * 8 / oracle._BE[K4] == 4.5            # "約 4.5" bpw
    assert 2 + 2 + 12 + 128 == 144                                # d, dmin, 8 x (6 + 6) bits, 256 x 4 bits
    per_expert = 3 * 4096 * 2048 // 256 * 144
    layer = 256 * per_expert
    assert layer == 3_623_878_656 and round(layer / 1e9, 1) == 3.6  # "約 3.6GB" per routed layer
    q2 = 256 * (2 * 2048 * 4096 // 256 * 66 + 4096 * 2048 // 256 * 84)
    assert round((layer - q2) / 1e9, 1) == 1.8                    # "約 1.8GB/層" to raise one layer


def _pack(d: int, dmin: int, sc, mn, codes) -> np.ndarray:
    """A block from its fields, written from the reading: scales/mins of
    sub-blocks 0-3 in the low 6 bits of bytes 0-3 / 4-7; sub-blocks 4-7 keep
    their low 4 bits in the nibbles of bytes 8-11 (scale low, min high) and
    their top 2 bits in the top bits of bytes 0-3 (scales) / 4-7 (mins); the
    code of element e in byte 32*(e//64) + e%32, nibble (e%64)//32."""
    blk = np.zeros(144, np.uint8)
    blk[0], blk[1], blk[2], blk[3] = d & 0xFF, d >> 8, dmin & 0xFF, dmin >> 8
    s = np.zeros(12, np.int64)
    for j in range(4):
        s[j] = (sc[j] & 63) | ((sc[j + 4] >> 4) << 6)
        s[j + 4] = (mn[j] & 63) | ((mn[j + 4] >> 4) << 6)
        s[j + 8] = (sc[j + 4] & 15) | ((mn[j + 4] & 15) << 4)
    blk[4:16] = s
    for e in range(256):
        blk[16 + 32 * (e // 64) + e % 32] |= int(codes[e]) << (4 * ((e % 64) // 32))
    return blk


def _decode(blk):
    return oracle.decode_row(K4, blk, 256)


def test_code_positions():
    """d = 1, no mins, every scale 1, code of e = e % 16: decodes to e % 16."""
    e = np.arange(256)
    y = _decode(_pack(0x3C00, 0, [1] * 8, [0] * 8, e % 16))
    assert np.array_equal(y, (e % 16).astype(np.float64))


def test_six_bit_scales():
    """d = 0.5, every code 1: sub-block j decodes to 0.5 * scale_j, with scales
    that use the top two bits (stored apart for j >= 4)."""
    sc = [1, 2, 3, 63, 17, 33, 48, 62]
    y = _decode(_pack(0x3800, 0, sc, [0] * 8, np.ones(256, np.int64)))
    assert np.array_equal(y, np.repeat(np.array(sc) * 0.5, 32))
    # the same values by hand for the split-stored ones: 17 = 0b01_0001, 62 = 0b11_1110
    assert y[4 * 32] == 8.5 and y[7 * 32] == 31.0


def test_six_bit_mins_are_subtracted():
    """dmin = 0.25, codes 0: sub-block j decodes to -0.25 * min_j."""
    mn = [0, 5, 16, 63, 1, 31, 47, 60]
    y = _decode(_pack(0x3C00, 0x3400, [9] * 8, mn, np.zeros(256, np.int64)))
    assert np.array_equal(y, np.repeat(-0.25 * np.array(mn), 32))


def test_random_fields_affine_form():
    """Random fields: every element is d*scale*q - dmin*min of its sub-block."""
    rng = np.random.default_rng(9)
    for _ in range(50):
        sc, mn = rng.integers(0, 64, 8), rng.integers(0, 64, 8)
        codes = rng.integers(0, 16, 256)
        dh, mh = int(rng.integers(0x1000, 0x4000)), int(rng.integers(0x1000, 0x4000))
        y = _decode(_pack(dh, mh, sc, mn, codes))
        d, dmin = oracle.f16(dh), oracle.f16(mh)
        j = np.arange(256) // 32
        assert np.array_equal(y, d * sc[j] * codes - dmin * mn[j])


def _q4k_matrix(rng, rows, cols):
    nb = cols // 256
    W = rng.integers(0, 256, (rows, nb, 144), dtype=np.uint8)
    d = np.float16(0.002 + 0.01 * rng.random((rows, nb))).view(np.uint16)
    m = np.float16(0.001 + 0.005 * rng.random((rows, nb))).view(np.uint16)
    W[:, :, 0], W[:, :, 1] = d & 0xFF, d >> 8
    W[:, :, 2], W[:, :, 3] = m & 0xFF, m >> 8
    return W.reshape(rows, nb * 144)


def test_layer_with_q4k_experts_matches_dequantised_reference():
    """The oracle layer on Q4_K gate/up/down against dequantise-then-multiply
    in numpy (rows decoded with the pinned decoder)."""
    rng = np.random.default_rng(10)
    H = I = Is = 256
    E, k, T = 4, 2, 3

    class Shape:
        hidden, inter, shared_inter, n_experts, top_k = H, I, Is, E, k

    W = {"gate": [_q4k_matrix(rng, I, H) for _ in range(E)], "up": [_q4k_matrix(rng, I, H) for _ in range(E)],
         "down": [_q4k_matrix(rng, H, I) for _ in range(E)], "gate_kind": K4, "down_kind": K4,
         "grid": np.zeros((256, 8), np.uint8)}
    for name, rows, cols in (("sh_gate", Is, H), ("sh_up", Is, H), ("sh_down", H, Is)):
        q = rng.integers(-127, 128, (rows, cols // 32, 32)).astype(np.int8).view(np.uint8)
        dd = np.full((rows, cols // 32, 1), np.float16(0.004)).view(np.uint8).reshape(rows, cols // 32, 2)
        W[name] = np.concatenate([dd, q], axis=2).reshape(rows, -1)
    x = rng.standard_normal((T, H))
    idx = np.array([[0, 2], [1, 3], [0, 3]], np.int32)
    w = np.array([[0.9, 0.6], [1.0, 0.5], [0.7, 0.8]])
    y = oracle.layer(W, Shape, x, idx, w)

    def deq(kind, M, rows, cols):
        return np.stack([oracle.decode_row(kind, M[r], cols) for r in range(rows)])

    def swiglu(g, u, dn, x):
        a, b = g @ x, u @ x
        return dn @ (a / (1 + np.exp(-a)) * b)

    K8 = oracle.KIND_Q80
    sh = [deq(K8, W["sh_gate"], Is, H), deq(K8, W["sh_up"], Is, H), deq(K8, W["sh_down"], H, Is)]
    ex = [[deq(K4, W["gate"][e], I, H), deq(K4, W["up"][e], I, H), deq(K4, W["down"][e], H, I)] for e in range(E)]
    ref = np.stack([swiglu(*sh, x[t]) + sum(w[t, i] * swiglu(*ex[idx[t, i]], x[t]) for i in range(k))
                    for t in range(T)])
    assert np.allclose(y, ref, rtol=1e-10, atol=1e-9 * np.abs(ref).max())
