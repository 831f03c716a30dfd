"""Pins for the CPU oracle: page figures, hand-built blocks, closed forms,
brute force and invariants.  Runs without a GPU."""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
import synth
from tests import blocks

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_kv(name):
    out = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = (p.strip() for p in line.split("="))
            out[k] = float(v) if "." in v else int(v)
    return out


# ----------------------------------------------------------------- sizes

def test_page_figures_match_block_arithmetic():
    p = _read_kv("page_figures.txt")
    s = synth.workload("decode_t1")
    assert (s.hidden, s.inter, s.n_experts, s.top_k) == (p["hidden_size"], p["moe_intermediate_size"],
                                                         p["n_routed_experts"], p["top_k"])
    assert s.routed_scaling == p["routed_scaling_factor"]
    assert s.vocab == p["vocab_size"]
    st = synth.workload("stack43_t8")
    assert st.layers == p["num_hidden_layers"] and st.hash_layers == p["hash_routed_layers"]
    assert 3 * s.hidden * s.inter == p["params_per_routed_expert"]
    assert synth.BLOCK_BYTES[synth.KIND_Q2K] == p["q2k_block_bytes"]
    assert synth.BLOCK_BYTES[synth.KIND_IQ2XXS] == p["iq2xxs_block_bytes"]
    assert synth.BLOCK_ELEMS[synth.KIND_Q2K] == p["q2k_block_elems"]
    # bits per weight against the bit-allocation table (rounded there)
    assert abs(66 * 8 / 256 - p["iq2xxs_bpw_approx"]) < 0.01
    assert abs(84 * 8 / 256 - p["q2k_bpw_approx"]) < 0.03
    assert abs(34 * 8 / 32 - p["q80_bpw_approx"]) < 1e-12
    # exact bytes of one routed expert and of a routed layer
    assert s.expert_bytes == 7_077_888
    assert abs(s.expert_bytes * 8 / p["params_per_routed_expert"] - 2.25) < 1e-12
    assert abs(s.expert_bytes * 8 / p["params_per_routed_expert"] - p["q2_mix_bpw_approx"]) < 0.1
    routed_layer = s.n_experts * s.expert_bytes
    assert routed_layer == 1_811_939_328
    assert abs(routed_layer / 1e9 - p["q2_routed_layer_gb_approx"]) < 0.05
    decode_routed = s.top_k * s.expert_bytes
    assert decode_routed == 42_467_328
    assert abs(decode_routed / 1e6 - p["decode_routed_mb_per_layer_approx"]) < 1.0
    assert s.shared_bytes == 26_738_688
    assert decode_routed + s.shared_bytes == 69_206_016


# ------------------------------------------------------------------- f16

def test_f16_all_codes_match_ieee_binary16():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = codes.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ------------------------------------------------------------------ Q2_K

def test_q2k_packing_expression_round_trip():
    rng = np.random.default_rng(11)
    codes = rng.integers(0, 4, 256)
    blk = blocks.q2k_block(codes, [1] * 16, [0] * 16, 1.0, 0.0)
    got = [oracle.q2k_elem(blk, e) for e in range(256)]
    assert got == [float(c) for c in codes]


def test_q2k_quarter_pattern_pins_shift_order():
    # codes depend only on which quarter (shift) of the 128-element half the
    # element is in; a decoder that reads the wrong shift sees other values
    codes = [(e % 128) // 32 for e in range(256)]
    blk = blocks.q2k_block(codes, [1] * 16, [0] * 16, 1.0, 0.0)
    assert [oracle.q2k_elem(blk, e) for e in range(256)] == [float(c) for c in codes]
    codes = [e // 128 * 3 for e in range(256)]
    blk = blocks.q2k_block(codes, [1] * 16, [0] * 16, 1.0, 0.0)
    assert [oracle.q2k_elem(blk, e) for e in range(256)] == [float(c) for c in codes]


def test_q2k_scale_nibble_per_16_elements():
    blk = blocks.q2k_block([1] * 256, list(range(16)), [0] * 16, 1.0, 0.0)
    assert [oracle.q2k_elem(blk, e) for e in range(256)] == [float(e // 16) for e in range(256)]


def test_q2k_min_is_subtracted():
    blk = blocks.q2k_block([0] * 256, [5] * 16, [1] * 16, 1.0, 1.0)
    assert all(oracle.q2k_elem(blk, e) == -1.0 for e in range(256))
    blk = blocks.q2k_block([2] * 256, [3] * 16, [2] * 16, 0.5, 0.25)
    assert all(oracle.q2k_elem(blk, e) == 0.5 * 3 * 2 - 0.25 * 2 for e in range(256))


def test_q2k_offsets_from_page():
    p = _read_kv("page_figures.txt")
    blk = np.zeros(84, dtype=np.uint8)
    b = blocks.f16_bits(2.0)
    blk[p["q2k_d_off"]], blk[p["q2k_d_off"] + 1] = b & 0xFF, b >> 8
    b = blocks.f16_bits(0.5)
    blk[p["q2k_dmin_off"]], blk[p["q2k_dmin_off"] + 1] = b & 0xFF, b >> 8
    blk[p["q2k_scales_off"] + 3] = 0x21  # sub-block 3: scale 1, min 2
    # byte qs[16] holds element 16 at shift 0 and element 48 at shift 2
    blk[p["q2k_qs_off"] + 16] = 0b11  # element 16 -> code 3, element 48 -> code 0
    # element 16 lies in sub-block 1 (scale 0, min 0); element 48 in sub-block 3
    assert oracle.q2k_elem(blk, 16) == 0.0
    assert oracle.q2k_elem(blk, 48) == 2.0 * 1 * 0 - 0.5 * 2
    blk[p["q2k_qs_off"] + 16] = 0b1100  # element 48 -> code 3
    assert oracle.q2k_elem(blk, 48) == 2.0 * 1 * 3 - 0.5 * 2


# --------------------------------------------------------------- IQ2_XXS

def _handbuilt_iq2():
    grid = np.full((256, 8), 8, dtype=np.uint8)
    grid[0] = [8, 25, 43, 8, 25, 43, 8, 25]
    grid[1] = [43, 43, 43, 43, 8, 8, 8, 8]
    groups = [([0, 0, 0, 0], [0, 0, 0, 0], 0)] * 8
    groups[0] = ([0, 0, 1, 0], [0b0000001, 0, 0b1111111, 0b0000011], 1)
    groups[5] = ([1, 1, 1, 1], [0, 0, 0, 0b1000000], 15)
    return blocks.iq2xxs_block(1.0, groups), grid


def test_iq2xxs_handbuilt_golden():
    blk, grid = _handbuilt_iq2()
    expect = _read_kv("iq2xxs_handbuilt.txt")
    for e, v in expect.items():
        assert oracle.iq2xxs_elem(blk, grid, int(e)) == v, e


def test_iq2xxs_sign_parity_cases():
    grid = np.full((256, 8), 25, dtype=np.uint8)
    for mask, neg in ((0, []), (0b1111111, list(range(8))), (0b0000001, [0, 7]), (0b0000011, [0, 1]),
                      (0b0100101, [0, 2, 5, 7])):
        blk = blocks.iq2xxs_block(0.5, [([3, 3, 3, 3], [mask] * 4, 2)] * 8)
        vals = [oracle.iq2xxs_elem(blk, grid, e) for e in range(8)]
        mag = 0.5 * 2.5 / 4 * 25
        assert vals == [-mag if l in neg else mag for l in range(8)], mask


def test_iq2xxs_even_negatives_on_random_blocks():
    grid = synth.grid(0)
    W = synth.routed(0, 0, synth.T_GATE, synth.KIND_IQ2XXS, 0, 1, 8, 256)[0]
    for r in range(8):
        row = oracle.decode_row(0, W[r], 256, grid)
        for v in range(32):
            assert (row[8 * v:8 * v + 8] < 0).sum() % 2 == 0
            assert np.all(row[8 * v:8 * v + 8] != 0)


def test_iq2xxs_scale_nibbles_distinct_and_nonzero():
    grid = np.full((256, 8), 8, dtype=np.uint8)
    vals = []
    for s in range(16):
        blk = blocks.iq2xxs_block(1.0, [([0] * 4, [0] * 4, s)] * 8)
        vals.append(oracle.iq2xxs_elem(blk, grid, 0))
    assert vals == [8 * (0.5 + s) / 4 for s in range(16)]


# ------------------------------------------------------------------ Q8_0

def test_q80_exact_halves_and_f16_scale():
    q = list(range(-127, -127 + 32))
    blk = blocks.q80_block(0.5, q)
    assert [oracle.q80_elem(blk, e) for e in range(32)] == [0.5 * v for v in q]
    blk = blocks.q80_block(0.0005, [1] * 32)
    d16 = float(np.float16(0.0005))
    assert d16 != 0.0005
    assert oracle.q80_elem(blk, 7) == d16
    # the synthetic generator writes that same rounded scale
    W = synth.shared(0, 0, synth.T_SH_GATE, 1, 32)
    assert oracle.q80_elem(W[0], 0) == d16 * int(W[0][2:3].view(np.int8)[0])


# ---------------------------------------------------------------- router

def test_sqrtsoftplus_closed_forms():
    assert oracle.sqrtsoftplus(0.0) == pytest.approx(math.sqrt(math.log(2.0)), rel=1e-15)
    for z in (-30.0, -3.0, -0.5, 0.7, 4.0, 20.0):
        assert oracle.sqrtsoftplus(z) == pytest.approx(math.sqrt(math.log1p(math.exp(z))), rel=1e-14)
    assert oracle.sqrtsoftplus(800.0) == pytest.approx(math.sqrt(800.0), rel=1e-15)
    assert oracle.sqrtsoftplus(-800.0) == 0.0
    zs = np.linspace(-20, 20, 2001)
    s = np.array([oracle.sqrtsoftplus(z) for z in zs])
    assert np.all(np.diff(s) > 0)


def test_router_logits_one_hot_rows():
    H, E, T = 64, 16, 3
    Wr = np.zeros((E, H), dtype=np.float16)
    for e in range(E):
        Wr[e, 2 * e] = 1.0
        Wr[e, 2 * e + 1] = -0.5
    x = synth.activations(1, T, H)
    z = oracle.router_logits(x, Wr)
    for t in range(T):
        for e in range(E):
            assert z[t, e] == float(x[t, 2 * e]) - 0.5 * float(x[t, 2 * e + 1])


def _is_topk(keys, S):
    S = set(S)
    for i in S:
        for j in range(len(keys)):
            if j in S:
                continue
            if not (keys[i] > keys[j] or (keys[i] == keys[j] and i < j)):
                return False
    return True


def test_topk_brute_force_all_pairs_tiny():
    rng = np.random.default_rng(3)
    for trial in range(20):
        E, k = 16, 2
        z = rng.normal(0, 1.3, (1, E))
        bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
        idx, w, margin = oracle.select(z, bias, k)
        keys = [oracle.sqrtsoftplus(z[0, e]) + float(bias[e]) for e in range(E)]
        winners = [S for S in itertools.combinations(range(E), k) if _is_topk(keys, S)]
        assert len(winners) == 1
        assert list(idx[0]) == list(winners[0])
        srt = sorted(keys, reverse=True)
        assert margin[0] == srt[k - 1] - srt[k]


def test_topk_brute_force_random_small():
    rng = np.random.default_rng(4)
    for trial in range(60):
        E = int(rng.integers(2, 17))
        k = int(rng.integers(1, min(4, E) + 1))
        z = rng.normal(0, 1.0, (1, E))
        bias = rng.uniform(-0.2, 0.2, E).astype(np.float32)
        idx, w, _ = oracle.select(z, bias, k)
        keys = [oracle.sqrtsoftplus(z[0, e]) + float(bias[e]) for e in range(E)]
        winners = [S for S in itertools.combinations(range(E), k) if _is_topk(keys, S)]
        assert [list(s) for s in winners] == [list(idx[0])]


def test_ties_go_to_lower_id():
    E, k = 16, 4
    z = np.full((1, E), 0.3)
    bias = np.zeros(E, dtype=np.float32)
    idx, w, margin = oracle.select(z, bias, k)
    assert list(idx[0]) == [0, 1, 2, 3]
    assert np.allclose(w[0], 1.5 / k, rtol=1e-15, atol=0)
    assert margin[0] == 0.0
    # identical router rows and equal bias on a subset: lower ids of the tie win
    z = np.zeros((1, E))
    z[0, [3, 5, 9, 12, 14]] = 1.0
    idx, _, _ = oracle.select(z, bias, 3)
    assert list(idx[0]) == [3, 5, 9]


def test_bias_selects_but_does_not_weight():
    E, k = 8, 2
    z = np.array([[0.0, 0.1, 0.2, 0.3, 0.4, 0.5, 0.6, 0.7]])
    bias = np.array([1.0, 0, 0, 0, 0, 0, 0, 0.9], dtype=np.float32)
    idx, w, _ = oracle.select(z, bias, k, 1.5)
    assert list(idx[0]) == [0, 7]
    s0, s7 = oracle.sqrtsoftplus(0.0), oracle.sqrtsoftplus(0.7)
    assert w[0, 0] == pytest.approx(1.5 * s0 / (s0 + s7), rel=1e-15)
    assert w[0, 1] == pytest.approx(1.5 * s7 / (s0 + s7), rel=1e-15)


def test_weights_sum_to_scaling_on_seeded_tiny():
    s = synth.workload("tiny")
    x = synth.activations(0, 64, s.hidden)
    Wr = synth.router_weight(0, 0, s.n_experts, s.hidden)
    b = synth.bias(0, 0, s.n_experts, False)
    idx, w, margin = oracle.route(x, Wr, b, s.top_k)
    assert np.all(np.abs(w.sum(1) - 1.5) <= 1e-12)
    assert np.all(np.diff(idx, axis=1) > 0)
    assert np.all(margin >= 0)


def test_hash_route_uniform_weights():
    tab = synth.tid2eid(0, 0, 1000, 256, 6)
    ids = synth.token_ids(0, 50, 1000)
    idx, w = oracle.hash_route(ids, tab, 6)
    assert np.all(w == 0.25)
    for t in range(50):
        assert list(idx[t]) == sorted(tab[ids[t]])


def test_hash_route_rejects_token_ids_outside_the_table():
    """A token id outside [0, vocab) names no table row: an error, not row 0."""
    tab = synth.tid2eid(0, 0, 1000, 256, 6)
    for bad in (-1, 1000, 1 << 30):
        ids = np.array([3, bad, 7], dtype=np.int32)
        with pytest.raises(ValueError, match="token id"):
            oracle.hash_route(ids, tab, 6)


@pytest.mark.parametrize("entry", [-1, 256, 999])
def test_hash_route_rejects_table_rows_outside_the_experts(entry):
    tab = synth.tid2eid(0, 0, 100, 256, 6).copy()
    tab[5, 2] = entry
    with pytest.raises(ValueError, match="table row"):
        oracle.hash_route(np.array([5], np.int32), tab, 6)
    # rows of other tokens are not looked at
    idx, _ = oracle.hash_route(np.array([4, 6], np.int32), tab, 6)
    assert list(idx[0]) == sorted(tab[4]) and list(idx[1]) == sorted(tab[6])


def test_hash_route_rejects_a_repeated_expert_in_a_row():
    tab = synth.tid2eid(0, 0, 100, 256, 6).copy()
    tab[9, 4] = tab[9, 1]
    with pytest.raises(ValueError, match="table row"):
        oracle.hash_route(np.array([9], np.int32), tab, 6)


@pytest.mark.parametrize("q4k", [False, True])
def test_threaded_layer_equals_single_thread_bitwise(q4k):
    """oracle.layer(threads=n) splits the tokens into consecutive slices (7
    tokens over 3 threads: 3, 2, 2); every token's output must be the
    single-thread result bit for bit, so a slice offset error in x, idx, w or
    y shows here.  Both routed formats (q2 build and Q4_K layers)."""
    s = synth.workload("tiny", tokens=7)
    x = synth.activations(4, 7, s.hidden).astype(np.float64)
    Wr = synth.router_weight(4, 0, s.n_experts, s.hidden)
    b = synth.bias(4, 0, s.n_experts, False)
    idx, w, _ = oracle.route(x, Wr, b, s.top_k)
    W = synth.host_layer(4, 0, s, experts=np.unique(idx), q4k=q4k)
    y1 = oracle.layer(W, s, x, idx, w, threads=1)
    for n in (2, 3, 7, 16):
        yn = oracle.layer(W, s, x, idx, w, threads=n)
        assert np.array_equal(y1.view(np.uint64), yn.view(np.uint64)), n
    # each token's row is that token's layer alone
    for t in (0, 3, 6):
        yt = oracle.layer(W, s, x[t:t + 1], idx[t:t + 1], w[t:t + 1])
        assert np.array_equal(yt[0].view(np.uint64), y1[t].view(np.uint64))


@pytest.mark.parametrize("q4k", [False, True])
def test_dense_layer_route_equals_the_row_by_row_layer(q4k):
    """oracle.layer_dense (decode every used matrix, then numpy fp64 matrix
    products) against oracle.layer (row-by-row fused route): the same layer up
    to the order of fp64 additions.  Tiny shapes, 23 tokens, router routing."""
    s = synth.workload("tiny", tokens=23)
    x = synth.activations(8, 23, s.hidden).astype(np.float64)
    Wr = synth.router_weight(8, 1, s.n_experts, s.hidden)
    b = synth.bias(8, 1, s.n_experts, True)
    idx, w, _ = oracle.route(x, Wr, b, s.top_k)
    W = synth.host_layer(8, 1, s, experts=np.unique(idx), q4k=q4k)
    ref = oracle.layer(W, s, x, idx, w)
    got = oracle.layer_dense(W, s, x, idx, w, threads=3)
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_dense_layer_route_at_full_shape_one_token():
    s = synth.workload("decode_t1")
    x = synth.activations(2, 1, s.hidden).astype(np.float64)
    Wr = synth.router_weight(2, 0, s.n_experts, s.hidden)
    b = synth.bias(2, 0, s.n_experts, False)
    idx, w, _ = oracle.route(x, Wr, b, s.top_k)
    W = synth.host_layer(2, 0, s, experts=np.unique(idx))
    ref = oracle.layer(W, s, x, idx, w)
    got = oracle.layer_dense(W, s, x, idx, w)
    assert np.max(np.abs(got - ref)) <= 1e-11 * np.max(np.abs(ref))


# ---------------------------------------------------------------- matvec

@pytest.mark.parametrize("kind,rows,cols", [(0, 12, 512), (1, 12, 512), (2, 12, 256)])
def test_fused_matvec_equals_dequantise_then_gemv(kind, rows, cols):
    grid = synth.grid(5)
    tensor = {0: synth.T_GATE, 1: synth.T_DOWN, 2: synth.T_SH_UP}[kind]
    W = synth.routed(5, 0, tensor, kind, 0, 1, rows, cols)[0]
    x = np.random.default_rng(9).normal(size=cols)
    fused = oracle.matvec(kind, W, rows, cols, x, grid)
    dense = oracle.decode_matrix(kind, W, rows, cols, grid) @ x
    assert np.allclose(fused, dense, rtol=1e-12, atol=1e-12 * np.abs(dense).max())


# ----------------------------------------------------------------- layer

def _closed_form_layer(T=3):
    """H = I = Is = 256, E = 4, k = 2 with constant weights: every gate, up
    and down element of expert e is a known constant, so each output is a
    closed form of sum(x)."""
    H = I = Is = 256
    E, k = 4, 2
    shape = synth.LayerShape(H, I, Is, E, k, T)
    grid = np.full((256, 8), 8, dtype=np.uint8)
    grid[1] = 25
    consts = {}
    gate, up, down = {}, {}, {}
    for e in range(E):
        dg, sg = [0.25, 0.5, 0.125, 0.0625][e], e  # gate value dg*(0.5+sg)/4*8
        du, su = [0.125, 0.25, 0.5, 0.25][e], 3
        gate[e] = blocks.constant_iq2_rows(I, H, dg, sg, 0)
        up[e] = blocks.constant_iq2_rows(I, H, du, su, 1)
        qd, scd, mnd, dd, dmd = [(1, 2, 1, 0.01, 0.005), (2, 3, 4, 0.02, 0.01), (3, 1, 0, 0.005, 0.0),
                                 (0, 7, 9, 0.001, 0.002)][e]
        down[e] = blocks.constant_q2k_rows(H, I, qd, scd, mnd, dd, dmd)
        G = float(np.float16(dg)) * (0.5 + sg) / 4 * 8
        U = float(np.float16(du)) * (0.5 + su) / 4 * 25
        D = float(np.float16(dd)) * scd * qd - float(np.float16(dmd)) * mnd
        consts[e] = (G, U, D)
    sh = dict(sh_gate=blocks.constant_q80_rows(Is, H, 0.0078125, 3),
              sh_up=blocks.constant_q80_rows(Is, H, 0.0078125, -2),
              sh_down=blocks.constant_q80_rows(H, Is, 0.001953125, 5))
    SG, SU, SD = 0.0078125 * 3, 0.0078125 * -2, 0.001953125 * 5
    weights = dict(gate=gate, up=up, down=down, grid=grid, **sh)
    return shape, weights, consts, (SG, SU, SD)


def _silu(u):
    return u / (1 + math.exp(-u))


def test_layer_closed_form_constant_experts():
    shape, weights, consts, (SG, SU, SD) = _closed_form_layer()
    H, I, Is = shape.hidden, shape.inter, shape.shared_inter
    x = np.random.default_rng(2).normal(0, 0.05, (3, H))
    # router: zero logits; bias picks experts 1 and 3
    z = np.zeros((3, 4))
    bias = np.array([0.0, 0.5, 0.0, 0.25], dtype=np.float32)
    idx, w, _ = oracle.select(z, bias, 2)
    assert idx.tolist() == [[1, 3]] * 3 and np.all(w == 0.75)
    y = oracle.layer(weights, shape, x, idx, w)
    for t in range(3):
        X = x[t].sum()
        expect = Is * SD * _silu(SG * X) * (SU * X)
        for e in (1, 3):
            G, U, D = consts[e]
            expect += 0.75 * I * D * _silu(G * X) * (U * X)
        assert np.allclose(y[t], expect, rtol=1e-12, atol=1e-15)


def test_layer_gate_and_up_are_not_interchangeable():
    shape, weights, consts, _ = _closed_form_layer(T=1)
    x = np.full((1, shape.hidden), 0.01)
    idx = np.array([[0, 2]], dtype=np.int32)
    w = np.array([[0.75, 0.75]])
    y1 = oracle.layer(weights, shape, x, idx, w)
    swapped = dict(weights, gate=weights["up"], up=weights["gate"])
    y2 = oracle.layer(swapped, shape, x, idx, w)
    assert not np.allclose(y1, y2)


def test_layer_zero_gate_scale_gives_shared_only():
    s = synth.workload("tiny")
    W = synth.host_layer(0, 0, s)
    x = synth.activations(0, s.tokens, s.hidden).astype(np.float64)
    idx, w, _ = oracle.route(x.astype(np.float32), W["router_w"], W["bias"], s.top_k)
    zero = W["gate"].copy()
    zero.reshape(-1, 66)[:, 0:2] = 0  # d = 0 in every gate block
    W0 = dict(W, gate=zero)
    y = oracle.layer(W0, s, x, idx, w)
    sh = np.stack([oracle.swiglu_expert(W["sh_gate"], W["sh_up"], W["sh_down"], s.hidden, s.shared_inter,
                                        x[t], gate_kind=2, down_kind=2) for t in range(s.tokens)])
    assert np.array_equal(y, sh)


def test_layer_linear_in_routing_weights_and_shared_additive():
    s = synth.workload("tiny")
    W = synth.host_layer(1, 0, s)
    x = synth.activations(1, s.tokens, s.hidden).astype(np.float64)
    idx = np.array([[0, 5], [3, 15], [7, 8], [1, 2]], dtype=np.int32)
    w1 = np.full((4, 2), 0.75)
    zsh = dict(W, sh_gate=np.zeros_like(W["sh_gate"]))  # shared expert off (d = 0)
    y1 = oracle.layer(zsh, s, x, idx, w1)
    y2 = oracle.layer(zsh, s, x, idx, 2 * w1)
    assert np.allclose(y2, 2 * y1, rtol=1e-12, atol=1e-9)
    # one slot at a time adds up to both slots
    ya = oracle.layer(zsh, s, x, idx, np.stack([w1[:, 0], np.zeros(4)], 1))
    yb = oracle.layer(zsh, s, x, idx, np.stack([np.zeros(4), w1[:, 1]], 1))
    assert np.allclose(ya + yb, y1, rtol=1e-12, atol=1e-9)


def test_all_experts_selected_when_k_equals_E():
    E = k = 4
    z = np.random.default_rng(1).normal(size=(2, E))
    idx, w, margin = oracle.select(z, np.zeros(E, dtype=np.float32), k)
    assert idx.tolist() == [[0, 1, 2, 3]] * 2
    s = np.array([[oracle.sqrtsoftplus(v) for v in row] for row in z])
    assert np.allclose(w, 1.5 * s / s.sum(1, keepdims=True), rtol=1e-15)
    assert np.all(np.isinf(margin))


# ----------------------------------------------------------- permutation

def test_permutation_brute_force():
    rng = np.random.default_rng(8)
    for T, k, E in ((1, 6, 256), (5, 2, 16), (33, 6, 64), (100, 3, 7)):
        idx = np.stack([np.sort(rng.choice(E, k, replace=False)) for _ in range(T)]).astype(np.int32)
        offsets, perm = oracle.permutation(idx, E)
        pairs = sorted(((int(idx[t, i]), t, i) for t in range(T) for i in range(k)))
        assert perm.tolist() == [t * k + i for _, t, i in pairs]
        counts = np.bincount(idx.ravel(), minlength=E)
        assert offsets.tolist() == [0] + np.cumsum(counts).tolist()
        assert offsets[-1] == T * k


def test_permutation_degenerate_all_on_one_expert():
    idx = np.zeros((10, 1), dtype=np.int32) + 5
    offsets, perm = oracle.permutation(idx, 8)
    assert offsets.tolist() == [0, 0, 0, 0, 0, 0, 10, 10, 10]
    assert perm.tolist() == list(range(10))


# --------------------------------------------------------------- RMSNorm

def test_rmsnorm_invariant():
    x = np.random.default_rng(0).normal(0, 3, (4, 4096))
    eps = 1e-6
    out = oracle.rmsnorm(x, eps)
    for t in range(4):
        ms = np.mean(x[t] ** 2)
        assert np.mean(out[t] ** 2) == pytest.approx(1 / (1 + eps / ms), rel=1e-12)
        assert np.all(np.sign(out[t]) == np.sign(x[t]))
