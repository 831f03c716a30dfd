"""Parity of the CUDA layer against the fp64 oracle for the small-T path
(T <= 32: mma.sync int8 GEMV kernels), routing for every T, and the layer's
error paths.  Everything goes through the C ABI."""
import numpy as np
import pytest

import oracle
import synth
from tests import harness

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


def _run(moe, s, seed, layer, T, mode=0, flags=0, weights=None):
    router = mode == moe.MOE_ROUTE_ROUTER
    W = weights if weights is not None else harness.device_layer(s, seed, layer, router=router)
    cfg = harness.config_for(s, mode, flags)
    L = moe.Layer(cfg, W, max_tokens=T)
    x_np = synth.activations(seed, T, s.hidden, stream=layer)
    tok_np = synth.token_ids(seed, T, s.vocab, stream=layer)
    x = torch.from_numpy(x_np).cuda()
    tok = torch.from_numpy(tok_np).cuda()
    y = L.forward(x, tok)
    idx, w = L.route(x, tok)
    torch.cuda.synchronize()
    L.poll()
    out = dict(x=x_np, tok=tok_np, y=y.cpu().numpy(), idx=idx.cpu().numpy(), w=w.cpu().numpy(), layer=L, W=W)
    return out


def _check(s, got, seed, layer, router=True, prenorm=False, rel=harness.GEMV_REL_L2):
    idx, w, yref, margin = harness.oracle_layer(s, seed, layer, got["x"], got["tok"], router=router,
                                                prenorm=prenorm)
    assert np.array_equal(got["idx"], idx), (got["idx"], idx, margin)
    assert np.allclose(got["w"], w, rtol=1e-6, atol=1e-7)
    rel_l2, max_abs = harness.errors(got["y"], yref)
    assert rel_l2 <= rel, rel_l2
    assert max_abs <= harness.MAX_ABS_FRAC, max_abs
    return rel_l2, max_abs


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 8])
def test_tiny_layer_matches_oracle(moe, T):
    s = synth.workload("tiny", tokens=T)
    got = _run(moe, s, 0, 0, T)
    _check(s, got, 0, 0)


@pytest.mark.parametrize("T", [9, 16, 32])
def test_tiny_layer_medium_token_counts(moe, T):
    """9..32 tokens: the shared expert's tokens run in token groups of one
    unit's width, each with its own tile counters."""
    s = synth.workload("tiny", tokens=T)
    got = _run(moe, s, 0, 0, T)
    _check(s, got, 0, 0)


def test_experts_with_more_tokens_than_a_unit_are_split(moe):
    """The skewed bias sends (nearly) every token to experts 0 and 8, so they
    hold more pairs than one unit takes and are split into several jobs."""
    s = synth.workload("tiny", tokens=24, skew=True)
    got = _run(moe, s, 1, 0, 24)
    counts = np.bincount(got["idx"].ravel(), minlength=s.n_experts)
    assert counts.max() > 8, counts
    _check(s, got, 1, 0)


def test_tiny_hash_routed_layer(moe):
    s = synth.workload("tiny", tokens=6)
    got = _run(moe, s, 3, 1, 6, mode=moe.MOE_ROUTE_HASH)
    _check(s, got, 3, 1, router=False)
    assert np.all(got["w"] == np.float32(0.75))


def test_tiny_prenorm_residual(moe):
    s = synth.workload("tiny", tokens=4)
    got = _run(moe, s, 5, 2, 4, flags=moe.MOE_FLAG_PRENORM_RESIDUAL)
    _check(s, got, 5, 2, prenorm=True)


def test_tiny_skewed_bias_and_other_seed(moe):
    s = synth.workload("tiny", tokens=8, skew=True)
    got = _run(moe, s, 11, 4, 8)
    _check(s, got, 11, 4)


def test_full_decode_one_token(moe):
    s = synth.workload("decode_t1")
    got = _run(moe, s, 0, 0, 1)
    rel, mx = _check(s, got, 0, 0)
    print(f"decode_t1 rel_l2={rel:.3e} max_abs_frac={mx:.3e}")


def test_full_decode_eight_tokens_prenorm(moe):
    s = synth.workload("decode_t1", tokens=8)
    got = _run(moe, s, 2, 7, 8, flags=moe.MOE_FLAG_PRENORM_RESIDUAL)
    _check(s, got, 2, 7, prenorm=True)


def test_full_decode_32_tokens_every_row(moe):
    """V4-Flash shapes at 32 tokens with the skewed bias (the largest call of
    the small-T kernels): routing of every token bit-exact and every output
    row within the GEMV tolerance.  Split experts, the shared expert's token
    groups and single-token jobs all occur in this call."""
    s = synth.workload("decode_t32")
    T = s.tokens
    got = _run(moe, s, 3, 1, T)
    idx, w, yref, margin = harness.oracle_layer_dense(s, 3, 1, got["x"])
    assert np.array_equal(got["idx"], idx), margin
    assert np.allclose(got["w"], w, rtol=1e-6, atol=1e-7)
    counts = np.bincount(idx.ravel(), minlength=s.n_experts)
    assert counts.max() > 2 and (counts == 1).any()  # split experts and one-token jobs
    rel_l2, max_abs = harness.errors(got["y"], yref)
    print(f"decode_t32 every row: rel_l2={rel_l2:.3e} max_abs_frac={max_abs:.3e}")
    assert rel_l2 <= harness.GEMV_REL_L2, rel_l2
    assert max_abs <= harness.MAX_ABS_FRAC, max_abs
    # row by row as well: no single token may hide behind the others
    for t in range(T):
        r, _ = harness.errors(got["y"][t], yref[t])
        assert r <= harness.GEMV_REL_L2, (t, r)


def test_full_decode_hash_layer(moe):
    s = synth.workload("decode_t1", tokens=3)
    got = _run(moe, s, 4, 0, 3, mode=moe.MOE_ROUTE_HASH)
    _check(s, got, 4, 0, router=False)


def test_repeat_calls_are_bitwise_identical(moe):
    s = synth.workload("tiny", tokens=5)
    got = _run(moe, s, 9, 0, 5)
    L = got["layer"]
    x = torch.from_numpy(got["x"]).cuda()
    for _ in range(3):
        y2 = L.forward(x).cpu().numpy()
        assert np.array_equal(y2, got["y"])


def test_constructed_ties_go_to_lower_id(moe):
    s = synth.workload("tiny", tokens=4)
    W = harness.device_layer(s, 0, 0)
    Wr = W["router_w"].clone()
    for e in (5, 9, 12):
        Wr[e] = Wr[3]
    W["router_w"] = Wr
    b = W["bias"].clone()
    b[:] = -1.0
    b[[3, 5, 9, 12]] = 0.0
    W["bias"] = b
    got = _run(moe, s, 0, 0, 4, weights=W)
    assert got["idx"].tolist() == [[3, 5]] * 4


def test_zero_tokens_is_a_no_op(moe):
    s = synth.workload("tiny", tokens=1)
    W = harness.device_layer(s, 0, 0)
    L = moe.Layer(harness.config_for(s), W, max_tokens=1)
    x = torch.zeros((0, s.hidden), device="cuda")
    y = torch.zeros((0, s.hidden), device="cuda")
    moe.moe_ffn_forward(L.handle, x, None, 0, y, L.scratch)
    L.poll()


def test_codebook_entry_above_127_is_reported(moe):
    s = synth.workload("tiny", tokens=1)
    W = harness.device_layer(s, 0, 0)
    W["grid"][0, 0] = 200
    L = moe.Layer(harness.config_for(s), W, max_tokens=1)
    x = torch.from_numpy(synth.activations(0, 1, s.hidden)).cuda()
    L.forward(x)
    with pytest.raises(moe.MoeError) as ei:
        L.poll()
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_SHAPE
    L.poll()  # the word was cleared


def test_out_of_range_token_id_is_reported(moe):
    s = synth.workload("tiny", tokens=2)
    W = harness.device_layer(s, 0, 0, router=False)
    L = moe.Layer(harness.config_for(s, mode=moe.MOE_ROUTE_HASH), W, max_tokens=2)
    x = torch.from_numpy(synth.activations(0, 2, s.hidden)).cuda()
    tok = torch.tensor([5, s.vocab + 3], dtype=torch.int32, device="cuda")
    L.forward(x, tok)
    with pytest.raises(moe.MoeError) as ei:
        L.poll()
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("bad", ["out_of_range", "negative", "repeated"])
def test_bad_token_table_is_rejected_at_init(moe, bad):
    """Hash mode: moe_init checks that every tid2eid row holds top_k distinct
    ids in [0, n_experts) and creates no handle otherwise."""
    s = synth.workload("tiny", tokens=2)
    W = harness.device_layer(s, 0, 0, router=False)
    tab = W["tid2eid"].clone()
    row = s.vocab - 7
    if bad == "out_of_range":
        tab[row, 1] = s.n_experts
    elif bad == "negative":
        tab[row, 0] = -3
    else:
        tab[row, 1] = tab[row, 0]
    W["tid2eid"] = tab
    with pytest.raises(moe.MoeError) as ei:
        moe.Layer(harness.config_for(s, mode=moe.MOE_ROUTE_HASH), W, max_tokens=2)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    assert f"row {row}" in str(ei.value)
    # the unchanged table is accepted
    W["tid2eid"] = harness.device_layer(s, 0, 0, router=False)["tid2eid"]
    moe.Layer(harness.config_for(s, mode=moe.MOE_ROUTE_HASH), W, max_tokens=2).poll()


def test_scratch_too_small_is_rejected(moe):
    s = synth.workload("tiny", tokens=8)
    W = harness.device_layer(s, 0, 0)
    L = moe.Layer(harness.config_for(s), W, max_tokens=2)
    x = torch.from_numpy(synth.activations(0, 8, s.hidden)).cuda()
    with pytest.raises(moe.MoeError) as ei:
        L.forward(x)
    assert ei.value.status == moe.MOE_ERR_WORKSPACE_TOO_SMALL


# ----------------------------------------------------------------- routing

@pytest.mark.parametrize("name,T", [("tiny", 300), ("decode_t32", 32), ("prefill_t4096", 4096)])
def test_route_and_permutation_bit_exact(moe, name, T):
    s = synth.workload(name, tokens=T)
    W = harness.device_layer(s, 1, 3)
    L = moe.Layer(harness.config_for(s), W, max_tokens=T)
    x_np = synth.activations(1, T, s.hidden, stream=3)
    x = torch.from_numpy(x_np).cuda()
    idx, w, off, perm = L.route(x, with_perm=True)
    torch.cuda.synchronize()
    L.poll()
    Wr = synth.router_weight(1, 3, s.n_experts, s.hidden)
    b = synth.bias(1, 3, s.n_experts, s.skew)
    ridx, rw, margin = oracle.route(x_np, Wr, b, s.top_k, s.routed_scaling)
    gidx = idx.cpu().numpy()
    bad = np.nonzero(np.any(gidx != ridx, axis=1))[0]
    assert bad.size == 0, (bad[:10], margin[bad[:10]])
    assert np.allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=1e-7)
    roff, rperm = oracle.permutation(ridx, s.n_experts)
    assert np.array_equal(off.cpu().numpy(), roff)
    assert np.array_equal(perm.cpu().numpy(), rperm)
    print(f"{name}: min margin {margin.min():.3e}, counts min/max {np.diff(roff).min()}/{np.diff(roff).max()}")


@pytest.mark.parametrize("name,T", [("tiny", 40), ("decode_t32", 64)])
def test_chunked_small_token_calls(moe, name, T):
    """From 33 to 64 tokens a q2 layer runs the small-token kernels on the
    first 32 tokens and then on the rest: the output equals, bit for bit, the
    two calls made separately, and matches the oracle at the small-token
    tolerance (every row)."""
    s = synth.workload(name, tokens=T)
    W = harness.device_layer(s, 4, 3)
    L = moe.Layer(harness.config_for(s), W, max_tokens=T)
    x_np = synth.activations(4, T, s.hidden, stream=3)
    x = torch.from_numpy(x_np).cuda()
    y = L.forward(x).cpu().numpy()
    y0 = L.forward(x[:32].contiguous()).cpu().numpy()
    y1 = L.forward(x[32:].contiguous()).cpu().numpy()
    L.poll()
    assert np.array_equal(y.view(np.uint32), np.concatenate([y0, y1]).view(np.uint32))
    _, _, yref, _ = harness.oracle_layer_dense(s, 4, 3, x_np)
    rel, mx = harness.errors(y, yref)
    assert rel <= harness.GEMV_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)
    for t in range(T):
        r, _ = harness.errors(y[t], yref[t])
        assert r <= harness.GEMV_REL_L2, (t, r)
