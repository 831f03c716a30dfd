"""GPU checks for the Q4_K routed-expert variant (the q2-q4 build's upgraded
layers), through the C ABI against the fp64 oracle: the generator's device
fill (byte-identical to the host fill the oracle reads); the small-token path
(tiny layer at T = 1, 3, 8, 32, hash routing with the pre-norm residual,
V4-Flash shapes at T = 1 and 8); the batched path (tiny layer at T = 33, 64,
300, hash routing with pre-norm, V4-Flash shapes at T = 512 on sampled rows);
the tail of the q2-q4 stack; and the missing no-allocation forward."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def test_q4k_device_fill_is_byte_identical_to_host_fill():
    synth.build(device=True)
    for tensor, rows, cols, e0, ne in ((synth.T_GATE, 64, 4096, 7, 2), (synth.T_DOWN, 96, 2048, 0, 3)):
        host = synth.routed(3, 40, tensor, synth.KIND_Q4K, e0, ne, rows, cols)
        dev = torch.empty(host.shape, dtype=torch.uint8, device="cuda")
        synth.device_routed(dev, 3, 40, tensor, synth.KIND_Q4K, e0, ne, rows, cols)
        torch.cuda.synchronize()
        assert np.array_equal(dev.cpu().numpy(), host)


# ------------------------------------------------------------ the Q4_K layer

from tests import harness  # noqa: E402


@pytest.fixture(scope="module")
def moe():
    from bit_moe_expert_sqrtsoftplus_b200 import build
    build.build()
    import bit_moe_expert_sqrtsoftplus_b200 as m
    return m


def _run_q4k(moe, s, seed, layer, T, mode=0, flags=0):
    router = mode == moe.MOE_ROUTE_ROUTER
    W = harness.device_layer(s, seed, layer, router=router, q4k=True)
    L = moe.Layer(harness.config_for(s, mode, flags, q4k=True), W, max_tokens=T)
    x_np = synth.activations(seed, T, s.hidden, stream=layer)
    tok_np = synth.token_ids(seed, T, s.vocab, stream=layer)
    x = torch.from_numpy(x_np).cuda()
    tok = torch.from_numpy(tok_np).cuda()
    y = L.forward(x, tok)
    idx, w = L.route(x, tok)
    torch.cuda.synchronize()
    L.poll()
    return dict(x=x_np, tok=tok_np, y=y.cpu().numpy(), idx=idx.cpu().numpy(), w=w.cpu().numpy())


def _check_q4k(s, got, seed, layer, router=True, prenorm=False):
    idx, w, yref, margin = harness.oracle_layer(s, seed, layer, got["x"], got["tok"], router=router, prenorm=prenorm,
                                                q4k=True)
    assert np.array_equal(got["idx"], idx), margin
    assert np.allclose(got["w"], w, rtol=1e-6, atol=1e-7)
    rel_l2, max_abs = harness.errors(got["y"], yref)
    assert rel_l2 <= harness.GEMV_REL_L2, rel_l2
    assert max_abs <= harness.MAX_ABS_FRAC, max_abs


@pytest.mark.parametrize("T", [1, 3, 8, 32])
def test_tiny_q4k_layer_matches_oracle(moe, T):
    s = synth.workload("tiny", tokens=T)
    _check_q4k(s, _run_q4k(moe, s, 0, 0, T), 0, 0)


def test_tiny_q4k_hash_layer_with_prenorm_residual(moe):
    s = synth.workload("tiny", tokens=5)
    got = _run_q4k(moe, s, 2, 1, 5, mode=moe.MOE_ROUTE_HASH, flags=moe.MOE_FLAG_PRENORM_RESIDUAL)
    _check_q4k(s, got, 2, 1, router=False, prenorm=True)


def test_full_q4k_layer_one_and_eight_tokens(moe):
    """V4-Flash shapes (3.6 GB of Q4_K routed experts)."""
    for T, seed in ((1, 0), (8, 5)):
        s = synth.workload("decode_t1", tokens=T)
        _check_q4k(s, _run_q4k(moe, s, seed, 39, T), seed, 39)


def test_q4k_layer_has_no_noalloc_forward(moe):
    s = synth.workload("tiny", tokens=2)
    W = harness.device_layer(s, 0, 0, q4k=True)
    L = moe.Layer(harness.config_for(s, q4k=True), W, max_tokens=2)
    x = torch.from_numpy(synth.activations(0, 2, s.hidden)).cuda()
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_ffn_forward_noalloc(L.handle, x, None, 2, torch.empty_like(x))
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_SHAPE


# ------------------------------------------- the batched path with Q4_K (T > 32)

def _oracle_rows_q4k(s, seed, layer, x_np, tok_np, rows, router=True, prenorm=False):
    sub = synth.LayerShape(s.hidden, s.inter, s.shared_inter, s.n_experts, s.top_k, len(rows), vocab=s.vocab,
                           skew=s.skew)
    _, _, yref, _ = harness.oracle_layer(sub, seed, layer, x_np[rows], tok_np[rows], router=router, prenorm=prenorm,
                                         q4k=True)
    return yref


@pytest.mark.parametrize("T", [33, 64, 300])
def test_tiny_q4k_large_T(moe, T):
    s = synth.workload("tiny", tokens=T)
    got = _run_q4k(moe, s, 0, 0, T)
    yref = _oracle_rows_q4k(s, 0, 0, got["x"], got["tok"], np.arange(T))
    rel, mx = harness.errors(got["y"], yref)
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


def test_tiny_q4k_hash_prenorm_large_T(moe):
    s = synth.workload("tiny", tokens=100)
    got = _run_q4k(moe, s, 2, 1, 100, mode=moe.MOE_ROUTE_HASH, flags=moe.MOE_FLAG_PRENORM_RESIDUAL)
    yref = _oracle_rows_q4k(s, 2, 1, got["x"], got["tok"], np.arange(100), router=False, prenorm=True)
    rel, mx = harness.errors(got["y"], yref)
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


def test_full_q4k_512_tokens_every_row(moe):
    """V4-Flash shapes, 512 tokens with the skewed bias, Q4_K experts: every
    output row against the oracle (dense route)."""
    s = synth.workload("prefill_t4096", tokens=512)
    got = _run_q4k(moe, s, 3, 38, 512)
    _, _, yref, _ = harness.oracle_layer_dense(s, 3, 38, got["x"], q4k=True)
    rel, mx = harness.errors(got["y"], yref)
    print(f"q4k T=512 every row: rel_l2={rel:.3e} max_abs_frac={mx:.3e}")
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


def test_q2q4_stack_tail_teacher_forced(moe):
    """Layers 35-42 of the q2-q4 stack (37-42 with Q4_K routed experts) at
    T = 8 with the pre-norm residual, each checked against the oracle on the
    GPU's own input to that layer."""
    import os
    s = synth.workload("stack43_t8_q2q4")
    seed, T = 0, s.tokens
    threads = max(1, min(32, os.cpu_count() or 1))
    x0 = synth.activations(seed, T, s.hidden, stream=4343)
    x = torch.from_numpy(x0).cuda()
    tok = synth.token_ids(seed, T, s.vocab, stream=4343)
    tokd = torch.from_numpy(tok).cuda()
    for l in range(35, s.layers):
        sl = s.layer_shape(l)
        W = synth.device_layer(seed, l, sl, q4k=sl.q4k)
        L = moe.Layer(harness.config_for(sl, None, moe.MOE_FLAG_PRENORM_RESIDUAL, q4k=sl.q4k), W, max_tokens=T)
        xin = x.cpu().numpy()
        idx, _ = L.route(x, tokd)
        x = L.forward(x, tokd, y=x)
        torch.cuda.synchronize()
        L.poll()
        ridx, _, yref, margin = harness.oracle_layer(sl, seed, l, xin, tok, prenorm=True, threads=threads, q4k=sl.q4k)
        assert np.array_equal(idx.cpu().numpy(), ridx), (l, margin)
        rel, mx = harness.errors(x.cpu().numpy(), yref)
        assert rel <= harness.GEMV_REL_L2 and mx <= harness.MAX_ABS_FRAC, (l, rel, mx)
        del L, W
