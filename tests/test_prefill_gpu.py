"""Parity of the large-T path (T > 32: certified router, permutation, tcgen05
grouped GEMMs with f16/bf16 operands) against the fp64 oracle, through the C
ABI; the full-shape 32-token case runs on the small-T path."""
import numpy as np
import pytest

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


def _forward(moe, s, seed, layer, T, mode=0, flags=0):
    router = mode == moe.MOE_ROUTE_ROUTER
    W = harness.device_layer(s, seed, layer, router=router)
    L = moe.Layer(harness.config_for(s, mode, flags), W, max_tokens=T)
    x_np = synth.activations(seed, T, s.hidden, stream=layer)
    tok_np = synth.token_ids(seed, T, s.vocab, stream=layer)
    x = torch.from_numpy(x_np).cuda()
    tok = torch.from_numpy(tok_np).cuda()
    y = L.forward(x, tok)
    torch.cuda.synchronize()
    L.poll()
    return x_np, tok_np, y.cpu().numpy(), L


def _oracle_rows(s, seed, layer, x_np, tok_np, rows, router=True, prenorm=False):
    sub = synth.LayerShape(s.hidden, s.inter, s.shared_inter, s.n_experts, s.top_k, len(rows), vocab=s.vocab,
                           skew=s.skew)
    _, _, yref, _ = harness.oracle_layer(sub, seed, layer, x_np[rows], tok_np[rows], router=router,
                                         prenorm=prenorm)
    return yref


# 2100 tokens: the router GEMM's 128-token tiles with a ragged last tile
@pytest.mark.parametrize("T", [9, 64, 300, 2100])
def test_tiny_shapes_large_T(moe, T):
    s = synth.workload("tiny", tokens=T)
    x, tok, y, _ = _forward(moe, s, 0, 0, T)
    yref = _oracle_rows(s, 0, 0, x, tok, np.arange(T))
    rel, mx = harness.errors(y, yref)
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


def test_tiny_hash_prenorm_large_T(moe):
    s = synth.workload("tiny", tokens=100)
    x, tok, y, _ = _forward(moe, s, 2, 1, 100, mode=moe.MOE_ROUTE_HASH, flags=moe.MOE_FLAG_PRENORM_RESIDUAL)
    yref = _oracle_rows(s, 2, 1, x, tok, np.arange(100), router=False, prenorm=True)
    rel, mx = harness.errors(y, yref)
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


def test_decode32_full_shape(moe):
    """A second 32-token full-shape call (another seed and layer): it runs on
    the small-T kernels, so every row is held to the GEMV tolerance."""
    s = synth.workload("decode_t32")
    x, tok, y, _ = _forward(moe, s, 1, 2, 32)
    _, _, yref, _ = harness.oracle_layer_dense(s, 1, 2, x)
    rel, mx = harness.errors(y, yref)
    print(f"decode_t32 rel_l2={rel:.3e} max_abs_frac={mx:.3e}")
    assert rel <= harness.GEMV_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


def test_prefill_4096_every_row(moe):
    """The full prefill call (4096 tokens, skewed bias): every output row
    against the oracle (dense route).  The busiest and the quietest expert
    and an expert whose token count is not a multiple of the 256-column N
    tile are checked on their own tokens as well."""
    s = synth.workload("prefill_t4096")
    x, tok, y, L = _forward(moe, s, 0, 0, 4096)
    assert np.all(np.isfinite(y))
    idx_g, _ = L.route(torch.from_numpy(x).cuda())
    idx_g = idx_g.cpu().numpy()
    idx, _, yref, margin = harness.oracle_layer_dense(s, 0, 0, x)
    assert np.array_equal(idx_g, idx), margin
    counts = np.bincount(idx.ravel(), minlength=s.n_experts)
    rel, mx = harness.errors(y, yref)
    print(f"prefill_t4096 every row: rel_l2={rel:.3e} max_abs_frac={mx:.3e} "
          f"tokens/expert min {counts.min()} max {counts.max()}")
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)
    busiest = int(counts.argmax())
    quietest = int(np.argmin(np.where(counts > 0, counts, 1 << 30)))
    ragged = [e for e in np.argsort(-counts) if counts[e] > 256 and counts[e] % 256][:1]
    assert ragged, counts.max()
    for e in [busiest, quietest] + ragged:
        rows = np.nonzero((idx == e).any(1))[0]
        r, m = harness.errors(y[rows], yref[rows])
        assert r <= harness.MMA_REL_L2 and m <= harness.MAX_ABS_FRAC, (e, counts[e], r, m)


@pytest.mark.parametrize("name,T", [("tiny", 300), ("prefill_t4096", 4096)])
def test_deterministic_flag_repeats_bitwise(moe, name, T):
    """MOE_FLAG_DETERMINISTIC: the routed outputs are summed per token in
    ascending expert id, so two calls give the same bits; the result stays
    within the tensor-core tolerance of the oracle (tiny) and of the
    atomic-add combine (full shape)."""
    s = synth.workload(name, tokens=T)
    W = harness.device_layer(s, 2, 5)
    x_np = synth.activations(2, T, s.hidden, stream=5)
    x = torch.from_numpy(x_np).cuda()
    Ld = moe.Layer(harness.config_for(s, flags=moe.MOE_FLAG_DETERMINISTIC), W, max_tokens=T)
    y1 = Ld.forward(x).cpu().numpy()
    y2 = Ld.forward(x).cpu().numpy()
    Ld.poll()
    assert np.array_equal(y1.view(np.uint32), y2.view(np.uint32))
    if name == "tiny":
        _, _, yref, _ = harness.oracle_layer(s, 2, 5, x_np)
    else:
        La = moe.Layer(harness.config_for(s), W, max_tokens=T)
        yref = La.forward(x).cpu().numpy()
        La.poll()
    rel, mx = harness.errors(y1, yref)
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


def _tma_maps_written(L, s):
    """Whether the handle holds the batched path's tensor maps: they sit in
    the persist buffer after the 256-byte header and the E router-row norms,
    at the next 64-byte boundary (three 128-byte maps)."""
    base = L.persist.data_ptr()
    off = ((base + 256 + 4 * s.n_experts + 63) & ~63) - base
    return bool(L.persist[off:off + 384].any().item())


@pytest.mark.parametrize("flags", ["det", "atomic"])
def test_tma_staged_tiles_match_plain_loads(moe, monkeypatch, flags):
    """TMA staging of the packed IQ2_XXS / Q2_K tiles (rows of 528 and 336
    bytes: a 16-byte multiple, so the tensor maps exist) against producers
    that load the packed bytes themselves (MOE_GEMM_TMA=0 at init): the same
    decoded tiles and MMA order, so with the deterministic combine the outputs
    are bitwise equal, and without it equal up to the order of the atomic
    adds; both agree with the oracle.  16 experts, 300 tokens: several tiles
    per expert, ragged last tiles, 8 blocks per gate/up row and 4 per down row
    (every block offset from a 16-byte boundary occurs)."""
    s = synth.LayerShape(2048, 1024, 512, 16, 2, 300, vocab=1024)
    T = s.tokens
    W = harness.device_layer(s, 8, 2)
    x_np = synth.activations(8, T, s.hidden, stream=2)
    x = torch.from_numpy(x_np).cuda()
    fl = moe.MOE_FLAG_DETERMINISTIC if flags == "det" else 0
    Lt = moe.Layer(harness.config_for(s, flags=fl), W, max_tokens=T)
    monkeypatch.setenv("MOE_GEMM_TMA", "0")
    Lp = moe.Layer(harness.config_for(s, flags=fl), W, max_tokens=T)
    monkeypatch.delenv("MOE_GEMM_TMA")
    assert _tma_maps_written(Lt, s)
    yt = Lt.forward(x).cpu().numpy()
    yp = Lp.forward(x).cpu().numpy()
    Lt.poll()
    Lp.poll()
    if flags == "det":
        assert np.array_equal(yt.view(np.uint32), yp.view(np.uint32))
    else:
        np.testing.assert_allclose(yt, yp, rtol=1e-5, atol=1e-5 * float(np.abs(yp).max()))
    _, _, yref, _ = harness.oracle_layer_dense(s, 8, 2, x_np)
    rel, mx = harness.errors(yt, yref)
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


@pytest.mark.parametrize("name,T", [("tiny", 300), ("prefill_t4096", 4096)])
def test_dense_shared_expert_matches_per_tile_decoding(moe, monkeypatch, name, T):
    """From 257 tokens the shared expert's Q8_0 rows are expanded to 16 bits
    once per call and multiplied by TMA-fed GEMMs; its operands, tiles and
    MMA order are those of the per-tile decoding path (MOE_SHARED_DENSE=0 at
    init), so with the deterministic combine the outputs are the same bits.
    The tiny case is also checked against the oracle."""
    s = synth.workload(name, tokens=T)
    W = harness.device_layer(s, 9, 4)
    x_np = synth.activations(9, T, s.hidden, stream=4)
    x = torch.from_numpy(x_np).cuda()
    fl = moe.MOE_FLAG_DETERMINISTIC | moe.MOE_FLAG_PRENORM_RESIDUAL
    Ld = moe.Layer(harness.config_for(s, flags=fl), W, max_tokens=T)
    monkeypatch.setenv("MOE_SHARED_DENSE", "0")
    Lp = moe.Layer(harness.config_for(s, flags=fl), W, max_tokens=T)
    monkeypatch.delenv("MOE_SHARED_DENSE")
    yd = Ld.forward(x).cpu().numpy()
    yp = Lp.forward(x).cpu().numpy()
    Ld.poll()
    Lp.poll()
    assert np.array_equal(yd.view(np.uint32), yp.view(np.uint32))
    if name == "tiny":
        _, _, yref, _ = harness.oracle_layer(s, 9, 4, x_np, prenorm=True)
        rel, mx = harness.errors(yd, yref)
        assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)
