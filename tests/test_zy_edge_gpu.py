"""Degenerate configurations of the method on the GPU, through the C ABI,
against the fp64 oracle: a single selected expert (k = 1), every expert
selected with the largest top-k the ABI takes (k = E = 8), on the small-token
path (T = 1, 5, 32) and the batched path (T = 40), with router and hash
routing.  Routing must match exactly; outputs within the path's tolerance."""
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


CASES = [(16, 1), (8, 8)]  # (n_experts, top_k)


@pytest.mark.parametrize("E,k", CASES)
@pytest.mark.parametrize("T", [1, 5, 32, 40])
@pytest.mark.parametrize("router", [True, False])
def test_degenerate_top_k(moe, E, k, T, router):
    s = synth.workload("tiny", n_experts=E, top_k=k, tokens=T)
    seed, layer = 4, 2
    mode = moe.MOE_ROUTE_ROUTER if router else moe.MOE_ROUTE_HASH
    W = harness.device_layer(s, seed, layer, router=router)
    L = moe.Layer(harness.config_for(s, mode), W, max_tokens=T)
    x_np = synth.activations(seed, T, s.hidden, stream=layer)
    tok_np = synth.token_ids(seed, T, s.vocab, stream=layer)
    x = torch.from_numpy(x_np).cuda()
    tok = torch.from_numpy(tok_np).cuda()
    y = L.forward(x, tok)
    idx, w = L.route(x, tok)
    torch.cuda.synchronize()
    L.poll()
    ridx, rw, yref, margin = harness.oracle_layer(s, seed, layer, x_np, tok_np, router=router)
    assert np.array_equal(idx.cpu().numpy(), ridx), margin
    assert np.allclose(w.cpu().numpy(), rw, rtol=1e-6, atol=1e-7)
    if k == E:
        assert np.array_equal(ridx, np.tile(np.arange(E, dtype=np.int32), (T, 1)))
    rel, mx = harness.errors(y.cpu().numpy(), yref)
    tol = harness.GEMV_REL_L2 if T <= moe.MOE_SMALL_T_MAX else harness.MMA_REL_L2
    assert rel <= tol and mx <= harness.MAX_ABS_FRAC, (rel, mx)
