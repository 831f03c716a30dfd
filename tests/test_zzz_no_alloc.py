"""moe_ffn_forward_noalloc: the forward pass for callers that cannot allocate
device memory (a plugin whose host engine owns every device allocation, a
program with a fixed device-memory plan).  Its scratch lives in a buffer built
into the library instead of a caller-provided one.  This file is collected
last so that a run stopping at the first failure has run every other test.
"""
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


@pytest.mark.parametrize("name,T", [("tiny", 4), ("decode_t1", 1), ("decode_t1", 8)])
def test_noalloc_matches_scratch_forward_on_two_calls(moe, name, T):
    """Two calls in a row through the no-allocation entry point, each against
    the forward with caller scratch and against the fp64 oracle."""
    s = synth.workload(name, tokens=T)
    W = harness.device_layer(s, 6, 1)
    L = moe.Layer(harness.config_for(s), W, max_tokens=T)
    x_np = synth.activations(6, T, s.hidden, stream=1)
    x = torch.from_numpy(x_np).cuda()
    ref = L.forward(x).cpu().numpy()
    _, _, yref, _ = harness.oracle_layer_dense(s, 6, 1, x_np)
    rel, mx = harness.errors(ref, yref)
    assert rel <= harness.GEMV_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)
    for _ in range(2):
        y = torch.full_like(x, float("nan"))
        moe.moe_ffn_forward_noalloc(L.handle, x, None, T, y)
        torch.cuda.synchronize()
        L.poll()
        got = y.cpu().numpy()
        rel, mx = harness.errors(got, ref)
        assert rel <= harness.GEMV_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)
        rel, mx = harness.errors(got, yref)
        assert rel <= harness.GEMV_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


def test_noalloc_rejects_more_tokens_than_it_supports(moe):
    s = synth.workload("tiny", tokens=9)
    W = harness.device_layer(s, 0, 0)
    L = moe.Layer(harness.config_for(s), W, max_tokens=9)
    x = torch.zeros((9, s.hidden), device="cuda")
    y = torch.empty_like(x)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_ffn_forward_noalloc(L.handle, x, None, 9, y)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert "at most 8" in moe.moe_last_error() or "at most 8" in str(ei.value)
