"""The device-side timeout path.  Every wait a kernel makes on other warps'
results is bounded; moe_set_wait_limit shortens the bound to one clock cycle
so that, on an ordinary call, waits that are not satisfied at once run out.
The kernels then record MOE_ERR_TIMEOUT in the device error word and return
(no trap, no hang): the small-token kernel's waits for an h slice and for its
block's routing table, and the tensor-core kernel's role hand-offs.  The
next call with the default bound is correct."""
import time

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


def _expire(moe, L, x, tries=5):
    """Calls with the one-cycle bound until a wait has run out (the small-T
    kernel's waits race with its producers, so a call may find every flag
    already set); returns how many calls timed out."""
    timeouts = 0
    moe.moe_set_wait_limit(L.handle, 1)
    for _ in range(tries):
        t0 = time.time()
        L.forward(x)
        torch.cuda.synchronize()
        assert time.time() - t0 < 1.0  # nothing waited for the default bound
        try:
            L.poll()
        except moe.MoeError as e:
            assert e.status == moe.MOE_ERR_TIMEOUT, e
            timeouts += 1
            break
    moe.moe_set_wait_limit(L.handle, 0)
    L.poll()  # the word was cleared; the context is usable
    return timeouts


def test_small_token_waits_run_out_and_the_next_call_is_correct(moe):
    s = synth.workload("decode_t1")
    W = harness.device_layer(s, 5, 3)
    L = moe.Layer(harness.config_for(s), W, max_tokens=1)
    x_np = synth.activations(5, 1, s.hidden, stream=3)
    x = torch.from_numpy(x_np).cuda()
    y0 = L.forward(x).cpu().numpy()
    L.poll()
    assert _expire(moe, L, x) == 1
    y1 = L.forward(x).cpu().numpy()
    L.poll()
    assert np.array_equal(y0, y1)  # the small-T path is deterministic
    _, _, yref, _ = harness.oracle_layer(s, 5, 3, x_np)
    rel, mx = harness.errors(y1, yref)
    assert rel <= harness.GEMV_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


def test_tensor_core_hand_offs_run_out_and_the_next_call_is_correct(moe):
    s = synth.workload("tiny", tokens=300)
    W = harness.device_layer(s, 5, 4)
    L = moe.Layer(harness.config_for(s), W, max_tokens=300)
    x_np = synth.activations(5, 300, s.hidden, stream=4)
    x = torch.from_numpy(x_np).cuda()
    assert _expire(moe, L, x) == 1
    y = L.forward(x).cpu().numpy()
    L.poll()
    _, _, yref, _ = harness.oracle_layer(s, 5, 4, x_np)
    rel, mx = harness.errors(y, yref)
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)
