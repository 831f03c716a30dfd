"""GPU checks for the Q4_K routed-expert variant (the q2-q4 build's upgraded
layers): the device fill of the seeded generator is byte-identical to the
host fill the oracle reads."""
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
