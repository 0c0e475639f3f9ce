"""The special-function-unit probe behind the scan's roofline: it runs and reports a
rate in results per SM clock within reach of the unit's nominal 16."""
import pytest
import torch

from selective_state_space_18_b200 import ssscan

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("op", ["ex2", "tanh"])
def test_mufu_probe_rate(op):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    rate, rates = ssscan.mufu_rate(op, iters=1 << 12)
    assert len(rates) == torch.cuda.get_device_properties(0).multi_processor_count
    assert 4.0 < rate < 17.0, rates
