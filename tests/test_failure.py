"""Failure detection without a GPU fault: a device-side wait that can never be
satisfied must end on its time limit, report SS_ERR_TIMEOUT through the status word,
and leave the CUDA context usable.

The wait is made unsatisfiable on the host side: the workspace's work counter is set
past the first sequence segment, so every unit waits for a carry flag that no CTA will
ever publish.  The wait limit is shortened to 2 ms for the duration of the test only."""
import pytest
import torch

from selective_state_space_18_b200 import ssscan
from selective_state_space_18_b200.inputs import make_scan_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


def test_unsatisfiable_carry_wait_times_out_and_recovers():
    bt, ch, n, L = 1, 64, 16, 8192
    inp = make_scan_inputs(bt, ch, n, L, "bf16", seed=3)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    need = int(ssscan.load_library().ss_scan_workspace_bytes(bt, ch, n, L))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    groups = ch // 16  # 16 channels per CTA at state_dim 16
    # first 4 bytes of the workspace: the call's next work unit
    ws[:4] = torch.tensor([groups], dtype=torch.int32, device="cuda").view(torch.uint8)
    ssscan.ss_debug_set_wait_limit(2000)  # 2 ms
    try:
        ssscan.ss_scan_fwd(**d, workspace=ws)
        assert ssscan.ss_scan_status(ws) == "SS_ERR_TIMEOUT"
        # the status word is cleared by the read
        assert ssscan.ss_scan_status(ws) == "SS_OK"
    finally:
        ssscan.ss_debug_set_wait_limit(0)
    # the context is healthy: a fresh workspace gives the normal answer
    ws.zero_()
    y1, h1 = ssscan.ss_scan_fwd(**d, workspace=ws)
    y0, h0 = ssscan.ss_scan_fwd(**d, workspace=False)
    torch.cuda.synchronize()
    assert ssscan.ss_scan_status(ws) == "SS_OK"
    assert torch.equal(y1, y0) and torch.equal(h1, h0)
