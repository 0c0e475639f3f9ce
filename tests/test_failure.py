"""Failure detection without a GPU fault: a device-side wait that can never be
satisfied must end on its time limit, report SS_ERR_TIMEOUT through the status word,
and leave both the CUDA context and the workspace usable.

The wait is made unsatisfiable on the host side: the workspace's work counter is set
past the first sequence segment, so every unit waits for a carry flag that no CTA will
ever publish.  The wait limit is shortened to 2 ms for the duration of the test only."""
import pytest
import torch

from gpu_util import SCAN_KEYS, assert_close, dev, schedule
from selective_state_space_18_b200 import ssscan
from selective_state_space_18_b200.inputs import make_scan_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


@pytest.fixture(autouse=True)
def _single_pass():
    """The carry waits these tests block belong to the single-pass (chained) schedule;
    the two-level schedule has none."""
    with schedule(two_level=1):
        yield


def _block_first_segment(ws, groups):
    # first 4 bytes of the workspace: the call's next work unit
    ws[:4] = torch.tensor([groups], dtype=torch.int32, device=ws.device).view(torch.uint8)


def test_unsatisfiable_carry_wait_times_out_and_recovers(orc):
    bt, ch, n, L = 1, 64, 16, 8192
    inp = make_scan_inputs(bt, ch, n, L, "bf16", seed=3)
    d = dev(inp, SCAN_KEYS)
    need = int(ssscan.load_library().ss_scan_workspace_bytes(bt, ch, n, L))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    _block_first_segment(ws, ch // 16)  # 16 channels per CTA at state_dim 16
    ssscan.ss_debug_set_wait_limit(2000)  # 2 ms
    try:
        ssscan.ss_scan_fwd(**d, workspace=ws)
        assert ssscan.ss_scan_status(ws) == "SS_ERR_TIMEOUT"
        # the status word is cleared by the read
        assert ssscan.ss_scan_status(ws) == "SS_OK"
    finally:
        ssscan.ss_debug_set_wait_limit(0)
    # the same workspace, NOT zeroed again, gives the normal answer: the timed-out call
    # left it ready (its carry flags carry the old epoch)
    y1, h1 = ssscan.ss_scan_fwd(**d, workspace=ws)
    y0, h0 = ssscan.ss_scan_fwd(**d, workspace=False)
    torch.cuda.synchronize()
    assert ssscan.ss_scan_status(ws) == "SS_OK"
    assert torch.equal(y1, y0) and torch.equal(h1, h0)
    ref = orc.scan(**inp)
    assert_close(y1.cpu(), ref["y"], 1e-2, "y after recovery")
    assert_close(h1.cpu(), ref["h_last"], 1e-2, "h_last after recovery")


def test_default_cached_workspace_recovers_after_timeout(orc):
    """The binding's default path (workspace=True: one cached workspace per stream)
    keeps working after a timed-out call on it, with no re-zeroing by anyone."""
    bt, ch, n, L = 1, 96, 16, 6144
    inp = make_scan_inputs(bt, ch, n, L, "bf16", seed=4, reset_mean_doc=300)
    d = dev(inp, SCAN_KEYS)
    ws = ssscan.scan_workspace(bt, ch, n, L, torch.device("cuda", torch.cuda.current_device()))
    ssscan.ss_scan_fwd(**d)  # a normal call first: the cached workspace is in use
    torch.cuda.synchronize()
    _block_first_segment(ws, ch // 16)
    ssscan.ss_debug_set_wait_limit(2000)
    try:
        ssscan.ss_scan_fwd(**d)
        assert ssscan.ss_scan_status(ws) == "SS_ERR_TIMEOUT"
    finally:
        ssscan.ss_debug_set_wait_limit(0)
    assert ssscan.scan_workspace(bt, ch, n, L, ws.device) is ws  # still the cached one
    ref = orc.scan(**inp)
    for call in range(2):
        y, h = ssscan.ss_scan_fwd(**d)
        torch.cuda.synchronize()
        assert ssscan.ss_scan_status(ws) == "SS_OK"
        assert_close(y.cpu(), ref["y"], 1e-2, f"y, call {call} after the timeout")
        assert_close(h.cpu(), ref["h_last"], 1e-2, f"h_last, call {call} after the timeout")


def test_debug_status_reads_the_no_workspace_word():
    """ss_debug_status: the status word of calls made without a workspace (decode
    included) reads SS_OK after calls that completed."""
    inp = make_scan_inputs(1, 32, 16, 512, "bf16", seed=6)
    ssscan.ss_scan_fwd(**dev(inp, SCAN_KEYS), workspace=False)
    assert ssscan.ss_debug_status() == "SS_OK"
