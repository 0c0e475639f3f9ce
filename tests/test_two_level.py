"""The in-GPU two-level scan over the sequence ("s6_reset" blog draft, Associative
Boundary Resetting: the recurrence composes associatively, so segments of one sequence
can be scanned in parallel and joined).  Shapes with few channel groups and long
sequences take it when the workspace has ss_scan_workspace_bytes(); every output and
the final state are checked against the float64 oracle, and against the single-pass
schedule within rounding."""
import pytest
import torch

from gpu_util import SCAN_KEYS, TOL, assert_close, dev, gpu_scan, schedule
from selective_state_space_18_b200 import ssscan
from selective_state_space_18_b200.inputs import make_scan_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


def _plan(bt, ch, L, dtype):
    return ssscan.ss_scan_plan(bt, ch, 16, L, torch.bfloat16 if dtype == "bf16" else torch.float32)


@pytest.mark.parametrize("ch", [512, 1024])
@pytest.mark.parametrize("resets", [False, True])
def test_batch1_long_sequences(orc, ch, resets):
    """batch 1 x 512 / 1024 channels x 65536 tokens, bf16, z gate: every output."""
    bt, L = 1, 65536
    assert _plan(bt, ch, L, "bf16")["two_level"] == 1
    inp = make_scan_inputs(bt, ch, 16, L, "bf16", seed=1100 + ch, reset_mean_doc=512 if resets else 0,
                           a_perturb=True)
    y, h = gpu_scan(inp)
    ref = orc.scan(**inp)
    assert_close(y, ref["y"], 1e-2, "y")
    assert_close(h, ref["h_last"], 1e-2, "h_last")


CASES = [
    # batch, channels, seq, dtype, resets, h0
    (2, 64, 4096, "f32", False, True),
    (1, 40, 5000, "bf16", True, True),     # channel tail, ragged sequence (plain loads)
    (3, 16, 2048, "f32", True, False),     # a reset on many segment starts
    (1, 100, 8192, "bf16", False, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_small_shapes_against_oracle_and_single_pass(orc, case):
    bt, ch, L, dtype, resets, h0 = case
    assert _plan(bt, ch, L, dtype)["two_level"] == 1
    inp = make_scan_inputs(bt, ch, 16, L, dtype, seed=1200 + L + ch, h0=h0,
                           reset_mean_doc=300 if resets else 0, a_perturb=True)
    y, h = gpu_scan(inp)                     # the cached workspace: two-level
    y1, h1 = gpu_scan(inp, workspace=False)  # one CTA per channel group: single pass
    ref = orc.scan(**inp)
    tol = TOL[inp["x"].dtype]
    assert_close(y, ref["y"], tol, "y")
    assert_close(h, ref["h_last"], tol, "h_last")
    assert_close(y, y1.double().numpy(), tol, "y against the single pass")


def test_every_segment_start_is_a_reset(orc):
    """Resets exactly on the segment boundaries: each segment's decay is 0, so the
    entering states are discarded and each segment stands alone."""
    bt, ch, L = 1, 32, 4096
    p = _plan(bt, ch, L, "f32")
    assert p["two_level"] == 1
    inp = make_scan_inputs(bt, ch, 16, L, "f32", seed=1300, h0=True)
    mask = torch.zeros(bt, L, dtype=torch.uint8)
    mask[:, ::p["seg_len"]] = 1
    inp["reset"] = mask
    y, h = gpu_scan(inp)
    ref = orc.scan(**inp)
    assert_close(y, ref["y"], 1e-4, "y")
    assert_close(h, ref["h_last"], 1e-4, "h_last")


def test_workspace_without_room_for_composites_takes_the_single_pass(orc):
    """A workspace smaller than ss_scan_workspace_bytes is refused; one of that size
    runs the two-level schedule, and leaves itself ready for the next call."""
    bt, ch, L = 1, 64, 4096
    inp = make_scan_inputs(bt, ch, 16, L, "bf16", seed=1400)
    d = dev(inp, SCAN_KEYS)
    need = int(ssscan.load_library().ss_scan_workspace_bytes(bt, ch, 16, L))
    small = torch.zeros(need - 1, dtype=torch.uint8, device="cuda")
    with pytest.raises(ssscan.SSError, match="SS_ERR_WORKSPACE"):
        ssscan.ss_scan_fwd(**d, workspace=small)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    y, h = ssscan.ss_scan_fwd(**d, workspace=ws)
    torch.cuda.synchronize()
    ref = orc.scan(**inp)
    assert_close(y.cpu(), ref["y"], 1e-2, "y")
    assert_close(h.cpu(), ref["h_last"], 1e-2, "h_last")
    # a second call on the same workspace (the counter and epoch were left ready)
    y2, h2 = ssscan.ss_scan_fwd(**d, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y, y2) and torch.equal(h, h2)


FORCED = [
    # batch, channels, seq, dtype, resets, layout
    (2, 700, 2048, "bf16", True, 4),   # many groups, forced onto the two-level schedule
    (1, 320, 4096, "bf16", False, 2),
    (3, 33, 1031, "f32", True, 4),     # ragged everything
    (1, 16, 1024, "f32", False, 2),    # exactly two segments
]


@pytest.mark.parametrize("case", FORCED, ids=lambda c: "x".join(map(str, c)))
def test_forced_two_level_against_oracle(orc, case):
    bt, ch, L, dtype, resets, spl = case
    inp = make_scan_inputs(bt, ch, 16, L, dtype, seed=1500 + L + ch, h0=True,
                           reset_mean_doc=200 if resets else 0, a_perturb=True)
    with schedule(two_level=2, layout=spl):
        p = _plan(bt, ch, L, dtype)
        assert p["two_level"] == 1 and p["states_per_lane"] == spl and p["segments"] >= 2
        y, h = gpu_scan(inp)
    ref = orc.scan(**inp)
    tol = TOL[inp["x"].dtype]
    assert_close(y, ref["y"], tol, "y")
    assert_close(h, ref["h_last"], tol, "h_last")
