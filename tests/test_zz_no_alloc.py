"""ss_scan_fwd_static_scratch: the prompt scan with the library's fixed per-device
scratch in place of a caller workspace.  It must give the answer of ss_scan_fwd with
a workspace, on two calls in a row (the first call leaves the scratch ready for the
second), allocate no device memory, and refuse shapes beyond the scratch's size
before launching anything.

This file is collected last so that the scratch's first use also happens after
every other test in a full run; it passes alone as well."""
import ctypes

import pytest
import torch

from selective_state_space_18_b200 import build as ssbuild
from selective_state_space_18_b200 import ssscan
from selective_state_space_18_b200.inputs import make_scan_inputs

from gpu_util import SCAN_KEYS, TOL, assert_close, dev


def test_shape_beyond_scratch_is_refused_before_launch():
    """Host-side check only (fake pointers, never dereferenced): 993 channel groups
    of 16 need more than 1 MiB of workspace."""
    ssbuild.build()
    lib = ssscan.load_library()
    P = [ctypes.c_void_p(0x7f0000000000 + i * 0x100000000) for i in range(6)]
    ch = 16 * 993
    assert lib.ss_scan_workspace_bytes(1, ch, 16, 64) > ssscan.SS_STATIC_SCRATCH_BYTES
    assert lib.ss_scan_workspace_bytes(1, ch - 16, 16, 64) <= ssscan.SS_STATIC_SCRATCH_BYTES
    out = ctypes.c_void_p(0)
    st = lib.ss_scan_fwd_static_scratch(1, ch, 16, 64, ssscan.SS_BF16, P[0], P[1], P[2], P[3], P[4],
                                        None, None, None, None, None, 1, P[5], None, ctypes.byref(out),
                                        None)
    assert ssscan.STATUS[st] == "SS_ERR_SCRATCH_LIMIT"
    assert out.value is None  # nothing was set up
    assert b"SS_STATIC_SCRATCH_BYTES" in lib.ss_status_string(st)
    # unknown flag bits are refused too
    st = lib.ss_scan_fwd_static_scratch(1, 16, 16, 64, ssscan.SS_BF16, P[0], P[1], P[2], P[3], P[4],
                                        None, None, None, None, None, 4, P[5], None, None, None)
    assert ssscan.STATUS[st] == "SS_ERR_UNSUPPORTED"


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,resets", [("bf16", True), ("f32", False)])
def test_static_scratch_matches_workspace_call_twice(orc, dtype, resets):
    """Two calls in a row, each against ss_scan_fwd with a workspace (the entry point
    this one stands in for) and against the float64 oracle."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    bt, ch, n, L = 2, 320, 16, 3000  # 40 groups, ragged sequence tail
    inp = make_scan_inputs(bt, ch, n, L, dtype, seed=77, reset_mean_doc=500 if resets else 0, h0=True)
    d = dev(inp, SCAN_KEYS)
    y_ref, h_ref = ssscan.ss_scan_fwd(**d, workspace=True)
    tol = TOL[y_ref.dtype]
    ref = orc.scan(**inp)
    y_out = torch.empty_like(y_ref)
    h_out = torch.empty_like(h_ref)
    for call in range(2):
        y_out.fill_(float("nan"))
        h_out.fill_(float("nan"))
        free0 = torch.cuda.mem_get_info()[0]
        ssscan.ss_scan_fwd_static_scratch(**d, y=y_out, h_last=h_out)
        torch.cuda.synchronize()
        if call == 1:  # after the first call's one-time set-up, no device memory moves
            assert torch.cuda.mem_get_info()[0] == free0
        assert ssscan.static_scratch_status() == "SS_OK"
        assert_close(y_out.cpu(), y_ref.cpu().double().numpy(), tol, f"y, call {call}")
        assert_close(h_out.cpu(), h_ref.cpu().double().numpy(), 1e-4, f"h_last, call {call}")
        assert_close(y_out.cpu(), ref["y"], tol, f"y vs oracle, call {call}")
        assert_close(h_out.cpu(), ref["h_last"], tol, f"h_last vs oracle, call {call}")


@pytest.mark.gpu
def test_static_scratch_zero_flag_and_chaining(orc):
    """SS_SCRATCH_ZERO clears the scratch before the scan; a prompt split in two
    calls chained through h_last equals one call, and the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    bt, ch, n, L = 1, 512, 16, 4096
    inp = make_scan_inputs(bt, ch, n, L, "f32", seed=5)
    d = dev(inp, SCAN_KEYS)
    ref_o = orc.scan(**inp)
    y_all, h_all = ssscan.ss_scan_fwd_static_scratch(**d, zero_scratch=True)
    half = {k: (v[..., : L // 2].contiguous() if k in ("x", "dt", "z", "B", "C") and v is not None else v)
            for k, v in d.items()}
    rest = {k: (v[..., L // 2:].contiguous() if k in ("x", "dt", "z", "B", "C") and v is not None else v)
            for k, v in d.items()}
    y1, h1 = ssscan.ss_scan_fwd_static_scratch(**half)
    rest["h0"] = h1
    y2, h2 = ssscan.ss_scan_fwd_static_scratch(**rest)
    torch.cuda.synchronize()
    assert ssscan.static_scratch_status() == "SS_OK"
    ref = y_all.cpu().double().numpy()
    assert_close(torch.cat([y1, y2], -1).cpu(), ref, 1e-4, "chained y")
    assert_close(h2.cpu(), h_all.cpu().double().numpy(), 1e-4, "chained h_last")
    assert_close(y_all.cpu(), ref_o["y"], 1e-4, "y vs oracle")
    assert_close(h_all.cpu(), ref_o["h_last"], 1e-4, "h_last vs oracle")


@pytest.mark.gpu
def test_zero_flag_clears_carry_flags_of_a_larger_shape():
    """SS_SCRATCH_ZERO must clear the carry flags a LARGER earlier call left beyond the
    current shape's part of the scratch: the epoch restarts at zero, and a flag left
    by that earlier call at epoch zero would otherwise satisfy a later call's wait
    with a stale carry.  Large call A at epoch 0, a zeroing small call, then a zeroing
    large call B (epoch 0 again) on other inputs: B must equal ss_scan_fwd's single
    pass."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    big = (1, 2048, 16, 4096)   # 128 channel groups, several segments each
    small = (1, 64, 16, 512)    # 4 groups: its part of the scratch is a small prefix
    a = dev(make_scan_inputs(*big, "bf16", seed=11), SCAN_KEYS)
    s = dev(make_scan_inputs(*small, "bf16", seed=12), SCAN_KEYS)
    b = dev(make_scan_inputs(*big, "bf16", seed=13), SCAN_KEYS)
    # (the static scratch runs the single-pass schedule, which one CTA per channel group
    # reproduces bit for bit)
    y_ref, h_ref = ssscan.ss_scan_fwd(**b, workspace=False)
    ssscan.ss_scan_fwd_static_scratch(**a, zero_scratch=True)
    ssscan.ss_scan_fwd_static_scratch(**s, zero_scratch=True)
    y_b, h_b = ssscan.ss_scan_fwd_static_scratch(**b, zero_scratch=True)
    torch.cuda.synchronize()
    assert ssscan.static_scratch_status() == "SS_OK"
    assert torch.equal(y_b, y_ref) and torch.equal(h_b, h_ref)
