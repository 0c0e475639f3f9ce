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
def test_static_scratch_matches_workspace_call_twice(dtype, resets):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    bt, ch, n, L = 2, 320, 16, 3000  # 40 groups, ragged sequence tail
    inp = make_scan_inputs(bt, ch, n, L, dtype, seed=77, reset_mean_doc=500 if resets else 0, h0=True)
    d = dev(inp, SCAN_KEYS)
    y_ref, h_ref = ssscan.ss_scan_fwd(**d, workspace=True)
    tol = TOL[y_ref.dtype]
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


@pytest.mark.gpu
def test_static_scratch_zero_flag_and_chaining():
    """SS_SCRATCH_ZERO clears the scratch before the scan; a prompt split in two
    calls chained through h_last equals one call."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    bt, ch, n, L = 1, 512, 16, 4096
    inp = make_scan_inputs(bt, ch, n, L, "f32", seed=5)
    d = dev(inp, SCAN_KEYS)
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
