"""The index-checked debug build (libssscan_bounds.so, compiled with SS_BOUNDS_CHECK):
every runtime-computed global and shared-memory index of the scan and decode kernels
is checked before its access.  On ragged, unaligned and small shapes, in every form
and schedule, no check may fail, and the outputs must equal the normal build's within
rounding (the checks skip nothing when they pass and change no operation, but the
compiler may contract multiply-adds differently in the checked build)."""
import ctypes

import pytest
import torch

from gpu_util import SCAN_KEYS, UPDATE_KEYS, dev, schedule
from selective_state_space_18_b200 import build as ssbuild
from selective_state_space_18_b200 import ssscan
from selective_state_space_18_b200.inputs import make_scan_inputs, make_update_inputs


def test_normal_build_reports_no_checks():
    ssbuild.build()
    lib = ssscan.load_library()
    site = ctypes.c_int(0)
    assert lib.ss_debug_bounds_status(None, ctypes.byref(site)) == 5 and site.value == -1


@pytest.fixture(scope="module")
def checked():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    path = ssbuild.build(bounds_check=True)
    normal = ssscan.load_library()
    with ssscan._lock:
        ssscan._lib = None
    lib = ssscan.load_library(path)
    try:
        yield normal, lib
    finally:
        with ssscan._lock:
            ssscan._lib = normal


def _site(lib):
    site = ctypes.c_int(-2)
    assert lib.ss_debug_bounds_status(None, ctypes.byref(site)) == 0
    return site.value


def _run_both(checked, fn):
    normal, lib = checked
    out_checked = fn()
    torch.cuda.synchronize()
    assert _site(lib) == 0, "an index check failed"
    with ssscan._lock:
        ssscan._lib = normal
    try:
        out_normal = fn()
        torch.cuda.synchronize()
    finally:
        with ssscan._lock:
            ssscan._lib = lib
    for a, b in zip(out_checked, out_normal):
        if a is not None:
            tol = 1e-2 if a.dtype == torch.bfloat16 else 1e-4
            d = (a.double() - b.double()).abs() / (1.0 + b.double().abs())
            assert torch.isfinite(a).all() and float(d.max()) <= tol


SHAPES = [
    # batch, channels, N, seq, dtype, resets
    (1, 3, 4, 1, "f32", False),
    (2, 5, 8, 7, "bf16", True),
    (1, 17, 16, 100, "bf16", False),
    (3, 33, 16, 65, "f32", True),
    (2, 70, 4, 129, "bf16", True),
    (1, 40, 16, 4100, "bf16", True),   # ragged, long enough for the two-level schedule
    (2, 100, 16, 2048, "bf16", False), # tile-load path
]


@pytest.mark.gpu
@pytest.mark.parametrize("shape", SHAPES, ids=lambda c: "x".join(map(str, c)))
@pytest.mark.parametrize("layout", [2, 4])
def test_scan_forms_pass_every_check(checked, shape, layout):
    bt, ch, n, L, dtype, resets = shape
    inp = make_scan_inputs(bt, ch, n, L, dtype, seed=1700 + L + ch, h0=True, reset_mean_doc=40 if resets else 0)
    d = dev(inp, SCAN_KEYS)
    g = torch.Generator().manual_seed(1701)
    w = (torch.randn(ch, 4, generator=g) * 0.5).cuda()
    cs = torch.randn(bt, ch, 3, generator=g).cuda()
    with schedule(layout=layout):
        for two_level in (1, 2):
            with schedule(two_level=two_level, layout=layout):
                _run_both(checked, lambda: ssscan.ss_scan_fwd(**d))
                _run_both(checked, lambda: ssscan.ss_scan_fwd(**d, workspace=False))
        _run_both(checked, lambda: ssscan.ss_scan_fwd(**d, return_states=True))
        _run_both(checked, lambda: ssscan.ss_scan_fwd(**d, return_states=True, return_betas=True))
        _run_both(checked, lambda: ssscan.ss_scan_fwd(**d, return_betas=True))  # (y, h_last, None, betas)
        _run_both(checked, lambda: tuple(ssscan.ss_scan_fwd_conv(
            d["x"], w, d["dt"], d["A"], d["B"], d["C"], d["D"], d["z"], d["dt_bias"], d["reset"], d["h0"],
            conv_state=cs, return_x=True).values()))


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_unaligned_views_pass_every_check(checked, dtype):
    inp = make_scan_inputs(2, 24, 16, 96, dtype, seed=1710, reset_mean_doc=20)
    d = {}
    for k, v in inp.items():
        if v is None:
            d[k] = None
            continue
        buf = torch.empty(v.numel() + 1, dtype=v.dtype, device="cuda")
        d[k] = buf[1:].view(v.shape)
        d[k].copy_(v)
    _run_both(checked, lambda: ssscan.ss_scan_fwd(**d))


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [(3, 37, 4, "f32"), (2, 300, 16, "bf16"), (5, 64, 8, "bf16")])
def test_decode_passes_every_check(checked, shape):
    bt, ch, n, dtype = shape
    inp = make_update_inputs(bt, ch, n, dtype, seed=1720 + ch)

    def run():
        du = dev(inp, UPDATE_KEYS)
        y = ssscan.ss_state_update(**du)
        return y, du["state"]
    _run_both(checked, run)
