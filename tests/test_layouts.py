"""The two layouts of the state_dim-16 prompt scan -- two and four state rows per scan
lane -- each forced on shapes where the automatic choice would not pick it, against
the float64 oracle: the plain, segmented, per-token-states and fused-conv forms, the
tile-load and the ragged paths, resets, h0 and chaining.  Within one layout the forms
stay bit-identical to each other."""
import contextlib

import pytest
import torch

from gpu_util import SCAN_KEYS, TOL, assert_close, dev, gpu_scan, schedule
from selective_state_space_18_b200 import ssscan
from selective_state_space_18_b200.inputs import make_scan_inputs, make_workload


@contextlib.contextmanager
def layout(spl):
    ssscan.ss_debug_set_scan_layout(spl)
    try:
        yield
    finally:
        ssscan.ss_debug_set_scan_layout(0)


def test_layout_setter_rejects_other_values():
    from selective_state_space_18_b200 import build as ssbuild
    ssbuild.build()
    lib = ssscan.load_library()
    assert lib.ss_debug_set_scan_layout(3) == 5
    assert lib.ss_debug_set_scan_layout(8) == 5
    assert lib.ss_debug_set_scan_layout(0) == 0


CASES = [
    # batch, channels, seq, dtype, resets, h0
    (1, 17, 100, "bf16", False, True),     # channel tail inside one group, ragged seq
    (3, 33, 65, "f32", True, True),
    (2, 16, 130, "bf16", True, False),
    (1, 48, 513, "f32", False, True),
    (2, 100, 1000, "bf16", True, True),    # tile-load path, channel tail
    (1, 96, 3001, "bf16", True, False),    # ragged path at a size with many chunks
    (1, 256, 4096, "bf16", False, True),   # several groups, many segments
]


@pytest.mark.gpu
@pytest.mark.parametrize("spl", [2, 4])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_layout_matches_oracle(orc, spl, case):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    bt, ch, L, dtype, resets, h0 = case
    inp = make_scan_inputs(bt, ch, 16, L, dtype, seed=900 + L + ch, h0=h0,
                           reset_mean_doc=60 if resets else 0, a_perturb=True)
    ref = orc.scan(**inp)
    tol = TOL[inp["x"].dtype]
    with layout(spl), schedule(two_level=1):
        y_seg, h_seg = gpu_scan(inp, workspace=True)
        y_one, h_one = gpu_scan(inp, workspace=False)
    assert_close(y_seg, ref["y"], tol, "y")
    assert_close(h_seg, ref["h_last"], tol, "h_last")
    # the segmented schedule passes the exact carry: bit-identical to one CTA per group
    assert torch.equal(y_seg, y_one) and torch.equal(h_seg, h_one)


@pytest.mark.gpu
@pytest.mark.parametrize("spl", [2, 4])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_layout_states_form(orc, spl, dtype):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    inp = make_scan_inputs(2, 40, 16, 264 if dtype == "bf16" else 100, dtype, seed=931, h0=True,
                           reset_mean_doc=30)
    ref = orc.scan(**inp, return_states=True)
    d = dev(inp, SCAN_KEYS)
    with layout(spl):
        y0, h0 = ssscan.ss_scan_fwd(**d)
        y1, h1, hall = ssscan.ss_scan_fwd(**d, return_states=True)
        torch.cuda.synchronize()
    assert torch.equal(y0, y1) and torch.equal(h0, h1)
    assert_close(hall.cpu(), ref["h_all"], 1e-4, "h_all")
    assert_close(y1.cpu(), ref["y"], TOL[inp["x"].dtype], "y")
    assert torch.equal(hall[:, :, -1, :], h1)


@pytest.mark.gpu
@pytest.mark.parametrize("spl", [2, 4])
def test_layout_conv_form(orc, spl):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    bt, ch, L, K = 2, 72, 530, 4
    inp = make_scan_inputs(bt, ch, 16, L, "bf16", seed=940, h0=True, reset_mean_doc=90)
    g = torch.Generator().manual_seed(941)
    conv_w = torch.randn(ch, K, generator=g) * 0.5
    conv_b = torch.randn(ch, generator=g) * 0.1
    conv_state = torch.randn(bt, ch, K - 1, generator=g)
    cv = orc.conv_silu(inp["x"], conv_w, conv_b, conv_state)
    ref = orc.scan(x=cv["x"], dt=inp["dt"], A=inp["A"], B=inp["B"], C=inp["C"], D=inp["D"], z=inp["z"],
                   dt_bias=inp["dt_bias"], reset=inp["reset"], h0=inp["h0"])
    d = dev(inp, SCAN_KEYS)
    with layout(spl):
        out = ssscan.ss_scan_fwd_conv(d["x"], conv_w.cuda(), d["dt"], d["A"], d["B"], d["C"], d["D"], d["z"],
                                      d["dt_bias"], d["reset"], d["h0"], conv_b=conv_b.cuda(),
                                      conv_state=conv_state.cuda(), return_x=True)
        torch.cuda.synchronize()
    assert_close(out["y"].cpu(), ref["y"], 1e-2, "y")
    assert_close(out["h_last"].cpu(), ref["h_last"], 1e-2, "h_last")
    assert_close(out["x"].cpu(), cv["x"], 1e-2, "x")


@pytest.mark.gpu
def test_layouts_chain_into_each_other(orc):
    """The final state of a scan in one layout continues in the other: layouts only
    change how the work is split, not what the state means."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    inp = make_scan_inputs(1, 64, 16, 2048, "f32", seed=950)
    ref = orc.scan(**inp)
    d = dev(inp, SCAN_KEYS)
    half = {k: (v[..., :1024].contiguous() if k in ("x", "dt", "z", "B", "C") and v is not None else v)
            for k, v in d.items()}
    rest = {k: (v[..., 1024:].contiguous() if k in ("x", "dt", "z", "B", "C") and v is not None else v)
            for k, v in d.items()}
    with layout(4):
        y1, h1 = ssscan.ss_scan_fwd(**half)
    rest["h0"] = h1
    with layout(2):
        y2, h2 = ssscan.ss_scan_fwd(**rest)
    torch.cuda.synchronize()
    assert_close(torch.cat([y1, y2], -1).cpu(), ref["y"], 1e-4, "chained y")
    assert_close(h2.cpu(), ref["h_last"], 1e-4, "chained h_last")


@pytest.mark.gpu
@pytest.mark.parametrize("spl", [2, 4])
def test_layout_mamba130m_layer_full(orc, spl):
    """8 x 1536 x 16 x 2048, bf16: every output under each layout."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    inp = make_workload("mamba130m_layer")
    ref = orc.scan(**inp)
    with layout(spl):
        y, h = gpu_scan(inp)
    assert_close(y, ref["y"], 1e-2, "y")
    assert_close(h, ref["h_last"], 1e-2, "h_last")
