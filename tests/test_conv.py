"""The scan with the causal depthwise conv + SiLU fused in front (ss_scan_fwd_conv)
against the oracle composition: conv + SiLU (TransformerLens ssm_mixer: the scan's x is
SiLU of the conv1d output), then the selective scan."""
import numpy as np
import pytest
import torch

from gpu_util import TOL, assert_close
from selective_state_space_18_b200 import ssscan
from selective_state_space_18_b200.inputs import make_scan_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


def _inputs(bt, ch, n, L, dtype, K, seed, state=True, bias=True, resets=False):
    inp = make_scan_inputs(bt, ch, n, L, dtype, seed=seed, reset_mean_doc=25 if resets else 0, h0=True)
    g = torch.Generator().manual_seed(seed + 1)
    inp["u"] = inp.pop("x")
    inp["conv_w"] = torch.randn(ch, K, generator=g) * 0.5
    inp["conv_b"] = torch.randn(ch, generator=g) * 0.1 if bias else None
    inp["conv_state"] = torch.randn(bt, ch, K - 1, generator=g) if state and K > 1 else None
    return inp


def _gpu(inp, **kw):
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    out = ssscan.ss_scan_fwd_conv(d["u"], d["conv_w"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["z"], d["dt_bias"],
                                  d["reset"], d["h0"], conv_b=d["conv_b"], conv_state=d["conv_state"], return_x=True,
                                  **kw)
    torch.cuda.synchronize()
    return {k: (None if v is None else v.cpu()) for k, v in out.items()}


def _oracle(orc, inp):
    cv = orc.conv_silu(inp["u"], inp["conv_w"], inp["conv_b"], inp["conv_state"])
    sc = orc.scan(x=cv["x"], dt=inp["dt"], A=inp["A"], B=inp["B"], C=inp["C"], D=inp["D"], z=inp["z"],
                  dt_bias=inp["dt_bias"], reset=inp["reset"], h0=inp["h0"])
    return cv, sc


@pytest.mark.parametrize("case", [
    (2, 40, 16, 264, "bf16", 4, True, True, False),   # tile-load path
    (2, 40, 16, 77, "bf16", 4, True, True, True),     # ragged path, resets
    (1, 24, 8, 100, "f32", 3, False, True, False),
    (3, 20, 4, 50, "f32", 2, True, False, True),
    (2, 16, 16, 40, "f32", 1, False, False, False),
    (1, 8, 16, 2, "f32", 4, True, True, False),       # shorter than the conv window
    (1, 320, 16, 2048, "bf16", 4, True, True, False), # many channel groups, segmented schedule
], ids=lambda c: "x".join(str(v) for v in c))
def test_matches_oracle_composition(orc, case):
    bt, ch, n, L, dtype, K, state, bias, resets = case
    inp = _inputs(bt, ch, n, L, dtype, K, seed=600 + L + K, state=state, bias=bias, resets=resets)
    out = _gpu(inp)
    cv, sc = _oracle(orc, inp)
    tol = TOL[inp["u"].dtype]
    assert_close(out["y"], sc["y"], tol, "y")
    assert_close(out["h_last"], sc["h_last"], tol, "h_last")
    assert_close(out["x"], cv["x"], tol, "x")
    if K > 1:  # a copy of inputs: exact
        np.testing.assert_array_equal(out["conv_state"].double().numpy(), cv["state"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_two_calls_chained_through_both_states(dtype):
    """A prompt split in two calls (conv state and scan state handed over) equals one call."""
    inp = _inputs(2, 48, 16, 640, dtype, 4, seed=650, state=False)
    full = _gpu(inp)
    a, b = dict(inp), dict(inp)
    for k in ("u", "dt", "z", "B", "C"):
        a[k] = inp[k][:, :, :296].contiguous()
        b[k] = inp[k][:, :, 296:].contiguous()
    oa = _gpu(a)
    b["conv_state"], b["h0"] = oa["conv_state"], oa["h_last"]
    ob = _gpu(b)
    assert_close(torch.cat([oa["y"], ob["y"]], -1), full["y"].double().numpy(), 1e-6, "y")
    assert_close(ob["h_last"], full["h_last"].double().numpy(), 1e-6, "h_last")
    assert torch.equal(ob["conv_state"], full["conv_state"])


def _upd_inputs(bt, ch, n, dtype, K, seed):
    from selective_state_space_18_b200.inputs import make_update_inputs
    inp = make_update_inputs(bt, ch, n, dtype, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    inp["u"] = inp.pop("x")
    inp["conv_w"] = torch.randn(ch, K, generator=g) * 0.5
    inp["conv_b"] = torch.randn(ch, generator=g) * 0.1
    inp["conv_state"] = torch.randn(bt, ch, K - 1, generator=g)
    return inp


@pytest.mark.parametrize("case", [(256, 5120, 16, "bf16", 4), (3, 37, 8, "f32", 3), (5, 64, 4, "f32", 2),
                                  (4, 100, 16, "bf16", 1), (3, 1000, 16, "bf16", 4), (2, 1000, 16, "f32", 3)],
                         ids=lambda c: "x".join(str(v) for v in c))
def test_decode_conv_matches_oracle(orc, case):
    bt, ch, n, dtype, K = case
    inp = _upd_inputs(bt, ch, n, dtype, K, seed=700 + K)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    y = ssscan.ss_state_update_conv(d["state"], d["conv_state"] if K > 1 else None, d["conv_w"], d["u"], d["dt"],
                                    d["A"], d["B"], d["C"], d["D"], d["z"], d["dt_bias"], conv_b=d["conv_b"])
    torch.cuda.synchronize()
    cv = orc.conv_silu(inp["u"][:, :, None], inp["conv_w"], inp["conv_b"], inp["conv_state"] if K > 1 else None)
    ref = orc.update(state=inp["state"], x=cv["x"][:, :, 0], dt=inp["dt"], A=inp["A"], B=inp["B"], C=inp["C"],
                     D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"])
    assert_close(y.cpu(), ref["y"], TOL[inp["u"].dtype], "y")
    assert_close(d["state"].cpu(), ref["state"], 1e-4, "state")
    if K > 1:  # the shifted inputs: exact
        np.testing.assert_array_equal(d["conv_state"].cpu().double().numpy(), cv["state"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_conv_continues_the_fused_prompt(dtype):
    """Prompt over L-1 tokens, then one decode step from its two states, equals the
    prompt over L tokens at the last token."""
    inp = _inputs(2, 64, 16, 97, dtype, 4, seed=710, state=True)
    full = _gpu(inp)
    head = dict(inp)
    for k in ("u", "dt", "z", "B", "C"):
        head[k] = inp[k][:, :, :-1].contiguous()
    oh = _gpu(head)
    st, cs = oh["h_last"].cuda(), oh["conv_state"].cuda()
    last = {k: inp[k][:, :, -1].contiguous().cuda() for k in ("u", "dt", "z", "B", "C")}
    y = ssscan.ss_state_update_conv(st, cs, inp["conv_w"].cuda(), last["u"], last["dt"], inp["A"].cuda(), last["B"],
                                    last["C"], inp["D"].cuda(), last["z"], inp["dt_bias"].cuda(),
                                    conv_b=inp["conv_b"].cuda())
    torch.cuda.synchronize()
    tol = 1e-5 if dtype == "f32" else TOL[torch.bfloat16]
    assert_close(y.cpu(), full["y"][:, :, -1].double().numpy(), tol, "y")
    assert_close(st.cpu(), full["h_last"].double().numpy(), max(tol, 1e-5), "state")
    assert torch.equal(cs.cpu(), full["conv_state"])


def test_layer_workload_full_size_sampled(orc):
    """The fused conv form at the 2.8B layer shape it is timed on (1 x 5120 x 16 x 16384,
    bf16, conv_k 4 with a bias, no conv state, in the benchmark's launch configuration):
    every output and final-state entry of sampled channels -- the first and last channel
    group and both sides of a group boundary -- against the oracle composition run on
    those channels."""
    from selective_state_space_18_b200.inputs import make_workload
    inp = make_workload("mamba2p8b_layer_long")
    ch = inp["x"].shape[1]
    g = torch.Generator().manual_seed(4242)
    cw = torch.randn(ch, 4, generator=g) * 0.5
    cb = torch.randn(ch, generator=g) * 0.1
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    out = ssscan.ss_scan_fwd_conv(d["x"], cw.cuda(), d["dt"], d["A"], d["B"], d["C"], d["D"], d["z"], d["dt_bias"],
                                  conv_b=cb.cuda(), return_conv_state=False)
    torch.cuda.synchronize()
    chans = [0, 1, 15, 16, 2559, 2560, 5118, 5119]
    y, h = out["y"][:, chans].cpu(), out["h_last"][:, chans].cpu()
    sub = {"u": inp["x"][:, chans], "conv_w": cw[chans], "conv_b": cb[chans], "conv_state": None,
           "dt": inp["dt"][:, chans], "A": inp["A"][chans], "B": inp["B"], "C": inp["C"],
           "D": None if inp["D"] is None else inp["D"][chans], "z": None if inp["z"] is None else inp["z"][:, chans],
           "dt_bias": None if inp["dt_bias"] is None else inp["dt_bias"][chans], "reset": inp.get("reset"),
           "h0": None if inp.get("h0") is None else inp["h0"][:, chans]}
    cv, sc = _oracle(orc, sub)
    assert_close(y, sc["y"], TOL[torch.bfloat16], "y")
    assert_close(h, sc["h_last"], 1e-2, "h_last")
