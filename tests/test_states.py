"""The state after every token (ss_scan_fwd_states) against the oracle's per-token
states (nnterp selective_scan: the state after each token, for the interpretability
readers; TransformerLens ssm_mixer: the unrolled state S_t at every position)."""
import numpy as np
import pytest
import torch

from gpu_util import SCAN_KEYS, TOL, assert_close, dev
from selective_state_space_18_b200 import ssscan
from selective_state_space_18_b200.inputs import make_scan_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


def _gpu(inp, **kw):
    y, h, hall = ssscan.ss_scan_fwd(**dev(inp, SCAN_KEYS), return_states=True, **kw)
    torch.cuda.synchronize()
    return y.cpu(), h.cpu(), hall.cpu()


@pytest.mark.parametrize("n", [4, 8, 16])
@pytest.mark.parametrize("dtype,L", [("f32", 100), ("bf16", 264), ("bf16", 77)])
@pytest.mark.parametrize("resets", [False, True])
def test_states_match_oracle(orc, n, dtype, L, resets):
    inp = make_scan_inputs(2, 40, n, L, dtype, seed=400 + n + L, h0=True, reset_mean_doc=30 if resets else 0)
    y, h, hall = _gpu(inp)
    ref = orc.scan(**inp, return_states=True)
    tol = TOL[inp["x"].dtype]
    assert_close(y, ref["y"], tol, "y")
    # states are fp32 whatever the storage type: the fp32 state tolerance
    assert_close(hall, ref["h_all"], 1e-4, "h_all")
    assert torch.equal(hall[:, :, -1, :], h)  # the last state is h_last, bit for bit


def test_states_leave_y_and_h_last_unchanged():
    """Emitting the states changes nothing else, bit for bit, in either schedule."""
    inp = make_scan_inputs(3, 96, 16, 1500, "bf16", seed=420, h0=True, reset_mean_doc=200)
    d = dev(inp, SCAN_KEYS)
    for ws in (True, False):
        y0, h0 = ssscan.ss_scan_fwd(**d, workspace=ws)
        y1, h1, hall = ssscan.ss_scan_fwd(**d, workspace=ws, return_states=True)
        torch.cuda.synchronize()
        assert torch.equal(y0, y1) and torch.equal(h0, h1)
        assert torch.equal(hall[:, :, -1, :], h1)


def test_states_segmented_equals_static():
    inp = make_scan_inputs(1, 320, 16, 4096, "bf16", seed=421)
    d = dev(inp, SCAN_KEYS)
    _, _, a = ssscan.ss_scan_fwd(**d, workspace=True, return_states=True)
    _, _, b = ssscan.ss_scan_fwd(**d, workspace=False, return_states=True)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_states_sampled_rows_medium(orc):
    """A shape with many channel groups and a ragged tail: sampled rows, every token."""
    inp = make_scan_inputs(2, 512, 16, 3001, "bf16", seed=422, reset_mean_doc=300)
    y, h, hall = _gpu(inp)
    rows = [(0, 0), (0, 17), (1, 255), (1, 511), (0, 300)]
    sub = {k: v for k, v in inp.items()}
    for b, c in rows:
        one = dict(sub)
        for k in ("x", "dt", "z"):
            one[k] = inp[k][b:b + 1, c:c + 1]
        for k in ("B", "C", "reset"):
            one[k] = inp[k][b:b + 1] if inp[k] is not None else None
        one["A"] = inp["A"][c:c + 1]
        for k in ("D", "dt_bias"):
            one[k] = inp[k][c:c + 1] if inp[k] is not None else None
        one["h0"] = None
        ref = orc.scan(**one, return_states=True)
        assert_close(hall[b, c], ref["h_all"][0, 0], 1e-4, f"h_all row {(b, c)}")
        assert_close(y[b, c], ref["y"][0, 0], TOL[torch.bfloat16], f"y row {(b, c)}")


def test_states_layer_workload_full_size_sampled(orc):
    """The 2.8B layer shape the states form is timed on (1 x 5120 x 16 x 16384, bf16,
    h_all given as the benchmark gives it, 5.4 GB of states): every token's state and
    output of sampled channels -- the first and last channel group and both sides of a
    group boundary -- against the oracle run on those rows."""
    from selective_state_space_18_b200.inputs import make_workload
    inp = make_workload("mamba2p8b_layer_long")
    d = dev(inp, SCAN_KEYS)
    bt, ch, L = d["x"].shape
    n = d["A"].shape[1]
    y = torch.empty(bt, ch, L, device="cuda", dtype=torch.bfloat16)
    hl = torch.empty(bt, ch, n, device="cuda")
    hall = torch.empty(bt, ch, L, n, device="cuda")
    ssscan.ss_scan_fwd(**d, y=y, h_last=hl, h_all=hall)
    torch.cuda.synchronize()
    chans = [0, 1, 15, 16, 2559, 2560, 5118, 5119]
    hs, ys, hls = hall[0, chans].cpu(), y[0, chans].cpu(), hl[0, chans].cpu()
    del hall
    for i, c in enumerate(chans):
        one = dict(inp)
        for k in ("x", "dt", "z"):
            one[k] = inp[k][:, c:c + 1]
        one["A"] = inp["A"][c:c + 1]
        for k in ("D", "dt_bias"):
            one[k] = inp[k][c:c + 1] if inp[k] is not None else None
        one["h0"] = inp["h0"][:, c:c + 1] if inp.get("h0") is not None else None
        ref = orc.scan(**one, return_states=True)
        assert_close(hs[i], ref["h_all"][0, 0], 1e-4, f"h_all channel {c}")
        assert_close(hls[i], ref["h_last"][0, 0], 1e-4, f"h_last channel {c}")
        assert_close(ys[i], ref["y"][0, 0], TOL[torch.bfloat16], f"y channel {c}")


# ---- the step size of every token ("betas" of the nnterp selective_scan page) ------------

@pytest.mark.parametrize("n", [4, 8, 16])
@pytest.mark.parametrize("dtype,L", [("f32", 100), ("bf16", 264), ("bf16", 77), ("f32", 31)])
@pytest.mark.parametrize("softplus", [True, False])
def test_betas_match_oracle(orc, n, dtype, L, softplus):
    """Every token's step size against the oracle's, with the states, across tile-load
    and ragged lengths; and the log decays betas * A against the oracle's dt * A."""
    inp = make_scan_inputs(2, 40, n, L, dtype, seed=430 + n + L, h0=True, reset_mean_doc=30)
    if not softplus:  # positive steps without the softplus (the bias is negative): the raw steps alone
        inp["dt"] = (inp["dt"].float().abs() * 0.1).to(inp["dt"].dtype)
        inp["dt_bias"] = None
    d = dev(inp, SCAN_KEYS)
    y, h, hall, betas = ssscan.ss_scan_fwd(**d, dt_softplus=softplus, return_states=True, return_betas=True)
    torch.cuda.synchronize()
    ref = orc.scan(**inp, dt_softplus=softplus, return_states=True, return_betas=True)
    assert_close(betas.cpu(), ref["betas"], 1e-4, "betas")
    assert_close(hall.cpu(), ref["h_all"], 1e-4, "h_all")
    assert_close(y.cpu(), ref["y"], TOL[inp["x"].dtype], "y")
    A = inp["A"].double().numpy()
    assert_close(betas.cpu()[..., None] * inp["A"][None, :, None, :], ref["betas"][..., None] * A[None, :, None, :],
                 1e-4, "log decays")


def test_betas_alone_change_nothing_else():
    """The step sizes asked for without the states: y and h_last bit-identical to the
    plain scan's, the step sizes bit-identical to those emitted beside the states, in
    either schedule."""
    inp = make_scan_inputs(3, 96, 16, 1500, "bf16", seed=440, h0=True, reset_mean_doc=200)
    d = dev(inp, SCAN_KEYS)
    for ws in (True, False):
        y0, h0 = ssscan.ss_scan_fwd(**d, workspace=ws)
        y1, h1, none, b1 = ssscan.ss_scan_fwd(**d, workspace=ws, return_betas=True)
        _, _, _, b2 = ssscan.ss_scan_fwd(**d, workspace=ws, return_states=True, return_betas=True)
        torch.cuda.synchronize()
        assert none is None
        assert torch.equal(y0, y1) and torch.equal(h0, h1)
        assert torch.equal(b1, b2)


def test_betas_sampled_rows_medium(orc):
    """Many channel groups and a ragged tail: every token's step size of sampled rows."""
    inp = make_scan_inputs(2, 512, 16, 3001, "bf16", seed=441)
    _, _, _, betas = ssscan.ss_scan_fwd(**dev(inp, SCAN_KEYS), return_betas=True)
    torch.cuda.synchronize()
    rows = [(0, 0), (0, 17), (1, 255), (1, 511), (0, 300)]
    for b, c in rows:
        one = dict(inp)
        for k in ("x", "dt", "z"):
            one[k] = inp[k][b:b + 1, c:c + 1]
        one["B"], one["C"] = inp["B"][b:b + 1], inp["C"][b:b + 1]
        one["A"] = inp["A"][c:c + 1]
        for k in ("D", "dt_bias"):
            one[k] = inp[k][c:c + 1] if inp[k] is not None else None
        one["h0"], one["reset"] = None, None
        ref = orc.scan(**one, return_betas=True)
        assert_close(betas[b, c].cpu(), ref["betas"][0, 0], 1e-4, f"betas row {(b, c)}")
