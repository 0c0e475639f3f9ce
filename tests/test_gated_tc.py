"""The chunked tensor-core form of the gated state scan ("Mamba 2 Gated State Scan"
exercise page: S_t = gamma_t S_{t-1} + k_t v_t^T, y_t = q_t^T S_t), which ss_gated_scan
runs for bf16 inputs with dk = 128 and dv a multiple of 64: every output and the final
state against the float64 oracle, and against the token-by-token kernel on the same
inputs, both within the bf16 tolerance -- across ragged chunk tails, several value
tiles, an initial state, and gates of exactly 0 and 1 (on chunk boundaries too)."""
import contextlib

import pytest
import torch

from gpu_util import TOL, assert_close
from selective_state_space_18_b200 import ssscan
from selective_state_space_18_b200.inputs import make_gated_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


@contextlib.contextmanager
def recurrent():
    ssscan.ss_debug_set_gated_path(1)
    try:
        yield
    finally:
        ssscan.ss_debug_set_gated_path(0)


def _gpu(inp):
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    out = ssscan.ss_gated_scan(**d)
    torch.cuda.synchronize()
    return out["outputs"].cpu(), out["final_state"].cpu()


def _check(orc, inp, what):
    y, fs = _gpu(inp)
    with recurrent():
        y1, fs1 = _gpu(inp)
    ref = orc.gated_scan(**inp)
    tol = TOL[torch.bfloat16]
    assert_close(y, ref["outputs"], tol, f"{what}: outputs")
    assert_close(fs, ref["final_state"], tol, f"{what}: final_state")
    assert_close(y, y1.double().numpy(), tol, f"{what}: outputs against the recurrent kernel")
    assert_close(fs, fs1.double().numpy(), tol, f"{what}: final_state against the recurrent kernel")


@pytest.mark.parametrize("shape", [(2, 128, 64), (3, 300, 64), (2, 1000, 128), (1, 2048, 192), (5, 1, 64),
                                   (2, 127, 64), (1, 4100, 64)])
@pytest.mark.parametrize("h0", [False, True])
def test_chunked_form_matches_oracle(orc, shape, h0):
    B, S, dv = shape
    inp = make_gated_inputs(B, S, 128, dv, "bf16", seed=1900 + B * S + dv, h0=h0)
    _check(orc, inp, f"{shape}")


@pytest.mark.parametrize("pattern", ["zeros_on_boundaries", "all_ones", "all_zeros", "zero_first", "negative",
                                     "above_one", "tiny"])
def test_exact_gates(orc, pattern):
    """Gates the decay mask must take exactly as the recurrence does: zeros (the state
    is discarded), ones, negative gates (signs of the products), magnitudes above 1 (the
    element-by-element form of the mask) and gates below the smallest normal float."""
    B, S, dv = 2, 520, 64
    inp = make_gated_inputs(B, S, 128, dv, "bf16", seed=1950, h0=True)
    g = inp["gamma"].clone()
    gen = torch.Generator().manual_seed(1951)
    if pattern == "zeros_on_boundaries":
        g[:, ::128] = 0.0          # the state is discarded exactly where a chunk starts
        g[1, 255] = 0.0            # and on a chunk's last token
    elif pattern == "all_ones":
        g[:] = 1.0                 # no decay: the state is a running sum
    elif pattern == "all_zeros":
        g[:] = 0.0                 # every token stands alone: S_t = k_t v_t^T
    elif pattern == "zero_first":
        g[:, 0] = 0.0              # the initial state is discarded at once
    elif pattern == "negative":
        flip = torch.rand(g.shape, generator=gen) < 0.3
        g = torch.where(flip, -g, g)  # about a third of the gates negative
        g[0, 130] = -1.0
    elif pattern == "above_one":
        g = 0.9 + 0.2 * torch.rand(g.shape, generator=gen)  # |gamma| in [0.9, 1.1]
        g[1, 300:310] = 1.5
    else:
        g[:, 5::37] = 1e-39        # subnormal gates: the terms they scale vanish
    inp["gamma"] = g.float().contiguous()
    _check(orc, inp, pattern)


def test_chunked_form_chains_through_its_final_state(orc):
    """Two calls chained through the final state (given back as h0, fp32) equal one
    call over the whole sequence within the bf16 tolerance (the final state between
    the calls is rounded to bf16, as the page's output dtype asks)."""
    inp = make_gated_inputs(2, 700, 128, 64, "bf16", seed=1960)
    y, fs = _gpu(inp)
    a = {k: v[:, :384].contiguous() for k, v in inp.items() if v is not None}
    b = {k: v[:, 384:].contiguous() for k, v in inp.items() if v is not None}
    ya, fa = _gpu(a)
    b["h0"] = fa.float()
    yb, fb = _gpu(b)
    tol = TOL[torch.bfloat16]
    assert_close(torch.cat([ya, yb], 1), y.double().numpy(), tol, "outputs")
    assert_close(fb, fs.double().numpy(), tol, "final_state")


def test_timed_out_waits_report_and_recover(orc):
    """Failure detection in the tensor-core form without a GPU fault: with the compute
    warps' first "L o S written" arrival withheld (a flag nothing sets) and the wait
    limit cut to 2 ms, the issuer's wait for it gives up, the status word reports
    SS_ERR_TIMEOUT, and the kernel still drains its loads and products before freeing
    its tensor memory -- the next call, normal again, gives the normal answer."""
    inp = make_gated_inputs(2, 2048, 128, 64, "bf16", seed=1970, h0=True)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    assert ssscan.ss_debug_status() == "SS_OK"
    ssscan.ss_debug_set_wait_limit(2000)
    ssscan.ss_debug_set_gated_path(3)
    try:
        ssscan.ss_gated_scan(**d)
        torch.cuda.synchronize()
        assert ssscan.ss_debug_status() == "SS_ERR_TIMEOUT"
    finally:
        ssscan.ss_debug_set_gated_path(0)
        ssscan.ss_debug_set_wait_limit(0)
    out = ssscan.ss_gated_scan(**d)
    torch.cuda.synchronize()
    assert ssscan.ss_debug_status() == "SS_OK"
    ref = orc.gated_scan(**inp)
    tol = TOL[torch.bfloat16]
    assert_close(out["outputs"].cpu(), ref["outputs"], tol, "outputs after the timeout")
    assert_close(out["final_state"].cpu(), ref["final_state"], tol, "final_state after the timeout")


def test_bench_workload_full_size_sampled(orc):
    """The workload the gated benchmark times, at full size and in its launch
    configuration (512 items x 2048 tokens, dk 128, dv 64, bf16, the same seed): every
    output and final-state entry of sampled items -- the first, second, middle and last
    item, so the first and last CTAs of the grid -- against the oracle run on those items."""
    inp = make_gated_inputs(512, 2048, 128, 64, "bf16", seed=77)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    out = ssscan.ss_gated_scan(d["q"], d["k"], d["v"], d["gamma"])
    torch.cuda.synchronize()
    assert ssscan.ss_debug_status() == "SS_OK"
    items = [0, 1, 255, 256, 510, 511]
    y = out["outputs"][items].cpu()
    fs = out["final_state"][items].cpu()
    tol = TOL[torch.bfloat16]
    for i, b in enumerate(items):
        sub = {k: (v[b:b + 1] if v is not None else None) for k, v in inp.items()}
        ref = orc.gated_scan(**sub)
        assert_close(y[i:i + 1], ref["outputs"], tol, f"outputs item {b}")
        assert_close(fs[i:i + 1], ref["final_state"], tol, f"final_state item {b}")
