"""The gated state scan on the GPU (ss_gated_scan) against the oracle ("Mamba 2 Gated
State Scan" exercise page: S_t = gamma_t S_{t-1} + k_t v_t^T, y_t = q_t^T S_t)."""
import json
import os

import numpy as np
import pytest
import torch

from gpu_util import TOL, assert_close
from selective_state_space_18_b200 import ssscan
from selective_state_space_18_b200.inputs import make_gated_inputs

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


def _gpu(inp):
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    out = ssscan.ss_gated_scan(**d)
    torch.cuda.synchronize()
    return out["outputs"].cpu(), out["final_state"].cpu()


def test_page_examples_on_gpu():
    with open(os.path.join(GOLDEN, "gated_state_scan_page_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        inp = {"q": torch.tensor(c["q"], dtype=torch.float32), "k": torch.tensor(c["k"], dtype=torch.float32),
               "v": torch.tensor(c["v"], dtype=torch.float32), "gamma": torch.tensor(c["gamma"], dtype=torch.float32)}
        y, fs = _gpu(inp)
        assert torch.equal(y, torch.tensor(c["outputs"], dtype=torch.float32)), c["name"]
        assert torch.equal(fs, torch.tensor(c["final_state"], dtype=torch.float32)), c["name"]


@pytest.mark.parametrize("shape", [(3, 37, 16, 24), (2, 100, 64, 64), (2, 65, 128, 70), (1, 9, 1, 1),
                                   (4, 33, 33, 130), (2, 8, 128, 257)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_matches_oracle(orc, shape, dtype):
    B, S, dk, dv = shape
    inp = make_gated_inputs(B, S, dk, dv, dtype, seed=500 + B * S + dk + dv, h0=(dtype == "f32"))
    y, fs = _gpu(inp)
    ref = orc.gated_scan(**inp)
    tol = TOL[inp["q"].dtype]
    assert_close(y, ref["outputs"], tol, "outputs")
    assert_close(fs, ref["final_state"], tol, "final_state")
    assert y.dtype == inp["q"].dtype and fs.dtype == inp["q"].dtype


def test_chaining_through_final_state():
    inp = make_gated_inputs(3, 90, 64, 48, "f32", seed=510)
    y, fs = _gpu(inp)
    a = {k: v[:, :41].contiguous() for k, v in inp.items() if v is not None}
    b = {k: v[:, 41:].contiguous() for k, v in inp.items() if v is not None}
    ya, fa = _gpu(a)
    b["h0"] = fa
    yb, fb = _gpu(b)
    assert_close(torch.cat([ya, yb], 1), y.double().numpy(), 1e-5, "outputs")
    assert_close(fb, fs.double().numpy(), 1e-5, "final_state")


def test_noncontiguous_inputs_unchanged(orc):
    """Inputs may be non-contiguous views; they are never modified."""
    base = make_gated_inputs(2, 40, 32, 16, "bf16", seed=511)
    q = base["q"].transpose(1, 2).contiguous().transpose(1, 2)   # same values, strided view
    assert not q.is_contiguous()
    dq = q.cuda()
    keep = dq.clone()
    d = {"q": dq, "k": base["k"].cuda(), "v": base["v"].cuda(), "gamma": base["gamma"].cuda()}
    out = ssscan.ss_gated_scan(**d)
    torch.cuda.synchronize()
    assert torch.equal(dq, keep)
    ref = orc.gated_scan(base["q"], base["k"], base["v"], base["gamma"])
    assert_close(out["outputs"].cpu(), ref["outputs"], TOL[torch.bfloat16], "outputs")


def test_large_batch_sampled(orc):
    """Many batch items and column tiles: every output of a sample of items."""
    inp = make_gated_inputs(96, 300, 128, 64, "bf16", seed=512)
    y, fs = _gpu(inp)
    for b in (0, 1, 47, 95):
        sub = {k: (v[b:b + 1] if v is not None else None) for k, v in inp.items()}
        ref = orc.gated_scan(**sub)
        assert_close(y[b:b + 1], ref["outputs"], TOL[torch.bfloat16], f"outputs item {b}")
        assert_close(fs[b:b + 1], ref["final_state"], TOL[torch.bfloat16], f"final_state item {b}")
