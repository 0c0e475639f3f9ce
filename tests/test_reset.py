"""Enforced boundary resets on the GPU path ("s6_reset" blog draft, Enforced
Boundary Resetting; flags on each document's first token, state zeroed before that
token's update).

Bit-exactness is read as: (i) outputs at and after a reset do not depend, bit for
bit, on anything before it (inputs or h0); (ii) the reset token's own output equals,
bit for bit, the same kernel run on that document alone from zeros; (iii) every
later position matches the oracle's document-alone run within the dtype tolerance;
(iv) resets act at exactly the flagged index, including chunk and lane edges."""
import numpy as np
import pytest
import torch

from gpu_util import TOL, assert_close, gpu_scan
from selective_state_space_18_b200.inputs import make_scan_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


def _same_bits(a, b):
    """Equal as values, treating +0 and -0 as equal."""
    return torch.equal(a.float(), b.float())


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("r", [1, 7, 8, 63, 64, 65, 100, 511])
def test_prefix_cannot_leak_past_reset(dtype, r):
    L = 600
    inp = make_scan_inputs(2, 40, 16, L, dtype, seed=500 + r, h0=True)
    mask = torch.zeros(2, L, dtype=torch.uint8)
    mask[:, r] = 1
    mask[1, 0] = 1
    inp["reset"] = mask
    y1, h1 = gpu_scan(inp)
    pert = dict(inp)
    g = torch.Generator().manual_seed(r)
    for k in ("x", "dt", "z", "B", "C"):
        v = inp[k].clone()
        noise = torch.randn(v[:, :, :r].shape, generator=g).to(v.dtype)
        v[:, :, :r] = noise
        pert[k] = v
    pert["h0"] = torch.randn(inp["h0"].shape, generator=g)
    y2, h2 = gpu_scan(pert)
    assert _same_bits(y1[:, :, r:], y2[:, :, r:])
    assert _same_bits(h1, h2)
    assert not torch.equal(y1[:, :, :r], y2[:, :, :r])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_reset_token_equals_document_alone(orc, dtype):
    L = 1500
    inp = make_scan_inputs(2, 36, 16, L, dtype, seed=601, reset_mean_doc=97, h0=True)
    y, h = gpu_scan(inp)
    ref = orc.scan(**inp)
    tol = TOL[inp["x"].dtype]
    assert_close(y, ref["y"], tol, "packed y")
    mask = inp["reset"].numpy()
    for b in range(2):
        starts = list(np.flatnonzero(mask[b])) + [L]
        assert len(starts) > 4
        for s0, s1 in zip(starts[:-1], starts[1:]):
            alone = {k: None for k in inp}
            for k in ("x", "dt", "z", "B", "C"):
                alone[k] = inp[k][b:b + 1, :, s0:s1].contiguous()
            for k in ("A", "D", "dt_bias"):
                alone[k] = inp[k]
            ya, _ = gpu_scan(alone)
            assert _same_bits(ya[0, :, 0], y[b, :, s0]), (b, s0)
            oref = orc.scan(**alone)
            assert_close(y[b, :, s0:s1], oref["y"][0], tol, f"document {(b, s0, s1)}")


@pytest.mark.parametrize("positions", [[0], [0, 1], [31, 32, 33], [63, 64], [127, 128, 129],
                                       [7, 8, 15, 16], [255], [999]])
def test_reset_positions_exact(orc, positions):
    L = 1000
    inp = make_scan_inputs(1, 24, 16, L, "f32", seed=700 + positions[0], h0=True)
    mask = torch.zeros(1, L, dtype=torch.uint8)
    mask[0, positions] = 1
    inp["reset"] = mask
    y, h = gpu_scan(inp)
    ref = orc.scan(**inp)
    assert_close(y, ref["y"], 1e-4, "y")
    assert_close(h, ref["h_last"], 1e-4, "h_last")
    # one token later than flagged gives a different answer: the index is exact
    shifted = dict(inp)
    m2 = torch.zeros(1, L, dtype=torch.uint8)
    m2[0, [min(p + 1, L - 1) for p in positions]] = 1
    shifted["reset"] = m2
    if not torch.equal(m2, mask):
        y2, _ = gpu_scan(shifted)
        p = positions[0]
        assert not torch.equal(y[0, :, p], y2[0, :, p])


def test_every_token_reset():
    """Resets on every token: h_t = dt_t B_t x_t, nothing carries over."""
    inp = make_scan_inputs(1, 16, 16, 256, "f32", seed=801, h0=True)
    inp["reset"] = torch.ones(1, 256, dtype=torch.uint8)
    y, h = gpu_scan(inp)
    one = make_scan_inputs(1, 16, 16, 256, "f32", seed=801, h0=True)
    for t in (0, 1, 100, 255):
        alone = {k: None for k in one}
        for k in ("x", "dt", "z", "B", "C"):
            alone[k] = one[k][:, :, t:t + 1].contiguous()
        for k in ("A", "D", "dt_bias"):
            alone[k] = one[k]
        ya, _ = gpu_scan(alone)
        assert _same_bits(ya[0, :, 0], y[0, :, t])
