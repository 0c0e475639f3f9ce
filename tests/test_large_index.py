"""Shapes whose element counts pass 2^31, so that any 32-bit index arithmetic in the kernels
would wrap: the prompt scan over more than 2^31 (b, c, t) positions in both of its
schedules, and the per-token states form writing more than 2^31 state elements.  The large
tensors are drawn on the device from a seeded generator (as the shared input module draws
them on the host: standard normal x, dt_raw and z in bf16, B and C in bf16, the per-channel
parameters from the input module); the sampled rows are copied to the host and run through
the float64 oracle, every token of each."""
import pytest
import torch

from gpu_util import TOL, assert_close, schedule
from selective_state_space_18_b200 import ssscan
from selective_state_space_18_b200.inputs import make_scan_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    free, _ = torch.cuda.mem_get_info()
    if free < 40 * 2**30:
        pytest.skip("needs 40 GB of free device memory")


def _big_inputs(channels, seq, seed):
    """x, dt_raw, z [1, channels, seq] bf16 drawn on the device; B, C [1, 16, seq] bf16 and
    A, D, dt_bias [channels] from host generators."""
    small = make_scan_inputs(1, channels, 16, 1, "bf16", seed=seed, a_perturb=True)
    gd = torch.Generator(device="cuda").manual_seed(seed + 1)
    gh = torch.Generator().manual_seed(seed + 2)
    d = {k: torch.randn(1, channels, seq, generator=gd, device="cuda", dtype=torch.bfloat16) for k in ("x", "dt", "z")}
    for k in ("B", "C"):
        d[k] = torch.randn(1, 16, seq, generator=gh).to(torch.bfloat16).cuda()
    for k in ("A", "D", "dt_bias"):
        d[k] = small[k].cuda()
    return d


def _oracle_row(orc, d, c, **kw):
    one = {"x": d["x"][:, c:c + 1].cpu(), "dt": d["dt"][:, c:c + 1].cpu(), "z": d["z"][:, c:c + 1].cpu(),
           "B": d["B"].cpu(), "C": d["C"].cpu(), "A": d["A"][c:c + 1].cpu(), "D": d["D"][c:c + 1].cpu(),
           "dt_bias": d["dt_bias"][c:c + 1].cpu()}
    return orc.scan(**one, **kw)


def test_scan_beyond_int32_positions(orc):
    """1 x 4096 x 16 x 524544: 2.15e9 (b, c, t) positions (x alone 4.3 GB), the chained
    single-pass schedule and the two-level one; every output and final-state entry of
    channels at both ends and around the middle, against the oracle."""
    channels, seq = 4096, 524288 + 256
    assert channels * seq > 2**31
    d = _big_inputs(channels, seq, seed=2300)
    keys = ("x", "dt", "A", "B", "C", "D", "z", "dt_bias")
    chans = [0, 1, 2047, 2048, 4094, 4095]
    refs = {c: _oracle_row(orc, d, c) for c in chans}
    for two_level in (1, 2):
        with schedule(two_level=two_level):
            assert ssscan.ss_scan_plan(1, channels, 16, seq)["two_level"] == (two_level == 2)
            y, h = ssscan.ss_scan_fwd(*[d[k] for k in keys])
            ws = ssscan.scan_workspace(1, channels, 16, seq, y.device)
        assert ssscan.ss_scan_status(ws) == "SS_OK"
        ys, hs = y[0, chans].cpu(), h[0, chans].cpu()
        del y, h
        for i, c in enumerate(chans):
            assert_close(ys[i], refs[c]["y"][0, 0], TOL[torch.bfloat16], f"y channel {c}, schedule {two_level}")
            assert_close(hs[i], refs[c]["h_last"][0, 0], 1e-2, f"h_last channel {c}, schedule {two_level}")


def test_states_beyond_int32_elements(orc):
    """1 x 1024 x 16 x 131136: the states output holds 2.15e9 fp32 elements (8.6 GB);
    every token's state and output of sampled channels against the oracle."""
    channels, seq = 1024, 131072 + 64
    assert channels * seq * 16 > 2**31
    d = _big_inputs(channels, seq, seed=2400)
    keys = ("x", "dt", "A", "B", "C", "D", "z", "dt_bias")
    y, h, hall = ssscan.ss_scan_fwd(*[d[k] for k in keys], return_states=True)
    assert ssscan.ss_scan_status(ssscan.scan_workspace(1, channels, 16, seq, y.device)) == "SS_OK"
    chans = [0, 511, 1022, 1023]
    hs, ys, hls = hall[0, chans].cpu(), y[0, chans].cpu(), h[0, chans].cpu()
    del hall, y, h
    for i, c in enumerate(chans):
        ref = _oracle_row(orc, d, c, return_states=True)
        assert_close(hs[i], ref["h_all"][0, 0], 1e-4, f"h_all channel {c}")
        assert_close(hls[i], ref["h_last"][0, 0], 1e-4, f"h_last channel {c}")
        assert_close(ys[i], ref["y"][0, 0], TOL[torch.bfloat16], f"y channel {c}")


@pytest.mark.parametrize("batch,channels", [(32769, 4096), (32768, 4100)])
def test_decode_beyond_int32_state_elements(orc, batch, channels):
    """A decode step whose state holds more than 2^31 fp32 elements (8.6 GB, updated in
    place), with x/dt/z rows of 16-byte multiples (vector loads) and not (4100 channels):
    every output and new state entry of sampled batch rows (the first, the last and two
    around the middle) against the oracle's update of those rows."""
    assert batch * channels * 16 > 2**31
    small = make_scan_inputs(1, channels, 16, 1, "bf16", seed=2500, a_perturb=True)
    gd = torch.Generator(device="cuda").manual_seed(2501)
    d = {"state": torch.randn(batch, channels, 16, generator=gd, device="cuda")}
    for k in ("x", "dt", "z"):
        d[k] = torch.randn(batch, channels, generator=gd, device="cuda", dtype=torch.bfloat16)
    for k in ("B", "C"):
        d[k] = torch.randn(batch, 16, generator=gd, device="cuda", dtype=torch.bfloat16)
    for k in ("A", "D", "dt_bias"):
        d[k] = small[k].cuda()
    rows = [0, batch // 2 - 1, batch // 2, batch - 1]
    before = {k: d[k][rows].cpu() for k in ("state", "x", "dt", "z", "B", "C")}
    y = ssscan.ss_state_update(**d)
    assert ssscan.ss_debug_status() == "SS_OK"
    ys, st = y[rows].cpu(), d["state"][rows].cpu()
    ref = orc.update(state=before["state"], x=before["x"], dt=before["dt"], A=small["A"], B=before["B"],
                     C=before["C"], D=small["D"], z=before["z"], dt_bias=small["dt_bias"])
    assert_close(ys, ref["y"], TOL[torch.bfloat16], "y")
    assert_close(st, ref["state"], 1e-4, "state")


def test_gated_tensor_core_beyond_int32_elements(orc):
    """The gated state scan's tensor-core form with q and k of more than 2^31 elements
    (8200 x 2048 x 128 bf16, 4.3 GB each; dv 64): every output and final-state entry of
    sampled batch items (the first, the last and two around the middle) against the oracle.
    Inputs drawn on the device as the input module draws them: q, k standard normal over
    sqrt(dk), v standard normal, gamma mostly in [0.5, 1) with about 1% exact zeros and 1%
    exact ones."""
    batch, seq, dk, dv = 8200, 2048, 128, 64
    assert batch * seq * dk > 2**31
    gd = torch.Generator(device="cuda").manual_seed(2600)
    sc = dk ** -0.5
    d = {"q": (torch.randn(batch, seq, dk, generator=gd, device="cuda") * sc).to(torch.bfloat16),
         "k": (torch.randn(batch, seq, dk, generator=gd, device="cuda") * sc).to(torch.bfloat16),
         "v": torch.randn(batch, seq, dv, generator=gd, device="cuda", dtype=torch.bfloat16)}
    g = 0.5 + 0.5 * torch.rand(batch, seq, generator=gd, device="cuda")
    u = torch.rand(batch, seq, generator=gd, device="cuda")
    d["gamma"] = torch.where(u < 0.01, torch.zeros_like(g), torch.where(u > 0.99, torch.ones_like(g), g)).contiguous()
    out = ssscan.ss_gated_scan(d["q"], d["k"], d["v"], d["gamma"])
    assert ssscan.ss_debug_status() == "SS_OK"
    items = [0, batch // 2 - 1, batch // 2, batch - 1]
    y, fs = out["outputs"][items].cpu(), out["final_state"][items].cpu()
    del out
    for i, b in enumerate(items):
        ref = orc.gated_scan(**{k: v[b:b + 1].cpu() for k, v in d.items()})
        assert_close(y[i:i + 1], ref["outputs"], TOL[torch.bfloat16], f"outputs item {b}")
        assert_close(fs[i:i + 1], ref["final_state"], TOL[torch.bfloat16], f"final_state item {b}")
