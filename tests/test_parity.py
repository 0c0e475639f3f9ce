"""GPU path (through the C ABI) against the float64 oracle on identical seeded
inputs, elementwise: max |out - ref| <= 1e-4 (1 + |ref|) for fp32 tensors and
<= 1e-2 (1 + |ref|) for bf16 ones (fp32 state and accumulation in both)."""
import pytest
import torch

from gpu_util import TOL, assert_close, gpu_scan, gpu_update, schedule
from selective_state_space_18_b200.inputs import make_scan_inputs, make_update_inputs, make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


# ---- the tiny fp32 workload, all optional-input combinations ----------------------------

@pytest.mark.parametrize("use_z", [True, False])
@pytest.mark.parametrize("use_bias", [True, False])
@pytest.mark.parametrize("use_h0", [False, True])
def test_tiny_fp32(orc, use_z, use_bias, use_h0):
    inp = make_workload("tiny_fp32", z=use_z, dt_bias=use_bias, h0=use_h0)
    ref = orc.scan(**inp)
    y, h = gpu_scan(inp)
    assert_close(y, ref["y"], 1e-4, "y")
    assert_close(h, ref["h_last"], 1e-4, "h_last")


# ---- ragged shapes: seq tails, channel tails, every state_dim, both dtypes ----------------

RAGGED = [
    # batch, channels, N, seq, dtype, resets
    (1, 3, 4, 1, "f32", False),
    (2, 5, 8, 7, "f32", False),
    (1, 17, 16, 100, "bf16", False),
    (3, 33, 16, 65, "f32", True),
    (2, 70, 4, 129, "bf16", True),
    (1, 16, 16, 64, "bf16", False),
    (1, 20, 8, 1000, "f32", True),
    (2, 16, 16, 130, "bf16", True),
    (1, 48, 16, 513, "f32", False),
    (2, 9, 8, 4096, "bf16", True),
]


@pytest.mark.parametrize("case", RAGGED, ids=lambda c: "x".join(map(str, c)))
@pytest.mark.parametrize("softplus", [True, False])
def test_ragged_shapes(orc, case, softplus):
    bt, ch, n, L, dt_, resets = case
    inp = make_scan_inputs(bt, ch, n, L, dt_, seed=1000 + L + ch, h0=True,
                           reset_mean_doc=37 if resets else 0, a_perturb=True)
    if not softplus:
        inp["dt"] = (inp["dt"].float().abs() * 0.05).to(inp["dt"].dtype)
        inp["dt_bias"] = inp["dt_bias"].abs() * 0.01
    ref = orc.scan(**inp, dt_softplus=softplus)
    y, h = gpu_scan(inp, dt_softplus=softplus)
    tol = TOL[inp["x"].dtype]
    assert_close(y, ref["y"], tol, "y")
    assert_close(h, ref["h_last"], tol, "h_last")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_unaligned_views_take_scalar_path(orc, dtype):
    """Tensors that start 1 element past a 16-byte boundary (aligned to their element
    size only) must give the same results as the vector path."""
    bt, ch, n, L = 2, 24, 16, 96
    inp = make_scan_inputs(bt, ch, n, L, dtype, seed=77, reset_mean_doc=20)
    ref = orc.scan(**inp)
    d = {}
    for k, v in inp.items():
        if v is None:
            d[k] = None
            continue
        buf = torch.empty(v.numel() + 1, dtype=v.dtype, device="cuda")
        view = buf[1:].view(v.shape)
        view.copy_(v)
        d[k] = view
    from selective_state_space_18_b200 import ssscan
    yb = torch.empty(inp["x"].numel() + 1, dtype=inp["x"].dtype, device="cuda")
    y = yb[1:].view(inp["x"].shape)
    ssscan.ss_scan_fwd(**d, y=y)
    torch.cuda.synchronize()
    assert_close(y.cpu(), ref["y"], TOL[inp["x"].dtype], "y")


# ---- the benchmark workloads at full size -------------------------------------------------

def test_mamba130m_layer_full(orc):
    """8 x 1536 x 16 x 2048, bf16 in/out: every output against the oracle."""
    inp = make_workload("mamba130m_layer")
    y, h = gpu_scan(inp)
    ref = orc.scan(**inp)
    assert_close(y, ref["y"], 1e-2, "y")
    assert_close(h, ref["h_last"], 1e-2, "h_last")


@pytest.mark.parametrize("name", ["mamba2p8b_layer_long", "packed_resets"])
def test_long_workloads_full(orc, name):
    """1 x 5120 x 16 x 16384 and 2 x 2048 x 16 x 32768 (with resets), in the launch
    configuration the benchmark times (the segmented schedule with the binding's
    cached workspace): every output and every final-state entry against the oracle."""
    inp = make_workload(name)
    y, h = gpu_scan(inp)
    ref = orc.scan(**inp)
    assert_close(y, ref["y"], 1e-2, "y")
    assert_close(h, ref["h_last"], 1e-2, "h_last")


def test_decode_workload_full(orc):
    """256 x 5120 x 16 decode update, state in place: every output and state entry."""
    inp = make_workload("decode_2p8b")
    y, st = gpu_update(inp)
    ref = orc.update(**inp)
    assert_close(y, ref["y"], 1e-2, "y")
    assert_close(st, ref["state"], 1e-4, "state")


@pytest.mark.parametrize("n", [4, 8, 16])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("extras", [True, False])
def test_decode_shapes(orc, n, dtype, extras):
    inp = make_update_inputs(3, 37, n, dtype, seed=300 + n, z=extras, dt_bias=extras, D=extras)
    y, st = gpu_update(inp)
    ref = orc.update(**inp)
    assert_close(y, ref["y"], TOL[inp["x"].dtype], "y")
    assert_close(st, ref["state"], 1e-4, "state")


@pytest.mark.parametrize("batch,ch,n,dtype", [
    (600, 1000, 16, "bf16"),   # several tiles per CTA, one channel block per CTA, partial tiles
    (300, 1001, 8, "f32"),     # x/dt/z rows not 16-byte aligned: loaded per channel
    (97, 3000, 4, "bf16"),     # 4 states: 1024 channels per tile
])
def test_decode_streaming_tiles(orc, batch, ch, n, dtype):
    inp = make_update_inputs(batch, ch, n, dtype, seed=310 + n)
    y, st = gpu_update(inp)
    ref = orc.update(**inp)
    assert_close(y, ref["y"], TOL[inp["x"].dtype], "y")
    assert_close(st, ref["state"], 1e-4, "state")


def test_decode_unaligned_state(orc):
    """A state that is not 16-byte aligned takes the per-thread kernel; same results."""
    from selective_state_space_18_b200 import ssscan
    inp = make_update_inputs(5, 70, 16, "bf16", seed=320)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    buf = torch.empty(d["state"].numel() + 1, dtype=torch.float32, device="cuda")
    state = buf[1:].view(d["state"].shape)
    state.copy_(d["state"])
    assert state.data_ptr() % 16 != 0
    y = ssscan.ss_state_update(state, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["z"], d["dt_bias"])
    torch.cuda.synchronize()
    ref = orc.update(**inp)
    assert_close(y.cpu(), ref["y"], TOL[torch.bfloat16], "y")
    assert_close(state.cpu(), ref["state"], 1e-4, "state")


# ---- properties the pages fix, on the GPU path ---------------------------------------------

def test_decode_equals_last_scan_step():
    """scan(x[:L-1]) then one decode step == scan(x[:L]) on the last token."""
    inp = make_scan_inputs(2, 40, 16, 77, "f32", seed=88, h0=True)
    yf, hf = gpu_scan(inp)
    head = dict(inp)
    for k in ("x", "dt", "z", "B", "C"):
        head[k] = inp[k][:, :, :-1].contiguous()
    _, h1 = gpu_scan(head)
    step = {"state": h1, "x": inp["x"][:, :, -1], "dt": inp["dt"][:, :, -1], "A": inp["A"],
            "B": inp["B"][:, :, -1], "C": inp["C"][:, :, -1], "D": inp["D"],
            "z": inp["z"][:, :, -1], "dt_bias": inp["dt_bias"]}
    step = {k: v.contiguous() for k, v in step.items()}
    ys, hs = gpu_update(step)
    assert_close(ys, yf[:, :, -1].double().numpy(), 1e-4, "y")
    assert_close(hs, hf.double().numpy(), 1e-4, "state")


def test_chaining_through_h0_and_in_place():
    from selective_state_space_18_b200 import ssscan
    inp = make_scan_inputs(2, 20, 16, 300, "f32", seed=89)
    yf, hf = gpu_scan(inp)
    a, b = dict(inp), dict(inp)
    for k in ("x", "dt", "z", "B", "C"):
        a[k] = inp[k][:, :, :131].contiguous()
        b[k] = inp[k][:, :, 131:].contiguous()
    ya, ha = gpu_scan(a)
    b["h0"] = ha
    yb, hb = gpu_scan(b)
    assert_close(torch.cat([ya, yb], dim=2), yf.double().numpy(), 1e-4, "y")
    assert_close(hb, hf.double().numpy(), 1e-4, "h_last")
    # h_last written over h0 in place
    d = {k: (None if v is None else v.cuda()) for k, v in b.items()}
    h = d["h0"].clone()
    d["h0"] = h
    ssscan.ss_scan_fwd(**d, h_last=h)
    torch.cuda.synchronize()
    assert torch.equal(h.cpu(), hb)


def test_inputs_unchanged_and_deterministic():
    from selective_state_space_18_b200 import ssscan
    inp = make_scan_inputs(2, 48, 16, 500, "bf16", seed=90, reset_mean_doc=50, h0=True)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    before = {k: v.clone() for k, v in d.items() if v is not None}
    y1, h1 = ssscan.ss_scan_fwd(**d)
    y2, h2 = ssscan.ss_scan_fwd(**d)
    torch.cuda.synchronize()
    for k, v in before.items():
        assert torch.equal(d[k], v), k
    assert torch.equal(y1, y2) and torch.equal(h1, h2)


def test_batch_items_independent():
    inp = make_scan_inputs(3, 24, 16, 200, "f32", seed=91, reset_mean_doc=30, h0=True)
    y, h = gpu_scan(inp)
    for b in range(3):
        one = {k: (None if v is None else (v if k in ("A", "D", "dt_bias") else v[b:b + 1]))
               for k, v in inp.items()}
        yb, hb = gpu_scan(one)
        assert torch.equal(yb[0], y[b]) and torch.equal(hb[0], h[b])


# ---- the segmented (workspace) schedule against the one-CTA-per-group schedule -------------

@pytest.mark.parametrize("shape", [(1, 64, 16, 8192, "bf16", 0), (2, 40, 16, 3000, "f32", 300),
                                   (3, 100, 8, 2051, "bf16", 97), (1, 8, 4, 4096, "f32", 0)])
def test_segmented_schedule_is_bit_identical(shape):
    """The carry handed between segments is an exact copy, so splitting the sequence
    into segments on different CTAs must not change a single bit."""
    from selective_state_space_18_b200 import ssscan
    bt, ch, n, L, dt_, doc = shape
    inp = make_scan_inputs(bt, ch, n, L, dt_, seed=L + ch, h0=True, reset_mean_doc=doc)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    with schedule(two_level=1):  # the single-pass schedule (chained segments)
        y_static, h_static = ssscan.ss_scan_fwd(**d, workspace=False)
        y_seg, h_seg = ssscan.ss_scan_fwd(**d)
        ws = torch.zeros(int(ssscan.load_library().ss_scan_workspace_bytes(bt, ch, n, L)),
                         dtype=torch.uint8, device="cuda")
        outs = [ssscan.ss_scan_fwd(**d, workspace=ws) for _ in range(4)]
        torch.cuda.synchronize()
    assert torch.equal(y_static, y_seg) and torch.equal(h_static, h_seg)
    for y, h in outs:
        assert torch.equal(y, y_seg) and torch.equal(h, h_seg)
    assert ssscan.ss_scan_status(ws) == "SS_OK"
    assert ssscan.ss_scan_status(None) == "SS_OK"
