"""ctypes binding of ``libssscan.so`` (C declarations: include/ss_scan.h).

Argument marshalling only: tensors are checked, made contiguous, outputs are
allocated with torch, and the device pointers plus the current CUDA stream are
handed to the C entry points of the same names.  Every step of the scan runs in
the library's kernels; there is no other code path, and a missing library is an
error, never a fallback.
"""
from __future__ import annotations

import ctypes
import functools
import itertools
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssscan.so")
# the same sources compiled with SS_BOUNDS_CHECK (a debug build, for the index-check tests)
BOUNDS_LIB_PATH = os.path.join(_PKG, "libssscan_bounds.so")

SS_F32, SS_BF16 = 0, 1
SS_DT_SOFTPLUS = 1
SS_SCRATCH_ZERO = 2
SS_STATIC_SCRATCH_BYTES = 1 << 20
STATUS = {0: "SS_OK", 1: "SS_ERR_NULL", 2: "SS_ERR_SHAPE", 3: "SS_ERR_DTYPE", 4: "SS_ERR_ALIGN",
          5: "SS_ERR_UNSUPPORTED", 6: "SS_ERR_CUDA", 7: "SS_ERR_TIMEOUT", 8: "SS_ERR_ALIAS",
          9: "SS_ERR_WORKSPACE", 10: "SS_ERR_SCRATCH_LIMIT"}
EXPORTS = ("ss_scan_fwd", "ss_scan_workspace_bytes", "ss_scan_plan", "ss_scan_status", "ss_debug_status",
           "ss_state_update",
           "ss_debug_set_wait_limit", "ss_debug_set_scan_layout", "ss_debug_set_scan_two_level",
           "ss_debug_set_gated_path",
           "ss_status_string", "ss_abi_version", "ss_debug_mufu_probe", "ss_debug_bounds_status",
           "ss_scan_fwd_static_scratch", "ss_scan_fwd_states", "ss_gated_scan", "ss_scan_fwd_conv",
           "ss_state_update_conv", "ss_segment_decay", "ss_join_segments")
ABI_MAJOR = 3

_lock = threading.Lock()
_lib = None
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64


class ScanPlan(ctypes.Structure):
    """ss_scan_plan_t: the launch plan of ss_scan_fwd for a shape."""
    _fields_ = [("grid", ctypes.c_int64), ("ctas_per_sm", ctypes.c_int64), ("sms", ctypes.c_int64),
                ("groups", ctypes.c_int64), ("segments", ctypes.c_int64), ("seg_len", ctypes.c_int64),
                ("states_per_lane", ctypes.c_int64), ("two_level", ctypes.c_int64)]


class SSError(RuntimeError):
    """A non-zero status returned by the library."""

    def __init__(self, fn: str, status: int):
        self.status = status
        msg = load_library().ss_status_string(status).decode()
        super().__init__(f"{fn} failed: {msg} (status {status})")


def load_library(path: str = LIB_PATH):
    """Load (once) and return the ctypes handle of ``libssscan.so``."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(
                    f"{path} is not built; run `python -m selective_state_space_18_b200.build`")
            lib = ctypes.CDLL(path)
            lib.ss_scan_fwd.argtypes = [_i64, _i64, _i64, _i64, ctypes.c_int] + [_vp] * 10 + [
                ctypes.c_uint32, _vp, _vp, _vp, ctypes.c_size_t, _vp]
            lib.ss_scan_fwd.restype = ctypes.c_int
            lib.ss_scan_fwd_states.argtypes = [_i64, _i64, _i64, _i64, ctypes.c_int] + [_vp] * 10 + [
                ctypes.c_uint32, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
            lib.ss_scan_fwd_states.restype = ctypes.c_int
            lib.ss_scan_fwd_static_scratch.argtypes = [_i64, _i64, _i64, _i64, ctypes.c_int] + [_vp] * 10 + [
                ctypes.c_uint32, _vp, _vp, ctypes.POINTER(_vp), _vp]
            lib.ss_scan_fwd_static_scratch.restype = ctypes.c_int
            lib.ss_scan_fwd_conv.argtypes = [_i64, _i64, _i64, _i64, ctypes.c_int] + [_vp] * 3 + [_i64] + [_vp] * 12 + [
                ctypes.c_uint32, _vp, _vp, _vp, ctypes.c_size_t, _vp]
            lib.ss_scan_fwd_conv.restype = ctypes.c_int
            lib.ss_state_update_conv.argtypes = [_i64, _i64, _i64, ctypes.c_int] + [_vp] * 4 + [_i64] + [_vp] * 8 + [
                ctypes.c_uint32, _vp, _vp]
            lib.ss_state_update_conv.restype = ctypes.c_int
            lib.ss_gated_scan.argtypes = [_i64, _i64, _i64, _i64, ctypes.c_int] + [_vp] * 7 + [_vp]
            lib.ss_gated_scan.restype = ctypes.c_int
            lib.ss_segment_decay.argtypes = [_i64, _i64, _i64, _i64, ctypes.c_int] + [_vp] * 4 + [
                ctypes.c_uint32, _vp, _vp]
            lib.ss_segment_decay.restype = ctypes.c_int
            lib.ss_join_segments.argtypes = [_i64, _i64, _vp, _i64, _vp, _vp, _vp]
            lib.ss_join_segments.restype = ctypes.c_int
            lib.ss_scan_plan.argtypes = [_i64, _i64, _i64, _i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.POINTER(ScanPlan)]
            lib.ss_scan_plan.restype = ctypes.c_int
            lib.ss_scan_workspace_bytes.argtypes = [_i64, _i64, _i64, _i64]
            lib.ss_scan_workspace_bytes.restype = _i64
            lib.ss_scan_status.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_int)]
            lib.ss_scan_status.restype = ctypes.c_int
            lib.ss_state_update.argtypes = [_i64, _i64, _i64, ctypes.c_int] + [_vp] * 9 + [
                ctypes.c_uint32, _vp, _vp]
            lib.ss_state_update.restype = ctypes.c_int
            lib.ss_status_string.argtypes = [ctypes.c_int]
            lib.ss_status_string.restype = ctypes.c_char_p
            lib.ss_debug_set_wait_limit.argtypes = [ctypes.c_uint32]
            lib.ss_debug_set_wait_limit.restype = ctypes.c_int
            lib.ss_debug_set_scan_layout.argtypes = [ctypes.c_int]
            lib.ss_debug_set_scan_layout.restype = ctypes.c_int
            lib.ss_debug_set_gated_path.argtypes = [ctypes.c_int]
            lib.ss_debug_set_gated_path.restype = ctypes.c_int
            lib.ss_debug_set_scan_two_level.argtypes = [ctypes.c_int]
            lib.ss_debug_set_scan_two_level.restype = ctypes.c_int
            lib.ss_debug_mufu_probe.argtypes = [ctypes.c_int, _i64, _i64, _vp, _vp, ctypes.POINTER(_i64), _vp]
            lib.ss_debug_mufu_probe.restype = ctypes.c_int
            lib.ss_debug_bounds_status.argtypes = [_vp, ctypes.POINTER(ctypes.c_int)]
            lib.ss_debug_bounds_status.restype = ctypes.c_int
            lib.ss_debug_status.argtypes = [_vp]
            lib.ss_debug_status.restype = ctypes.c_int
            lib.ss_abi_version.argtypes = []
            lib.ss_abi_version.restype = ctypes.c_int
            if lib.ss_abi_version() >> 16 != ABI_MAJOR:
                raise RuntimeError(f"{path}: ABI {lib.ss_abi_version() >> 16}, expected {ABI_MAJOR}")
            _lib = lib
    return _lib


def _on_tensor_device(fn):
    """Run a wrapper with the device of its first tensor argument current: the library
    looks up per-device state (kernel attributes, occupancy, status words, the static
    scratch) for the current device, which must be the one the launch goes to."""
    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        dev = next((a.device for a in itertools.chain(args, kwargs.values())
                    if isinstance(a, torch.Tensor)), None)
        if dev is None or dev.type != "cuda":
            return fn(*args, **kwargs)
        with torch.cuda.device(dev):
            return fn(*args, **kwargs)
    return wrapper


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SS_F32
    if t.dtype == torch.bfloat16:
        return SS_BF16
    raise TypeError(f"x must be float32 or bfloat16, got {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _prep(t, name, device, dtype=None, shape=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.contiguous()


def _out(t, name, device, dtype, shape):
    """A caller-supplied output: written in place, so it must already be contiguous."""
    if t.device != device or t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be a {dtype} tensor of shape {tuple(shape)} on {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


_workspaces = {}


def scan_workspace(batch, channels, state_dim, seq, device, stream=None):
    """A zero-initialised workspace for ss_scan_fwd, cached per (device, stream) and
    grown on demand.  Calls on one stream are ordered, so they may share it."""
    need = int(load_library().ss_scan_workspace_bytes(batch, channels, state_dim, seq))
    if need <= 0:
        raise ValueError("invalid scan shape")
    if stream is None:
        stream = torch.cuda.current_stream(device)
    key = (device.index, stream.cuda_stream)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < need:
        with torch.cuda.stream(stream):
            ws = torch.zeros(max(need, 1 << 16), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def ss_scan_plan(batch, channels, state_dim, seq, dtype=torch.bfloat16, *, has_reset=False, workspace=True,
                 device=None):
    """Launch plan of ss_scan_fwd for this shape on `device` (16-byte aligned tensors):
    dict(grid, ctas_per_sm, sms, groups, segments, seg_len, states_per_lane, two_level).
    Launches nothing."""
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    code = SS_BF16 if dtype == torch.bfloat16 else SS_F32
    plan = ScanPlan()
    with torch.cuda.device(device):
        st = load_library().ss_scan_plan(batch, channels, state_dim, seq, code, int(bool(has_reset)),
                                         int(bool(workspace)), ctypes.byref(plan))
    if st != 0:
        raise SSError("ss_scan_plan", st)
    return {name: int(getattr(plan, name)) for name, _ in ScanPlan._fields_}


def ss_scan_status(workspace=None, stream=None, device=None):
    """Read and clear the device status word of earlier scans (synchronises the
    stream): 'SS_OK' or 'SS_ERR_TIMEOUT'."""
    if device is None:
        device = workspace.device if workspace is not None else torch.device("cuda", torch.cuda.current_device())
    out = ctypes.c_int(-1)
    with torch.cuda.device(device):
        st = load_library().ss_scan_status(_ptr(workspace), _stream(stream, device), ctypes.byref(out))
    if st != 0:
        raise SSError("ss_scan_status", st)
    return STATUS[out.value]


def ss_debug_status(stream=None, device=None):
    """Read and clear the device status word of the calls made without a workspace on
    `device` (synchronises the stream): 'SS_OK' or 'SS_ERR_TIMEOUT'."""
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(device):
        st = load_library().ss_debug_status(_stream(stream, device))
    if st not in (0, 7):
        raise SSError("ss_debug_status", st)
    return STATUS[st]


def ss_debug_set_scan_layout(states_per_lane: int) -> None:
    """Force the state_dim-16 scan layout (2 or 4 states per scan lane; 0: automatic)
    for later calls.  A testing aid: both layouts compute the same results."""
    st = load_library().ss_debug_set_scan_layout(int(states_per_lane))
    if st != 0:
        raise SSError("ss_debug_set_scan_layout", st)


def ss_debug_set_scan_two_level(mode: int) -> None:
    """Schedule of later state_dim-16 scans with a workspace: 0 automatic, 1 never the
    two-level schedule, 2 whenever the sequence allows it.  A testing aid."""
    st = load_library().ss_debug_set_scan_two_level(int(mode))
    if st != 0:
        raise SSError("ss_debug_set_scan_two_level", st)


def mufu_rate(op="ex2", iters=1 << 16, device=None):
    """Measured results per clock per SM of the special-function unit (op "ex2" or
    "tanh"): one 512-thread CTA per SM, the SM cycle counter around the loop.  Returns
    (median rate, [per-SM rates])."""
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    code = {"ex2": 0, "tanh": 1}[op]
    with torch.cuda.device(device):
        sms = torch.cuda.get_device_properties(device).multi_processor_count
        cycles = torch.zeros(sms, dtype=torch.int64, device=device)
        sink = torch.zeros(512, dtype=torch.float32, device=device)
        ops = _i64(0)
        st = load_library().ss_debug_mufu_probe(code, int(iters), sms, _ptr(cycles), _ptr(sink),
                                                ctypes.byref(ops), _stream(None, device))
        if st != 0:
            raise SSError("ss_debug_mufu_probe", st)
        torch.cuda.synchronize(device)
    rates = [ops.value / float(c) for c in cycles.cpu().tolist() if c > 0]
    rates.sort()
    return rates[len(rates) // 2], rates


def ss_debug_set_gated_path(mode: int) -> None:
    """Kernel of later ss_gated_scan calls: 0 automatic (the tensor-core chunked form
    where it applies), 1 always the token-by-token recurrence, 3 automatic with the
    tensor-core form's first "L o S written" arrival withheld (its wait runs out on the
    wait limit: a failure-path test aid).  A testing aid."""
    st = load_library().ss_debug_set_gated_path(int(mode))
    if st != 0:
        raise SSError("ss_debug_set_gated_path", st)


def ss_debug_set_wait_limit(microseconds: int) -> None:
    """Cap device-side waits of later calls at `microseconds` (0: the 2 s default)."""
    st = load_library().ss_debug_set_wait_limit(int(microseconds))
    if st != 0:
        raise SSError("ss_debug_set_wait_limit", st)


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


@_on_tensor_device
def ss_scan_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, reset=None, h0=None, *,
                dt_softplus=True, y=None, h_last=None, return_last_state=True, stream=None,
                workspace=True, h_all=None, return_states=False, betas=None, return_betas=False):
    """Prompt scan.  x, dt, z: [batch, channels, seq]; B, C: [batch, state_dim, seq];
    A: [channels, state_dim] fp32; D, dt_bias: [channels] fp32; reset: [batch, seq]
    bool/uint8; h0: [batch, channels, state_dim] fp32.  Returns (y, h_last), or
    (y, h_last, h_all) with the state after every token [batch, channels, seq,
    state_dim] fp32 when return_states is set or h_all is given (ss_scan_fwd_states),
    or (y, h_last, h_all or None, betas) with every token's step size [batch, channels,
    seq] fp32 as well when return_betas is set or betas is given (the log decays are
    betas[..., None] * A[:, None, :] per batch row).

    workspace: True (a cached per-stream workspace: segmented, balanced schedule),
    False (none: one CTA per channel group) or a zero-initialised uint8 tensor."""
    if x.dim() != 3:
        raise ValueError("x must be [batch, channels, seq]")
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("ss_scan_fwd runs on CUDA tensors only")
    bt, ch, L = x.shape
    n = A.shape[-1]
    code = _dtype_code(x)
    x = _prep(x, "x", dev)
    dt = _prep(dt, "dt", dev, x.dtype, (bt, ch, L))
    z = _prep(z, "z", dev, x.dtype, (bt, ch, L))
    B = _prep(B, "B", dev, x.dtype, (bt, n, L))
    C = _prep(C, "C", dev, x.dtype, (bt, n, L))
    A = _prep(A, "A", dev, torch.float32, (ch, n))
    D = _prep(D, "D", dev, torch.float32, (ch,))
    dt_bias = _prep(dt_bias, "dt_bias", dev, torch.float32, (ch,))
    h0 = _prep(h0, "h0", dev, torch.float32, (bt, ch, n))
    if reset is not None:
        reset = _prep(reset, "reset", dev, None, (bt, L))
        if reset.dtype == torch.bool:
            reset = reset.view(torch.uint8)
        elif reset.dtype != torch.uint8:
            raise TypeError("reset must be bool or uint8")
    if y is None:
        y = torch.empty_like(x)
    else:
        y = _out(y, "y", dev, x.dtype, (bt, ch, L))
    if h_last is None and return_last_state:
        h_last = torch.empty(bt, ch, n, device=dev, dtype=torch.float32)
    elif h_last is not None:
        h_last = _out(h_last, "h_last", dev, torch.float32, (bt, ch, n))
    flags = SS_DT_SOFTPLUS if dt_softplus else 0
    lib = load_library()
    states = return_states or h_all is not None
    if h_all is None and states:
        h_all = torch.empty(bt, ch, L, n, device=dev, dtype=torch.float32)
    elif h_all is not None:
        h_all = _out(h_all, "h_all", dev, torch.float32, (bt, ch, L, n))
    steps = return_betas or betas is not None
    if betas is None and steps:
        betas = torch.empty(bt, ch, L, device=dev, dtype=torch.float32)
    elif betas is not None:
        betas = _out(betas, "betas", dev, torch.float32, (bt, ch, L))
    if workspace is True:
        workspace = scan_workspace(bt, ch, n, L, dev, stream)
    elif workspace is False or workspace is None:
        workspace = None
    elif workspace.device != dev or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous uint8 tensor on the inputs' device")
    ws_bytes = 0 if workspace is None else workspace.numel()
    if states or steps:
        st = lib.ss_scan_fwd_states(bt, ch, n, L, code, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                                    _ptr(D), _ptr(z), _ptr(dt_bias), _ptr(reset), _ptr(h0), flags,
                                    _ptr(y), _ptr(h_last), _ptr(h_all), _ptr(betas), _ptr(workspace), ws_bytes,
                                    _stream(stream, dev))
        if st != 0:
            raise SSError("ss_scan_fwd_states", st)
        return (y, h_last, h_all, betas) if steps else (y, h_last, h_all)
    st = lib.ss_scan_fwd(bt, ch, n, L, code, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                         _ptr(D), _ptr(z), _ptr(dt_bias), _ptr(reset), _ptr(h0), flags,
                         _ptr(y), _ptr(h_last), _ptr(workspace), ws_bytes, _stream(stream, dev))
    if st != 0:
        raise SSError("ss_scan_fwd", st)
    return y, h_last


@_on_tensor_device
def ss_state_update(state, x, dt, A, B, C, D=None, z=None, dt_bias=None, *, dt_softplus=True,
                    y=None, stream=None):
    """Decode step, ``state`` [batch, channels, state_dim] fp32 updated in place.
    x, dt, z: [batch, channels]; B, C: [batch, state_dim].  Returns y [batch, channels]."""
    if state.dim() != 3 or state.dtype != torch.float32:
        raise ValueError("state must be a [batch, channels, state_dim] float32 tensor")
    if not state.is_contiguous():
        raise ValueError("state must be contiguous (it is updated in place)")
    dev = state.device
    if dev.type != "cuda":
        raise ValueError("ss_state_update runs on CUDA tensors only")
    bt, ch, n = state.shape
    code = _dtype_code(x)
    x = _prep(x, "x", dev, None, (bt, ch))
    dt = _prep(dt, "dt", dev, x.dtype, (bt, ch))
    z = _prep(z, "z", dev, x.dtype, (bt, ch))
    B = _prep(B, "B", dev, x.dtype, (bt, n))
    C = _prep(C, "C", dev, x.dtype, (bt, n))
    A = _prep(A, "A", dev, torch.float32, (ch, n))
    D = _prep(D, "D", dev, torch.float32, (ch,))
    dt_bias = _prep(dt_bias, "dt_bias", dev, torch.float32, (ch,))
    if y is None:
        y = torch.empty(bt, ch, device=dev, dtype=x.dtype)
    else:
        y = _out(y, "y", dev, x.dtype, (bt, ch))
    flags = SS_DT_SOFTPLUS if dt_softplus else 0
    lib = load_library()
    st = lib.ss_state_update(bt, ch, n, code, _ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                             _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias), flags, _ptr(y),
                             _stream(stream, dev))
    if st != 0:
        raise SSError("ss_state_update", st)
    return y


_scratch_addr = {}


@_on_tensor_device
def ss_scan_fwd_static_scratch(x, dt, A, B, C, D=None, z=None, dt_bias=None, reset=None, h0=None, *,
                               dt_softplus=True, y=None, h_last=None, return_last_state=True,
                               stream=None, zero_scratch=False):
    """Prompt scan through the library's fixed per-device scratch instead of a
    workspace (for callers that cannot allocate device memory when they scan; the
    library call allocates nothing -- outputs not supplied here are allocated by
    torch before it).  Same tensors and results as ``ss_scan_fwd``; shapes that need
    more than SS_STATIC_SCRATCH_BYTES of workspace raise SS_ERR_SCRATCH_LIMIT.
    Calls on one device share the scratch, so they must not overlap in time."""
    if x.dim() != 3:
        raise ValueError("x must be [batch, channels, seq]")
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("ss_scan_fwd_static_scratch runs on CUDA tensors only")
    bt, ch, L = x.shape
    n = A.shape[-1]
    code = _dtype_code(x)
    x = _prep(x, "x", dev)
    dt = _prep(dt, "dt", dev, x.dtype, (bt, ch, L))
    z = _prep(z, "z", dev, x.dtype, (bt, ch, L))
    B = _prep(B, "B", dev, x.dtype, (bt, n, L))
    C = _prep(C, "C", dev, x.dtype, (bt, n, L))
    A = _prep(A, "A", dev, torch.float32, (ch, n))
    D = _prep(D, "D", dev, torch.float32, (ch,))
    dt_bias = _prep(dt_bias, "dt_bias", dev, torch.float32, (ch,))
    h0 = _prep(h0, "h0", dev, torch.float32, (bt, ch, n))
    if reset is not None:
        reset = _prep(reset, "reset", dev, None, (bt, L))
        if reset.dtype == torch.bool:
            reset = reset.view(torch.uint8)
        elif reset.dtype != torch.uint8:
            raise TypeError("reset must be bool or uint8")
    y = torch.empty_like(x) if y is None else _out(y, "y", dev, x.dtype, (bt, ch, L))
    if h_last is None and return_last_state:
        h_last = torch.empty(bt, ch, n, device=dev, dtype=torch.float32)
    elif h_last is not None:
        h_last = _out(h_last, "h_last", dev, torch.float32, (bt, ch, n))
    flags = (SS_DT_SOFTPLUS if dt_softplus else 0) | (SS_SCRATCH_ZERO if zero_scratch else 0)
    addr = _vp()
    st = load_library().ss_scan_fwd_static_scratch(
        bt, ch, n, L, code, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(dt_bias), _ptr(reset), _ptr(h0), flags, _ptr(y), _ptr(h_last), ctypes.byref(addr),
        _stream(stream, dev))
    if st != 0:
        raise SSError("ss_scan_fwd_static_scratch", st)
    _scratch_addr[dev.index] = addr.value
    return y, h_last


def static_scratch_status(stream=None, device=None):
    """Read and clear the device status word of ss_scan_fwd_static_scratch calls on
    `device` (synchronises the stream): 'SS_OK' or 'SS_ERR_TIMEOUT'."""
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    addr = _scratch_addr.get(device.index)
    if addr is None:
        raise RuntimeError("no ss_scan_fwd_static_scratch call has run on this device")
    out = ctypes.c_int(-1)
    with torch.cuda.device(device):
        st = load_library().ss_scan_status(_vp(addr), _stream(stream, device), ctypes.byref(out))
    if st != 0:
        raise SSError("ss_scan_status", st)
    return STATUS[out.value]


@_on_tensor_device
def ss_gated_scan(q, k, v, gamma, h0=None, *, stream=None):
    """Gated state scan S_t = gamma_t S_{t-1} + k_t v_t^T, y_t = q_t^T S_t.  q, k:
    [B, S, Dk]; v: [B, S, Dv] (float32 or bfloat16, same dtype); gamma: [B, S] float32;
    h0: [B, Dk, Dv] float32 or None.  Non-contiguous inputs are copied, never modified.
    Returns {"outputs": [B, S, Dv], "final_state": [B, Dk, Dv]} in the dtype of q."""
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("ss_gated_scan runs on CUDA tensors only")
    if q.dim() != 3:
        raise ValueError("q must be [B, S, Dk]")
    bt, sl, dk = q.shape
    dv = v.shape[-1]
    code = _dtype_code(q)
    q = _prep(q, "q", dev)
    k = _prep(k, "k", dev, q.dtype, (bt, sl, dk))
    v = _prep(v, "v", dev, q.dtype, (bt, sl, dv))
    gamma = _prep(gamma, "gamma", dev, torch.float32, (bt, sl))
    h0 = _prep(h0, "h0", dev, torch.float32, (bt, dk, dv))
    y = torch.empty(bt, sl, dv, device=dev, dtype=q.dtype)
    fs = torch.empty(bt, dk, dv, device=dev, dtype=q.dtype)
    st = load_library().ss_gated_scan(bt, sl, dk, dv, code, _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(h0),
                                      _ptr(y), _ptr(fs), _stream(stream, dev))
    if st != 0:
        raise SSError("ss_gated_scan", st)
    return {"outputs": y, "final_state": fs}


@_on_tensor_device
def ss_scan_fwd_conv(u, conv_w, dt, A, B, C, D=None, z=None, dt_bias=None, reset=None, h0=None, *,
                     conv_b=None, conv_state=None, dt_softplus=True, return_conv_state=True,
                     return_x=False, stream=None, workspace=True):
    """Prompt scan with the causal depthwise conv + SiLU fused in front: u is the conv
    input [batch, channels, seq] (the scan's x = silu(conv(u))); conv_w [channels, K]
    fp32 (K <= 4); conv_b [channels] fp32; conv_state [batch, channels, K-1] fp32 (the
    inputs before u).  Returns dict(y, h_last, conv_state (the last K-1 inputs, for the
    next call), x (when return_x))."""
    dev = u.device
    if dev.type != "cuda":
        raise ValueError("ss_scan_fwd_conv runs on CUDA tensors only")
    if u.dim() != 3:
        raise ValueError("u must be [batch, channels, seq]")
    bt, ch, L = u.shape
    n = A.shape[-1]
    K = conv_w.shape[-1]
    code = _dtype_code(u)
    u = _prep(u, "u", dev)
    conv_w = _prep(conv_w, "conv_w", dev, torch.float32, (ch, K))
    conv_b = _prep(conv_b, "conv_b", dev, torch.float32, (ch,))
    conv_state = _prep(conv_state, "conv_state", dev, torch.float32, (bt, ch, K - 1))
    dt = _prep(dt, "dt", dev, u.dtype, (bt, ch, L))
    z = _prep(z, "z", dev, u.dtype, (bt, ch, L))
    B = _prep(B, "B", dev, u.dtype, (bt, n, L))
    C = _prep(C, "C", dev, u.dtype, (bt, n, L))
    A = _prep(A, "A", dev, torch.float32, (ch, n))
    D = _prep(D, "D", dev, torch.float32, (ch,))
    dt_bias = _prep(dt_bias, "dt_bias", dev, torch.float32, (ch,))
    h0 = _prep(h0, "h0", dev, torch.float32, (bt, ch, n))
    if reset is not None:
        reset = _prep(reset, "reset", dev, None, (bt, L))
        reset = reset.view(torch.uint8) if reset.dtype == torch.bool else reset
    y = torch.empty_like(u)
    h_last = torch.empty(bt, ch, n, device=dev, dtype=torch.float32)
    cs_out = torch.empty(bt, ch, K - 1, device=dev, dtype=torch.float32) if return_conv_state and K > 1 else None
    x_out = torch.empty_like(u) if return_x else None
    if workspace is True:
        workspace = scan_workspace(bt, ch, n, L, dev, stream)
    elif workspace is False or workspace is None:
        workspace = None
    ws_bytes = 0 if workspace is None else workspace.numel()
    flags = SS_DT_SOFTPLUS if dt_softplus else 0
    st = load_library().ss_scan_fwd_conv(
        bt, ch, n, L, code, _ptr(u), _ptr(conv_w), _ptr(conv_b), K, _ptr(conv_state), _ptr(cs_out), _ptr(x_out),
        _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias), _ptr(reset), _ptr(h0), flags,
        _ptr(y), _ptr(h_last), _ptr(workspace), ws_bytes, _stream(stream, dev))
    if st != 0:
        raise SSError("ss_scan_fwd_conv", st)
    out = {"y": y, "h_last": h_last, "conv_state": cs_out}
    if return_x:
        out["x"] = x_out
    return out


@_on_tensor_device
def ss_state_update_conv(state, conv_state, conv_w, u, dt, A, B, C, D=None, z=None, dt_bias=None, *,
                         conv_b=None, dt_softplus=True, stream=None):
    """Decode step of the fused conv form: ``state`` [batch, channels, state_dim] fp32 and
    ``conv_state`` [batch, channels, K-1] fp32 are updated in place; u is the new conv
    input [batch, channels].  Returns y [batch, channels]."""
    dev = state.device
    if dev.type != "cuda":
        raise ValueError("ss_state_update_conv runs on CUDA tensors only")
    bt, ch, n = state.shape
    K = conv_w.shape[-1]
    code = _dtype_code(u)
    if state.dtype != torch.float32 or not state.is_contiguous():
        raise ValueError("state must be a contiguous float32 tensor (updated in place)")
    if K > 1 and (conv_state is None or conv_state.dtype != torch.float32 or not conv_state.is_contiguous()
                  or tuple(conv_state.shape) != (bt, ch, K - 1)):
        raise ValueError("conv_state must be a contiguous float32 [batch, channels, K-1] tensor (updated in place)")
    u = _prep(u, "u", dev, None, (bt, ch))
    dt = _prep(dt, "dt", dev, u.dtype, (bt, ch))
    z = _prep(z, "z", dev, u.dtype, (bt, ch))
    B = _prep(B, "B", dev, u.dtype, (bt, n))
    C = _prep(C, "C", dev, u.dtype, (bt, n))
    A = _prep(A, "A", dev, torch.float32, (ch, n))
    D = _prep(D, "D", dev, torch.float32, (ch,))
    dt_bias = _prep(dt_bias, "dt_bias", dev, torch.float32, (ch,))
    conv_w = _prep(conv_w, "conv_w", dev, torch.float32, (ch, K))
    conv_b = _prep(conv_b, "conv_b", dev, torch.float32, (ch,))
    y = torch.empty(bt, ch, device=dev, dtype=u.dtype)
    flags = SS_DT_SOFTPLUS if dt_softplus else 0
    st = load_library().ss_state_update_conv(bt, ch, n, code, _ptr(state), _ptr(conv_state if K > 1 else None),
                                             _ptr(conv_w), _ptr(conv_b), K, _ptr(u), _ptr(dt), _ptr(A), _ptr(B),
                                             _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias), flags, _ptr(y),
                                             _stream(stream, dev))
    if st != 0:
        raise SSError("ss_state_update_conv", st)
    return y


@_on_tensor_device
def ss_segment_decay(dt, A, dt_bias=None, reset=None, *, dt_softplus=True, out=None, stream=None):
    """Decay of one segment of a sequence: [batch, channels, state_dim] fp32 =
    exp(A * sum of the segment's step sizes), 0 where the segment holds a reset.
    dt: [batch, channels, seq] (the segment's slice); reset: [batch, seq] or None.
    ``out`` (contiguous fp32) is written in place when given."""
    if dt.dim() != 3:
        raise ValueError("dt must be [batch, channels, seq]")
    dev = dt.device
    if dev.type != "cuda":
        raise ValueError("ss_segment_decay runs on CUDA tensors only")
    bt, ch, L = dt.shape
    n = A.shape[-1]
    code = _dtype_code(dt)
    dt = _prep(dt, "dt", dev)
    A = _prep(A, "A", dev, torch.float32, (ch, n))
    dt_bias = _prep(dt_bias, "dt_bias", dev, torch.float32, (ch,))
    if reset is not None:
        reset = _prep(reset, "reset", dev, None, (bt, L))
        if reset.dtype == torch.bool:
            reset = reset.view(torch.uint8)
        elif reset.dtype != torch.uint8:
            raise TypeError("reset must be bool or uint8")
    if out is None:
        out = torch.empty(bt, ch, n, device=dev, dtype=torch.float32)
    else:
        out = _out(out, "out", dev, torch.float32, (bt, ch, n))
    flags = SS_DT_SOFTPLUS if dt_softplus else 0
    st = load_library().ss_segment_decay(bt, ch, n, L, code, _ptr(dt), _ptr(A), _ptr(dt_bias), _ptr(reset),
                                         flags, _ptr(out), _stream(stream, dev))
    if st != 0:
        raise SSError("ss_segment_decay", st)
    return out


@_on_tensor_device
def ss_join_segments(composites, rank=None, *, carry=None, final_state=None, want_final=True, stream=None):
    """Fold gathered segment composites [segments, 2, ...] (decay, end state; fp32,
    contiguous) in segment order.  Returns (carry, final_state): the state entering
    segment ``rank`` (None when rank is None) and, when ``want_final``, the state
    after the last segment; both have the composites' trailing shape."""
    if composites.dim() < 3 or composites.shape[1] != 2:
        raise ValueError("composites must be [segments, 2, ...]")
    dev = composites.device
    if dev.type != "cuda":
        raise ValueError("ss_join_segments runs on CUDA tensors only")
    if composites.dtype != torch.float32 or not composites.is_contiguous():
        raise ValueError("composites must be a contiguous float32 tensor")
    segs = composites.shape[0]
    shape = tuple(composites.shape[2:])
    count = composites[0, 0].numel()
    if rank is not None and carry is None:
        carry = torch.empty(shape, device=dev, dtype=torch.float32)
    elif carry is not None:
        carry = _out(carry, "carry", dev, torch.float32, shape)
    if want_final and final_state is None:
        final_state = torch.empty(shape, device=dev, dtype=torch.float32)
    elif final_state is not None:
        final_state = _out(final_state, "final_state", dev, torch.float32, shape)
    st = load_library().ss_join_segments(segs, count, _ptr(composites), -1 if rank is None else int(rank),
                                         _ptr(carry), _ptr(final_state), _stream(stream, dev))
    if st != 0:
        raise SSError("ss_join_segments", st)
    return carry, final_state
