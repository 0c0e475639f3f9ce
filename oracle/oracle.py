"""Python front end of the float64 CPU oracle (``ss_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / ``--impl reference`` legs are the only callers.
The product path (``selective_state_space_18_b200``) never imports this module,
and this module never imports the product package.

Every input is widened exactly to float64 (bf16 and fp32 values are exactly
representable) before the C code sees it; outputs stay float64.  The C library
is compiled with gcc on first use (or by ``build()``) into ``oracle/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ss_oracle.c")
_LIB = os.path.join(_HERE, "libssoracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile ``ss_oracle.c`` into ``libssoracle.so`` (gcc, -O2, OpenMP, IEEE math)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-fno-fast-math", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.ss_oracle_scan.argtypes = [_i64, _i64, _i64, _i64] + [_dp] * 8 + [
                _u8p, _dp, ctypes.c_int, _dp, _dp, _dp, _dp, ctypes.c_int]
            lib.ss_oracle_scan.restype = ctypes.c_int
            lib.ss_oracle_tree_scan.argtypes = [_i64, _i64, _i64, _i64] + [_dp] * 8 + [
                _u8p, _dp, ctypes.c_int, _dp, _dp, ctypes.c_int]
            lib.ss_oracle_tree_scan.restype = ctypes.c_int
            lib.ss_oracle_update.argtypes = [_i64, _i64, _i64, _dp] + [_dp] * 8 + [
                ctypes.c_int, _dp, ctypes.c_int]
            lib.ss_oracle_update.restype = ctypes.c_int
            lib.ss_oracle_conv_silu.argtypes = [_i64, _i64, _i64, _i64] + [_dp] * 6 + [ctypes.c_int]
            lib.ss_oracle_conv_silu.restype = ctypes.c_int
            lib.ss_oracle_gated_scan.argtypes = [_i64, _i64, _i64, _i64] + [_dp] * 7 + [ctypes.c_int]
            lib.ss_oracle_gated_scan.restype = ctypes.c_int
            lib.ss_oracle_segment.argtypes = [_i64, _i64, _i64, _i64] + [_dp] * 5 + [
                _u8p, ctypes.c_int, _dp, _dp, ctypes.c_int]
            lib.ss_oracle_segment.restype = ctypes.c_int
            lib.ss_oracle_num_threads.argtypes = []
            lib.ss_oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses by default (the host's cores)."""
    return int(_load().ss_oracle_num_threads())


def _f64(a):
    """Exact widening of a numpy array or torch tensor to contiguous float64."""
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor: widen with torch, then view as numpy
        a = a.detach().to("cpu").double().contiguous().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _u8(a):
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").contiguous().numpy()
    return np.ascontiguousarray(np.asarray(a).astype(np.uint8))


def _ptr(a, kind=_dp):
    return None if a is None else a.ctypes.data_as(kind)


def _check(status, what):
    if status != 0:
        raise RuntimeError(f"{what} failed with status {status}")


def _scan_args(x, dt, A, B, C, D, z, dt_bias, reset, h0):
    x, dt, A, B, C = (_f64(v) for v in (x, dt, A, B, C))
    D, z, dt_bias, h0 = (_f64(v) for v in (D, z, dt_bias, h0))
    reset = _u8(reset)
    if x.ndim != 3:
        raise ValueError("x must be [batch, channels, seq]")
    bt, ch, L = x.shape
    n = A.shape[1]
    if dt.shape != x.shape or A.shape != (ch, n) or B.shape != (bt, n, L) or C.shape != (bt, n, L):
        raise ValueError("inconsistent shapes")
    if z is not None and z.shape != x.shape:
        raise ValueError("z must match x")
    if D is not None and D.shape != (ch,):
        raise ValueError("D must be [channels]")
    if dt_bias is not None and dt_bias.shape != (ch,):
        raise ValueError("dt_bias must be [channels]")
    if reset is not None and reset.shape != (bt, L):
        raise ValueError("reset must be [batch, seq]")
    if h0 is not None and h0.shape != (bt, ch, n):
        raise ValueError("h0 must be [batch, channels, state_dim]")
    return (bt, ch, n, L), (x, dt, A, B, C, D, z, dt_bias, reset, h0)


def scan(x, dt, A, B, C, D=None, z=None, dt_bias=None, reset=None, h0=None, *,
         dt_softplus=True, return_states=False, return_betas=False, nthreads=None):
    """Token-loop oracle.  Returns dict(y [b,c,L], h_last [b,c,n], h_all [b,c,L,n] or None,
    betas [b,c,L] (the step size of every token) or None)."""
    (bt, ch, n, L), (x, dt, A, B, C, D, z, dt_bias, reset, h0) = _scan_args(
        x, dt, A, B, C, D, z, dt_bias, reset, h0)
    y = np.empty((bt, ch, L))
    h_last = np.empty((bt, ch, n))
    h_all = np.empty((bt, ch, L, n)) if return_states else None
    betas = np.empty((bt, ch, L)) if return_betas else None
    lib = _load()
    st = lib.ss_oracle_scan(bt, ch, n, L, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                            _ptr(D), _ptr(z), _ptr(dt_bias), _ptr(reset, _u8p), _ptr(h0),
                            int(bool(dt_softplus)), _ptr(y), _ptr(h_last), _ptr(h_all), _ptr(betas),
                            int(nthreads or num_threads()))
    _check(st, "ss_oracle_scan")
    return {"y": y, "h_last": h_last, "h_all": h_all, "betas": betas}


def tree_scan(x, dt, A, B, C, D=None, z=None, dt_bias=None, reset=None, h0=None, *,
              dt_softplus=True, nthreads=None):
    """Associative-scan ordering of the same recurrence.  Returns dict(y, h_last)."""
    (bt, ch, n, L), (x, dt, A, B, C, D, z, dt_bias, reset, h0) = _scan_args(
        x, dt, A, B, C, D, z, dt_bias, reset, h0)
    y = np.empty((bt, ch, L))
    h_last = np.empty((bt, ch, n))
    lib = _load()
    st = lib.ss_oracle_tree_scan(bt, ch, n, L, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                                 _ptr(D), _ptr(z), _ptr(dt_bias), _ptr(reset, _u8p), _ptr(h0),
                                 int(bool(dt_softplus)), _ptr(y), _ptr(h_last),
                                 int(nthreads or num_threads()))
    _check(st, "ss_oracle_tree_scan")
    return {"y": y, "h_last": h_last}


def update(state, x, dt, A, B, C, D=None, z=None, dt_bias=None, *, dt_softplus=True,
           nthreads=None):
    """Decode-step oracle on a COPY of ``state``.  Returns dict(y [b,c], state [b,c,n])."""
    st_arr = _f64(state).copy()
    x, dt, A, B, C = (_f64(v) for v in (x, dt, A, B, C))
    D, z, dt_bias = (_f64(v) for v in (D, z, dt_bias))
    bt, ch, n = st_arr.shape
    if x.shape != (bt, ch) or dt.shape != (bt, ch) or A.shape != (ch, n):
        raise ValueError("inconsistent shapes")
    if B.shape != (bt, n) or C.shape != (bt, n):
        raise ValueError("B, C must be [batch, state_dim]")
    if z is not None and z.shape != (bt, ch):
        raise ValueError("z must be [batch, channels]")
    y = np.empty((bt, ch))
    lib = _load()
    rc = lib.ss_oracle_update(bt, ch, n, _ptr(st_arr), _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                              _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
                              int(bool(dt_softplus)), _ptr(y), int(nthreads or num_threads()))
    _check(rc, "ss_oracle_update")
    return {"y": y, "state": st_arr}


def conv_silu(u, w, cb=None, state=None, *, nthreads=None):
    """Causal depthwise conv + SiLU oracle (TransformerLens ssm_mixer: the scan's x is
    SiLU of the conv1d output).  u [b, c, L]; w [c, K]; cb [c] or None; state [b, c, K-1]
    (the inputs before u, oldest first) or None.  Returns dict(x [b, c, L],
    state [b, c, K-1] = the last K-1 inputs of state ++ u)."""
    u, w, cb, state = _f64(u), _f64(w), _f64(cb), _f64(state)
    bt, ch, L = u.shape
    K = w.shape[1]
    if w.shape != (ch, K) or (cb is not None and cb.shape != (ch,)):
        raise ValueError("inconsistent conv shapes")
    if state is not None and state.shape != (bt, ch, K - 1):
        raise ValueError("state must be [b, c, K-1]")
    x = np.empty((bt, ch, L))
    so = np.empty((bt, ch, K - 1))
    rc = _load().ss_oracle_conv_silu(bt, ch, L, K, _ptr(u), _ptr(w), _ptr(cb), _ptr(state), _ptr(x), _ptr(so),
                                     int(nthreads or num_threads()))
    _check(rc, "ss_oracle_conv_silu")
    return {"x": x, "state": so}


def gated_scan(q, k, v, gamma, h0=None, *, nthreads=None):
    """Gated state scan oracle ("Mamba 2 Gated State Scan": S_t = gamma_t S_{t-1} +
    k_t v_t^T, y_t = q_t^T S_t).  q, k [B, S, Dk]; v [B, S, Dv]; gamma [B, S];
    h0 [B, Dk, Dv] or None.  Returns dict(outputs [B, S, Dv], final_state [B, Dk, Dv])."""
    q, k, v, gamma = (_f64(a) for a in (q, k, v, gamma))
    h0 = _f64(h0)
    bt, sl, dk = q.shape
    dv = v.shape[-1]
    if k.shape != (bt, sl, dk) or v.shape != (bt, sl, dv) or gamma.shape != (bt, sl):
        raise ValueError("inconsistent shapes")
    if h0 is not None and h0.shape != (bt, dk, dv):
        raise ValueError("h0 must be [B, Dk, Dv]")
    y = np.empty((bt, sl, dv))
    fs = np.empty((bt, dk, dv))
    rc = _load().ss_oracle_gated_scan(bt, sl, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(h0),
                                      _ptr(y), _ptr(fs), int(nthreads or num_threads()))
    _check(rc, "ss_oracle_gated_scan")
    return {"outputs": y, "final_state": fs}


def segment(x, dt, A, B, dt_bias=None, reset=None, *, dt_softplus=True, nthreads=None):
    """Composite of one segment ("s6_reset", Associative Boundary Resetting: the
    segment's maps folded with the resettable operator).  Returns dict(decay
    [b,c,n] = the product of the segment's decays, 0 when it holds a reset;
    state [b,c,n] = its end state entered from zero)."""
    x, dt, A, B, dt_bias = (_f64(v) for v in (x, dt, A, B, dt_bias))
    reset = _u8(reset)
    bt, ch, L = x.shape
    n = A.shape[1]
    if dt.shape != x.shape or A.shape != (ch, n) or B.shape != (bt, n, L):
        raise ValueError("inconsistent shapes")
    if dt_bias is not None and dt_bias.shape != (ch,):
        raise ValueError("dt_bias must be [channels]")
    if reset is not None and reset.shape != (bt, L):
        raise ValueError("reset must be [batch, seq]")
    decay = np.empty((bt, ch, n))
    state = np.empty((bt, ch, n))
    rc = _load().ss_oracle_segment(bt, ch, n, L, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(dt_bias),
                                   _ptr(reset, _u8p), int(bool(dt_softplus)), _ptr(decay), _ptr(state),
                                   int(nthreads or num_threads()))
    _check(rc, "ss_oracle_segment")
    return {"decay": decay, "state": state}


def join_segments(decays, states, h0=None):
    """Apply the composites of consecutive segments in order, starting from h0 (zeros
    when None): carry_0 = h0, carry_{s+1} = decay_s * carry_s + state_s.  Returns
    (carries, final): carries[s] is the state entering segment s, final the state
    after the last one."""
    carry = np.zeros_like(_f64(states[0])) if h0 is None else _f64(h0).copy()
    carries = []
    for d, st in zip(decays, states):
        carries.append(carry.copy())
        carry = _f64(d) * carry + _f64(st)
    return carries, carry


def scan_rows(inputs: dict, rows, *, dt_softplus=True, nthreads=1):
    """Oracle on a subset of (b, c) rows of a large problem, one row at a time.

    ``inputs`` holds the full tensors (x, dt, A, B, C and the optional ones);
    each row is cut out and run as a batch-1, channel-1 problem.  Returns
    (y [len(rows), L], h_last [len(rows), n]).
    """
    ys, hs = [], []
    for (b, c) in rows:
        sub = {
            "x": inputs["x"][b:b + 1, c:c + 1], "dt": inputs["dt"][b:b + 1, c:c + 1],
            "A": inputs["A"][c:c + 1], "B": inputs["B"][b:b + 1], "C": inputs["C"][b:b + 1],
        }
        for k in ("D", "dt_bias"):
            if inputs.get(k) is not None:
                sub[k] = inputs[k][c:c + 1]
        if inputs.get("z") is not None:
            sub["z"] = inputs["z"][b:b + 1, c:c + 1]
        if inputs.get("reset") is not None:
            sub["reset"] = inputs["reset"][b:b + 1]
        if inputs.get("h0") is not None:
            sub["h0"] = inputs["h0"][b:b + 1, c:c + 1]
        out = scan(**sub, dt_softplus=dt_softplus, nthreads=nthreads)
        ys.append(out["y"][0, 0])
        hs.append(out["h_last"][0, 0])
    return np.stack(ys), np.stack(hs)
