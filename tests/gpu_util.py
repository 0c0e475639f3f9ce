"""Helpers shared by the GPU test files: move seeded inputs to the device, call the
C ABI through the binding, and compare with the oracle elementwise."""
import contextlib

import numpy as np
import torch

from selective_state_space_18_b200 import ssscan

# max |out - ref| <= tol * (1 + |ref|), elementwise
TOL = {torch.float32: 1e-4, torch.bfloat16: 1e-2}

SCAN_KEYS = ("x", "dt", "A", "B", "C", "D", "z", "dt_bias", "reset", "h0")
UPDATE_KEYS = ("state", "x", "dt", "A", "B", "C", "D", "z", "dt_bias")


def dev(inp, keys):
    return {k: (None if inp.get(k) is None else inp[k].cuda()) for k in keys}


def gpu_scan(inp, **kw):
    y, h = ssscan.ss_scan_fwd(**dev(inp, SCAN_KEYS), **kw)
    torch.cuda.synchronize()
    return y.cpu(), (None if h is None else h.cpu())


def gpu_update(inp, **kw):
    d = dev(inp, UPDATE_KEYS)
    y = ssscan.ss_state_update(**d, **kw)
    torch.cuda.synchronize()
    return y.cpu(), d["state"].cpu()


def rel_err(out, ref):
    out = out.double().numpy() if hasattr(out, "numpy") else np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    assert out.shape == ref.shape, (out.shape, ref.shape)
    assert np.all(np.isfinite(out)), "non-finite output"
    return float(np.max(np.abs(out - ref) / (1.0 + np.abs(ref)))) if out.size else 0.0


def assert_close(out, ref, tol, what=""):
    e = rel_err(out, ref)
    assert e <= tol, f"{what}: max |d|/(1+|ref|) = {e:.3e} > {tol:.0e}"
    return e


@contextlib.contextmanager
def schedule(two_level=None, layout=None):
    """Pin the scan's schedule for the block: two_level 0 (automatic), 1 (never: the
    single-pass schedule, chained segments or one CTA per group) or 2 (whenever the
    sequence allows); layout 2 or 4 state rows per scan lane (0: automatic)."""
    if two_level is not None:
        ssscan.ss_debug_set_scan_two_level(two_level)
    if layout is not None:
        ssscan.ss_debug_set_scan_layout(layout)
    try:
        yield
    finally:
        ssscan.ss_debug_set_scan_two_level(0)
        ssscan.ss_debug_set_scan_layout(0)
