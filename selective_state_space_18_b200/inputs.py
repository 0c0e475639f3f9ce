"""Seeded synthetic inputs for the selective scan and the decode update.

This module draws random numbers and nothing else: it holds none of the scan's
arithmetic, so both the CUDA path and the float64 oracle can be fed from it.
All tensors are produced on the CPU with ``torch.Generator`` in float32/float64
and then rounded once to the requested storage dtype; the oracle widens the
rounded values, so both sides see identical numbers.

Distributions (the selective-scan workloads of the benchmark suite):
  x, z, B, C, dt_raw ~ N(0, 1)
  dt_bias = softplus^{-1}(u) = log(expm1(u)), u log-uniform in [1e-3, 1e-1]
  A[c, n] = -(n + 1)                      (S4D-real initialisation)
      optionally times (1 + clip(0.1 * N(0,1), -0.5, 0.5)), one draw per (c, n)
  D ~ N(0, 1)
  reset mask: per batch row, document lengths ~ Geometric(1/mean_doc) on
      {1, 2, ...}, laid out from t = 0; the flag marks each document's first token.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    """A named workload: shape, storage dtype and which optional inputs are on."""
    name: str
    batch: int
    channels: int
    state_dim: int
    seq: int                 # 1 and decode=True for the single-token update
    dtype: str               # "f32" or "bf16" for x, dt, z, B, C, y
    seed: int
    z: bool = True
    dt_bias: bool = True
    D: bool = True
    a_perturb: bool = False
    reset_mean_doc: int = 0  # 0: no reset mask
    decode: bool = False
    notes: str = field(default="", compare=False)

    @property
    def elems(self) -> int:
        """Scan elements batch * seq * channels * state_dim."""
        return self.batch * self.seq * self.channels * self.state_dim


# The five workloads of the benchmark suite, seeds 20260 + index.
WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_fp32", 1, 8, 4, 64, "f32", 20260,
                 notes="tiny prompt scan, fp32, h0 = 0, no resets"),
        Workload("mamba130m_layer", 8, 1536, 16, 2048, "bf16", 20261,
                 notes="Mamba-130M-layer-shaped prompt scan, bf16 in/out, fp32 state"),
        Workload("mamba2p8b_layer_long", 1, 5120, 16, 16384, "bf16", 20262, a_perturb=True,
                 notes="Mamba-2.8B-layer-shaped long prompt scan, bf16, fp32 state"),
        Workload("packed_resets", 2, 2048, 16, 32768, "bf16", 20263, reset_mean_doc=512,
                 notes="packed documents with enforced boundary resets, bf16"),
        Workload("decode_2p8b", 256, 5120, 16, 1, "bf16", 20264, a_perturb=True, decode=True,
                 notes="single-token decode state update, fp32 state in place"),
    ]
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _randn(g, shape, dtype):
    return torch.randn(shape, generator=g, dtype=torch.float32).to(DTYPES[dtype])


def _dt_bias(g, channels):
    lo, hi = math.log(1e-3), math.log(1e-1)
    u = torch.exp(lo + (hi - lo) * torch.rand(channels, generator=g, dtype=torch.float64))
    return torch.log(torch.expm1(u)).to(torch.float32)


def _A(g, channels, state_dim, perturb):
    base = -torch.arange(1, state_dim + 1, dtype=torch.float64).expand(channels, state_dim)
    if perturb:
        eps = (0.1 * torch.randn(channels, state_dim, generator=g, dtype=torch.float64)).clamp(-0.5, 0.5)
        base = base * (1.0 + eps)
    return base.to(torch.float32).contiguous()


def reset_mask(g, batch, seq, mean_doc):
    """Document-start flags [batch, seq] (uint8) with geometric document lengths."""
    p = 1.0 / float(mean_doc)
    mask = torch.zeros(batch, seq, dtype=torch.uint8)
    for b in range(batch):
        t = 0
        while t < seq:
            mask[b, t] = 1
            u = float(torch.rand((), generator=g, dtype=torch.float64))
            u = max(u, 1e-300)
            length = 1 + int(math.floor(math.log(u) / math.log1p(-p)))
            t += length
    return mask


def make_scan_inputs(batch, channels, state_dim, seq, dtype="bf16", *, seed=0, z=True,
                     dt_bias=True, D=True, a_perturb=False, reset_mean_doc=0, h0=False):
    """Seeded prompt-scan inputs as CPU tensors (x, dt, z, B, C in ``dtype``)."""
    g = _gen(seed)
    out = {
        "x": _randn(g, (batch, channels, seq), dtype),
        "dt": _randn(g, (batch, channels, seq), dtype),
        "z": _randn(g, (batch, channels, seq), dtype) if z else None,
        "B": _randn(g, (batch, state_dim, seq), dtype),
        "C": _randn(g, (batch, state_dim, seq), dtype),
        "D": torch.randn(channels, generator=g, dtype=torch.float32) if D else None,
        "dt_bias": _dt_bias(g, channels) if dt_bias else None,
    }
    out["A"] = _A(g, channels, state_dim, a_perturb)
    out["h0"] = torch.randn(batch, channels, state_dim, generator=g, dtype=torch.float32) if h0 else None
    out["reset"] = reset_mask(g, batch, seq, reset_mean_doc) if reset_mean_doc else None
    return out


def make_update_inputs(batch, channels, state_dim, dtype="bf16", *, seed=0, z=True,
                       dt_bias=True, D=True, a_perturb=False):
    """Seeded decode-step inputs: state [b,c,n] fp32, x/dt/z [b,c], B/C [b,n] in ``dtype``."""
    g = _gen(seed)
    out = {
        "state": torch.randn(batch, channels, state_dim, generator=g, dtype=torch.float32),
        "x": _randn(g, (batch, channels), dtype),
        "dt": _randn(g, (batch, channels), dtype),
        "z": _randn(g, (batch, channels), dtype) if z else None,
        "B": _randn(g, (batch, state_dim), dtype),
        "C": _randn(g, (batch, state_dim), dtype),
        "D": torch.randn(channels, generator=g, dtype=torch.float32) if D else None,
        "dt_bias": _dt_bias(g, channels) if dt_bias else None,
    }
    out["A"] = _A(g, channels, state_dim, a_perturb)
    return out


def make_gated_inputs(batch, seq, dk, dv, dtype="bf16", *, seed=0, h0=False):
    """Seeded gated-state-scan inputs: q, k [B, S, Dk] scaled by 1/sqrt(Dk), v [B, S, Dv]
    in ``dtype``; gamma [B, S] fp32 in [0, 1] -- mostly in [0.5, 1), with about 1% exact
    zeros (the state is discarded) and 1% exact ones (kept whole)."""
    g = _gen(seed)
    sc = 1.0 / math.sqrt(dk)
    q = (torch.randn(batch, seq, dk, generator=g) * sc).to(DTYPES[dtype])
    k = (torch.randn(batch, seq, dk, generator=g) * sc).to(DTYPES[dtype])
    v = _randn(g, (batch, seq, dv), dtype)
    gamma = 0.5 + 0.5 * torch.rand(batch, seq, generator=g)
    u = torch.rand(batch, seq, generator=g)
    gamma = torch.where(u < 0.01, torch.zeros_like(gamma), torch.where(u > 0.99, torch.ones_like(gamma), gamma))
    out = {"q": q, "k": k, "v": v, "gamma": gamma.float().contiguous()}
    out["h0"] = torch.randn(batch, dk, dv, generator=g) if h0 else None
    return out


def make_workload(name_or_workload, **overrides):
    """Inputs for a named workload (prompt scan or decode update)."""
    w = WORKLOADS[name_or_workload] if isinstance(name_or_workload, str) else name_or_workload
    kw = dict(seed=w.seed, z=w.z, dt_bias=w.dt_bias, D=w.D, a_perturb=w.a_perturb)
    kw.update(overrides)
    if w.decode:
        return make_update_inputs(w.batch, w.channels, w.state_dim, w.dtype, **kw)
    kw.setdefault("reset_mean_doc", w.reset_mean_doc)
    return make_scan_inputs(w.batch, w.channels, w.state_dim, w.seq, w.dtype, **kw)
