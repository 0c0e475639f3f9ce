"""Prompt scan of one long sequence cut into contiguous segments, one per rank of a
process group (one process per GPU).

The scan's recurrence composes associatively ("s6_reset" blog draft, Associative
Boundary Resetting: the property that makes long sequences scannable in parallel).
A segment acts on the state that enters it as h -> decay * h + state, so a rank
needs from the segments before its own only their composites (two float32 values
per state element), never their tokens:

  1. every rank scans its own segment: rank 0 from the caller's initial state (its
     result is final), every other rank from zero, and those also compute their
     segment's decay (``ss_segment_decay``);
  2. the composites (decay, end state) of all ranks are all-gathered: the one
     exchange step, batch * channels * state_dim * 8 bytes per rank;
  3. every rank but 0 folds the composites before its segment into the state that
     enters it (``ss_join_segments``) and rescans its segment from that state.

Rank 0 scans once and the others twice, so ``shard_bounds`` gives rank 0 twice the
tokens of each other rank.  Every step runs in the library's CUDA kernels; the
all-gather is NCCL's (torch.distributed).  ``local_pass`` and ``finish_pass`` are
the halves on either side of the exchange, usable without a process group (for
example to run several segments in one process).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import ssscan


def shard_bounds(seq: int, world: int, *, multiple: int = 8):
    """Token ranges [(start, stop), ...] of the ranks: rank 0 takes two shares of
    seq / (world + 1), every other rank one; inner cuts fall on multiples of
    `multiple` (16-byte rows for the vector path)."""
    if world < 1 or seq < 1:
        raise ValueError("need world >= 1 and seq >= 1")
    cuts = [0]
    for k in range(world - 1):
        c = (seq * (k + 2) // (world + 1)) // multiple * multiple
        if c <= cuts[-1]:
            raise ValueError(f"seq={seq} is too short for {world} segments of {multiple}-token multiples")
        cuts.append(c)
    if seq <= cuts[-1]:
        raise ValueError(f"seq={seq} is too short for {world} segments")
    cuts.append(seq)
    return list(zip(cuts[:-1], cuts[1:]))


class CudaSteps:
    """The three steps through the library's kernels (ctypes binding)."""

    state_dtype = torch.float32

    @staticmethod
    def scan(inp, h0, y, h_last):
        ssscan.ss_scan_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp.get("D"), inp.get("z"),
                           inp.get("dt_bias"), inp.get("reset"), h0, dt_softplus=inp.get("dt_softplus", True),
                           y=y, h_last=h_last)

    @staticmethod
    def segment_decay(inp, out):
        ssscan.ss_segment_decay(inp["dt"], inp["A"], inp.get("dt_bias"), inp.get("reset"),
                                dt_softplus=inp.get("dt_softplus", True), out=out)

    @staticmethod
    def join(composites, rank, want_final):
        return ssscan.ss_join_segments(composites, rank, want_final=want_final)


def _inputs(x, dt, A, B, C, D, z, dt_bias, reset, dt_softplus):
    return {"x": x, "dt": dt, "A": A, "B": B, "C": C, "D": D, "z": z, "dt_bias": dt_bias, "reset": reset,
            "dt_softplus": dt_softplus}


def local_pass(inp: dict, rank: int, h0=None, steps=CudaSteps):
    """Step 1 on one segment.  Returns (y, composite [2, batch, channels, state_dim]):
    y is final on rank 0 and provisional elsewhere; composite = (decay, end state),
    rank 0's decay being zeros (it is never read)."""
    x, A = inp["x"], inp["A"]
    bt, ch, _ = x.shape
    n = A.shape[-1]
    y = torch.empty_like(x)
    comp = torch.empty(2, bt, ch, n, device=x.device, dtype=steps.state_dtype)
    if rank == 0:
        comp[0].zero_()
        steps.scan(inp, h0, y, comp[1])
    else:
        steps.scan(inp, None, y, comp[1])
        steps.segment_decay(inp, comp[0])
    return y, comp


def finish_pass(inp: dict, rank: int, composites, y, *, want_final=False, steps=CudaSteps):
    """Step 3 on one segment, given the gathered composites [segments, 2, batch,
    channels, state_dim] in segment order.  Returns (y, h_last, final_state): this
    segment's outputs and end state, and the state after the whole sequence (None
    unless want_final)."""
    if rank == 0:
        final = steps.join(composites, None, True)[1] if want_final else None
        return y, composites[0, 1].clone(), final
    carry, final = steps.join(composites, rank, want_final)
    h_last = torch.empty_like(carry)
    steps.scan(inp, carry, y, h_last)
    return y, h_last, final


def seq_sharded_scan(x, dt, A, B, C, D=None, z=None, dt_bias=None, reset=None, h0=None, *,
                     dt_softplus=True, group=None, return_final_state=False, steps=CudaSteps):
    """Prompt scan of this rank's segment of a sequence split over `group`'s ranks in
    rank order.  x, dt, z: [batch, channels, seg_len] and B, C: [batch, state_dim,
    seg_len] are this rank's tokens; reset [batch, seg_len] its slice of the mask;
    A, D, dt_bias are the same on every rank; h0 (the state before the sequence's
    first token) is read on rank 0 only.  Returns dict(y, h_last = the state after
    this segment, final_state = the state after the whole sequence, on every rank,
    when return_final_state).  Every rank must call it (it holds one collective), with
    the same batch, channels and state_dim and the same dtype; only the segment length
    may differ between ranks.  `steps` carries out the scan, decay and join: the
    library's kernels (CudaSteps); the tests put float64 stand-ins there to check the
    exchange on CPU ranks."""
    if dist.is_available() and dist.is_initialized():
        world, rank = dist.get_world_size(group), dist.get_rank(group)
    else:
        world, rank = 1, 0
    inp = _inputs(x, dt, A, B, C, D, z, dt_bias, reset, dt_softplus)
    y, comp = local_pass(inp, rank, h0 if rank == 0 else None, steps)
    if world > 1:
        flat = torch.empty((world * 2,) + tuple(comp.shape[1:]), device=comp.device, dtype=comp.dtype)
        dist.all_gather_into_tensor(flat, comp, group=group)
        gathered = flat.view((world,) + tuple(comp.shape))
    else:
        gathered = comp.unsqueeze(0)
    y, h_last, final = finish_pass(inp, rank, gathered, y, want_final=return_final_state, steps=steps)
    out = {"y": y, "h_last": h_last}
    if return_final_state:
        out["final_state"] = final
    return out
