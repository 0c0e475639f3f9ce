"""Sequence cut into segments over ranks (selective_state_space_18_b200.seqshard).

CPU part: the exchange and ordering logic of ``seq_sharded_scan`` on gloo ranks (two
and three processes), with the three steps carried out by the float64 oracle, so
the test checks who scans from which state, the all-gather's layout and order, and
the join, against the oracle's scan of the whole sequence.

GPU part: the library's kernels.  ss_segment_decay and ss_join_segments against the
oracle's segment composite and join; and the whole method with several segments run
in one process on one GPU (``local_pass`` on every segment, the composites stacked
in segment order as the all-gather would, then ``finish_pass``), against the
oracle's scan of the whole sequence.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import oracle
from selective_state_space_18_b200 import seqshard
from selective_state_space_18_b200.inputs import make_scan_inputs


# ---- host logic ---------------------------------------------------------------------

@pytest.mark.parametrize("seq,world", [(16384, 2), (16384, 8), (1000, 3), (64, 4), (17, 1)])
def test_shard_bounds_cover_the_sequence(seq, world):
    b = seqshard.shard_bounds(seq, world)
    assert len(b) == world
    assert b[0][0] == 0 and b[-1][1] == seq
    for (s0, e0), (s1, _) in zip(b[:-1], b[1:]):
        assert e0 == s1 and e0 % 8 == 0
    assert all(e > s for s, e in b)
    if world > 1 and seq >= 64 * world:
        share = seq / (world + 1)
        assert abs((b[0][1] - b[0][0]) - 2 * share) <= 8      # rank 0 scans once: two shares
        for s, e in b[1:-1]:
            assert abs((e - s) - share) <= 16


def test_shard_bounds_refuse_too_short():
    with pytest.raises(ValueError):
        seqshard.shard_bounds(20, 4)


class OracleSteps:
    """The three steps by the float64 oracle, on CPU tensors."""

    state_dtype = torch.float64

    @staticmethod
    def scan(inp, h0, y, h_last):
        out = oracle.scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp.get("D"), inp.get("z"),
                          inp.get("dt_bias"), inp.get("reset"), h0, dt_softplus=inp["dt_softplus"], nthreads=1)
        y.copy_(torch.from_numpy(out["y"]))
        h_last.copy_(torch.from_numpy(out["h_last"]))

    @staticmethod
    def segment_decay(inp, out):
        comp = oracle.segment(inp["x"], inp["dt"], inp["A"], inp["B"], inp.get("dt_bias"), inp.get("reset"),
                              dt_softplus=inp["dt_softplus"], nthreads=1)
        out.copy_(torch.from_numpy(comp["decay"]))

    @staticmethod
    def join(comps, rank, want_final):
        carries, final = oracle.join_segments(comps[:, 0].numpy(), comps[:, 1].numpy())
        return (None if rank is None else torch.from_numpy(carries[rank]),
                torch.from_numpy(final) if want_final else None)


def _problem(L=480, variant="h0"):
    """variant "h0": initial state, softplus, resets (two of them on segment starts);
    "plain": no initial state, no softplus (positive raw steps, no bias), no resets."""
    if variant == "h0":
        inp = make_scan_inputs(2, 8, 4, L, "f32", seed=31, reset_mean_doc=90, h0=True)
    else:
        inp = make_scan_inputs(2, 8, 4, L, "f32", seed=32, dt_bias=False)
        inp["dt"] = inp["dt"].abs() * 0.05
    out = {k: (v.double() if torch.is_tensor(v) and v.is_floating_point() else v) for k, v in inp.items()}
    if variant == "h0":
        out["reset"][1, 240] = 1     # resets on the first token of a segment: the cut at 240 (three
        out["reset"][0, 320] = 1     # ranks) and at 320 (two ranks)
    return out


def _slice(p, a, b):
    q = {}
    for k, v in p.items():
        if v is None:
            q[k] = None
        elif k in ("x", "dt", "z", "B", "C"):
            q[k] = v[..., a:b].contiguous()
        elif k == "reset":
            q[k] = v[:, a:b].contiguous()
        else:
            q[k] = v
    return q


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_worker(rank, world, port, variant, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        p = _problem(variant=variant)
        a, b = seqshard.shard_bounds(p["x"].shape[-1], world)[rank]
        q = _slice(p, a, b)
        res = seqshard.seq_sharded_scan(q["x"], q["dt"], q["A"], q["B"], q["C"], q["D"], q["z"], q["dt_bias"],
                                        q["reset"], q["h0"] if rank == 0 else None, return_final_state=True,
                                        dt_softplus=variant == "h0", steps=OracleSteps)
        out[rank] = (a, b, res["y"].numpy(), res["h_last"].numpy(), res["final_state"].numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,variant", [(2, "h0"), (3, "h0"), (4, "plain")])
def test_gloo_ranks_join_to_the_whole_scan(world, variant):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_rank_worker, args=(world, _free_port(), variant, out), nprocs=world, join=True)
    p = _problem(variant=variant)
    whole = oracle.scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["z"], p["dt_bias"], p["reset"],
                        p["h0"], dt_softplus=variant == "h0", return_states=True)
    y = np.concatenate([out[r][2] for r in range(world)], axis=-1)
    scale = 1.0 + np.abs(whole["y"]).max()
    assert np.abs(y - whole["y"]).max() <= 1e-12 * scale
    for r in range(world):
        a, b, _, h_last, final = out[r]
        ref = whole["h_all"][:, :, b - 1]
        assert np.abs(h_last - ref).max() <= 1e-12 * (1.0 + np.abs(ref).max())
        assert np.abs(final - whole["h_last"]).max() <= 1e-12 * (1.0 + np.abs(whole["h_last"]).max())


def test_single_process_is_a_plain_scan():
    """Without a process group the call is one segment: the oracle's scan itself."""
    p = _problem()
    res = seqshard.seq_sharded_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["z"], p["dt_bias"],
                                    p["reset"], p["h0"], return_final_state=True, steps=OracleSteps)
    whole = oracle.scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["z"], p["dt_bias"], p["reset"], p["h0"])
    assert np.array_equal(res["y"].numpy(), whole["y"])
    assert np.array_equal(res["final_state"].numpy(), whole["h_last"])


# ---- GPU: the library's kernels --------------------------------------------------------

def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    return torch.device("cuda", 0)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n,L", [(16, 4096), (16, 1001), (4, 64), (8, 2000)])
@pytest.mark.parametrize("resets", [False, True])
def test_segment_decay_matches_oracle(dtype, n, L, resets):
    d = _cuda()
    inp = make_scan_inputs(2, 40, n, L, dtype, seed=L + n, reset_mean_doc=3000 if resets else 0)
    if resets:
        inp["reset"][1] = 0          # one batch row without a reset, one (probably) with
        inp["reset"][0, L // 2] = 1
    inp["A"] = inp["A"] * (64.0 / L)   # keep A * sum(dt) in the range where the decay is not ~0
    ref = oracle.segment(inp["x"], inp["dt"], inp["A"], inp["B"], inp["dt_bias"], inp["reset"])["decay"]
    out = seqshard.ssscan.ss_segment_decay(inp["dt"].to(d), inp["A"].to(d), inp["dt_bias"].to(d),
                                           None if inp["reset"] is None else inp["reset"].to(d))
    got = out.cpu().double().numpy()
    assert np.all(np.isfinite(got))
    assert np.all(got[ref == 0.0] == 0.0)
    assert np.median(ref[1]) > 1e-6          # batch row 1 has no reset: its decays are far from 0
    if resets:
        assert np.all(got[0] == 0.0)     # the row with a reset discards the entering state
    err = np.abs(got - ref) - 1e-4 * np.abs(ref)
    assert err.max() <= 1e-7, err.max()


@pytest.mark.gpu
def test_segment_decay_without_softplus():
    d = _cuda()
    inp = make_scan_inputs(1, 24, 16, 513, "f32", seed=2)
    inp["dt"] = inp["dt"].abs() * 0.01       # positive steps, no bias: decays in (0, 1]
    inp["A"] = inp["A"] * 0.05
    ref = oracle.segment(inp["x"], inp["dt"], inp["A"], inp["B"], None, dt_softplus=False)["decay"]
    got = seqshard.ssscan.ss_segment_decay(inp["dt"].to(d), inp["A"].to(d), None,
                                           dt_softplus=False).cpu().double().numpy()
    assert np.all(np.isfinite(got)) and np.median(ref) > 1e-6
    assert (np.abs(got - ref) - 1e-4 * np.abs(ref)).max() <= 1e-7


@pytest.mark.gpu
@pytest.mark.parametrize("segments", [1, 2, 5])
def test_join_matches_oracle(segments):
    d = _cuda()
    g = torch.Generator().manual_seed(segments)
    comp = torch.empty(segments, 2, 3, 33, 16)
    comp[:, 0] = torch.rand(segments, 3, 33, 16, generator=g)
    comp[:, 1] = torch.randn(segments, 3, 33, 16, generator=g)
    comp[0, 0] = float("nan")        # segment 0's decay is never read
    ref_decay = comp[:, 0].double().numpy().copy()
    ref_decay[0] = 0.0               # the oracle's join starts from zeros, so any finite value does
    carries, final = oracle.join_segments(ref_decay, comp[:, 1].double().numpy())
    for rank in range(1, segments):
        carry, fin = seqshard.ssscan.ss_join_segments(comp.to(d), rank)
        e = np.abs(carry.cpu().double().numpy() - carries[rank]) / (1 + np.abs(carries[rank]))
        assert e.max() <= 1e-5
        assert np.abs(fin.cpu().double().numpy() - final).max() <= 1e-5 * (1 + np.abs(final).max())
    _, fin = seqshard.ssscan.ss_join_segments(comp.to(d))
    assert np.abs(fin.cpu().double().numpy() - final).max() <= 1e-5 * (1 + np.abs(final).max())


def _emulate(inp_dev, world, want_final=True):
    """Every segment in one process: local_pass on each, the composites stacked in
    segment order (what the all-gather delivers), then finish_pass on each."""
    L = inp_dev["x"].shape[-1]
    bounds = seqshard.shard_bounds(L, world)
    parts, ys, comps = [], [], []
    for r, (a, b) in enumerate(bounds):
        q = _slice(inp_dev, a, b)
        q["dt_softplus"] = True
        parts.append(q)
        y, comp = seqshard.local_pass(q, r, inp_dev.get("h0") if r == 0 else None)
        ys.append(y)
        comps.append(comp)
    gathered = torch.stack(comps)
    res = [seqshard.finish_pass(q, r, gathered, y, want_final=want_final)
           for r, (q, y) in enumerate(zip(parts, ys))]
    torch.cuda.synchronize()
    return bounds, res


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("world", [2, 3, 4])
def test_emulated_ranks_match_the_whole_scan(dtype, world):
    d = _cuda()
    L = 6003
    inp = make_scan_inputs(2, 64, 16, L, dtype, seed=40 + world, reset_mean_doc=1500, h0=True)
    bounds = seqshard.shard_bounds(L, world)
    inp["reset"][1, bounds[1][0]] = 1            # a reset on the first token of segment 1
    inp["reset"][0, bounds[1][0]] = 0
    keys = ("x", "dt", "A", "B", "C", "D", "z", "dt_bias", "reset", "h0")
    inp_dev = {k: inp[k].to(d) for k in keys}
    _, res = _emulate(inp_dev, world)
    whole = oracle.scan(*(inp[k] for k in keys))
    tol = {"bf16": 1e-2, "f32": 1e-4}[dtype]
    y = torch.cat([r[0] for r in res], -1).cpu().double().numpy()
    assert np.all(np.isfinite(y))
    assert (np.abs(y - whole["y"]) / (1 + np.abs(whole["y"]))).max() <= tol
    for (a, b), (_, h_last, final) in zip(bounds, res):
        pre = oracle.scan(*(inp[k][..., :b] if k in ("x", "dt", "z", "B", "C") else
                            inp[k][:, :b] if k == "reset" else inp[k] for k in keys))["h_last"]
        assert (np.abs(h_last.cpu().double().numpy() - pre) / (1 + np.abs(pre))).max() <= 1e-4
        ref = whole["h_last"]
        assert (np.abs(final.cpu().double().numpy() - ref) / (1 + np.abs(ref))).max() <= 1e-4


@pytest.mark.gpu
def test_emulated_ranks_full_size_layer_sampled_rows():
    """The 2.8B-layer prompt (1 x 5120 x 16384, N = 16, bf16, z gate) cut into 8
    segments, checked on sampled channels against the oracle."""
    d = _cuda()
    inp = make_scan_inputs(1, 5120, 16, 16384, "bf16", seed=20262, a_perturb=True)
    keys = ("x", "dt", "A", "B", "C", "D", "z", "dt_bias")
    inp_dev = {k: inp[k].to(d) for k in keys}
    _, res = _emulate(inp_dev, 8)
    y = torch.cat([r[0] for r in res], -1)
    rows = [(0, c) for c in (0, 1, 777, 2048, 4095, 5119)]
    ref_y, ref_h = oracle.scan_rows(inp, rows)
    got = torch.stack([y[0, c] for _, c in rows]).cpu().double().numpy()
    assert (np.abs(got - ref_y) / (1 + np.abs(ref_y))).max() <= 1e-2
    fin = res[-1][2].cpu().double().numpy()
    got_h = np.stack([fin[0, c] for _, c in rows])
    assert (np.abs(got_h - ref_h) / (1 + np.abs(ref_h))).max() <= 1e-4


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_one_segment_is_the_plain_scan_bit_for_bit(dtype):
    d = _cuda()
    inp = make_scan_inputs(2, 48, 16, 2048, dtype, seed=9, reset_mean_doc=400, h0=True)
    keys = ("x", "dt", "A", "B", "C", "D", "z", "dt_bias", "reset", "h0")
    dd = {k: inp[k].to(d) for k in keys}
    res = seqshard.seq_sharded_scan(*(dd[k] for k in keys), return_final_state=True)
    y, h = seqshard.ssscan.ss_scan_fwd(*(dd[k] for k in keys))
    torch.cuda.synchronize()
    assert torch.equal(res["y"], y) and torch.equal(res["h_last"], h) and torch.equal(res["final_state"], h)


def _leaving_worker(rank, world, port, out):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        out[rank] = "left before the exchange"
        return  # the process ends without joining the all-gather
    p = _problem()
    a, b = seqshard.shard_bounds(p["x"].shape[-1], world)[rank]
    q = _slice(p, a, b)
    try:
        seqshard.seq_sharded_scan(q["x"], q["dt"], q["A"], q["B"], q["C"], q["D"], q["z"], q["dt_bias"],
                                  q["reset"], q["h0"], steps=OracleSteps)
        out[rank] = "returned"
    except Exception as e:  # the collective fails: the peer is gone or the timeout ran out
        out[rank] = f"error: {type(e).__name__}"


def test_a_rank_that_leaves_surfaces_as_an_error_not_a_hang():
    """Failure made on the host: rank 1 exits before the exchange step.  Rank 0's
    all-gather must end with an error (peer gone, or the 5 s process-group timeout)."""
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_leaving_worker, args=(r, 2, port, out)) for r in range(2)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=90)
    alive = [pr for pr in procs if pr.is_alive()]
    for pr in alive:
        pr.kill()
    assert not alive, "a rank hung"
    assert out[1] == "left before the exchange"
    assert out[0].startswith("error"), out[0]
