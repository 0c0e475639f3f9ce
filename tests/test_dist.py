"""Host-side multi-rank logic of bench.py on CPU: two gloo ranks, one process each.

The benchmark shards independent problems over ranks (weak scaling) and reports the
maximum device time over ranks; these are the only collectives it uses."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, local = bench._dist_env()
        mx = bench.max_over_ranks(10.0 + rank, w)
        sm = bench.sum_over_ranks(1.0 + rank, w)
        out[rank] = (w, r, local, mx, sm)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timings():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        w, r, local, mx, sm = out[rank]
        assert (w, r, local) == (world, rank, rank)
        assert mx == 11.0          # the slowest rank decides the time
        assert sm == 3.0


def test_single_rank_is_identity(monkeypatch):
    import bench
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert bench._dist_env()[0] == 1
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.sum_over_ranks(2.0, 1) == 2.0


def test_ranks_get_distinct_problems():
    """Weak scaling: each rank draws its own seeded inputs."""
    import bench
    a, _ = bench._inputs_on("cpu", 0)
    b, _ = bench._inputs_on("cpu", 2)
    assert not torch.equal(a["x"][0, 0, :64], b["x"][0, 0, :64])


def test_work_accounting_matches_shapes():
    import bench
    pw, dw = bench.prompt_work(), bench.decode_work()
    assert pw["elems"] == 1 * 16384 * 5120 * 16
    assert pw["exps"] == 5120 * 16384 * 18
    # x, dt, z, y in bf16 plus B, C: about 8 bytes per (t, c)
    assert 8 * 5120 * 16384 <= pw["bytes"] <= 8.1 * 5120 * 16384
    assert dw["elems"] == 256 * 5120 * 16
    assert dw["bytes"] >= 2 * 4 * 256 * 5120 * 16
