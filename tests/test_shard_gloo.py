"""Multi-rank path on the CPU: the shard plan covers every entry exactly once, and two
gloo ranks that each compress only their planned rows (halo included) reproduce the
single-process result when their outputs are gathered."""

from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from kv_token_compressor_b200 import shard, synth


@pytest.mark.parametrize("n,m,world,overlap", [(1024, 4, 2, True), (1027, 4, 3, True), (50, 4, 8, True),
                                               (640, 128, 3, False), (9, 4, 4, True), (4, 4, 2, True)])
def test_plan_covers_entries_once(n, m, world, overlap):
    p = shard.plan(n, m, world, overlap)
    assert [s.rank for s in p] == list(range(world))
    covered = [e for s in p for e in range(s.e0, s.e1)]
    assert covered == list(range(n // m))
    for s in p:
        if s.entries == 0:
            continue
        # the rank reads exactly the rows its entries' windows name, nothing else
        need = set()
        for e in range(s.e0, s.e1):
            need |= set(range(m * e, m * e + m))
            if overlap and e > 0:
                need |= set(range(m * (e - 1), m * e))
        assert set(range(s.row0, s.row1)) == need
        assert s.drop_first == (overlap and s.e0 > 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, n, m, q):
    from oracle import compressor as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = synth.stream_inputs("csa", 1, n, 16, m, "f32", seed=5)  # every rank draws the same
        s = shard.plan(n, m, world, True)[rank]
        loc = {k: (v[:, s.row0:s.row1] if v.ndim == 3 else v) for k, v in d.items()}
        part = O.csa_compress(loc["Ca"], loc["Cb"], loc["Za"], loc["Zb"], loc["Ba"], loc["Bb"], m, True)[0]
        if s.drop_first:
            part = part[1:]
        assert part.shape[0] == s.entries
        # ranks own unequal entry counts: pad to the largest, gather, then trim
        sizes = [None] * world
        dist.all_gather_object(sizes, int(part.shape[0]))
        t = torch.zeros((max(sizes), 16), dtype=torch.float64)
        t[:part.shape[0]] = torch.from_numpy(np.ascontiguousarray(part))
        gathered = [torch.zeros_like(t) for _ in range(world)]
        dist.all_gather(gathered, t)
        if rank == 0:
            full = O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"], m, True)[0]
            got = torch.cat([g[:k] for g, k in zip(gathered, sizes)]).numpy()
            q.put(bool(got.shape == full.shape and np.array_equal(got, full)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n,world", [(4 * 61 + 2, 2), (64, 2), (4 * 97 + 3, 3)])
def test_gloo_ranks_match_single_process(n, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n, 4, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    assert q.get(timeout=5) is True


def _timing_worker(rank, world, port, q):
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        # each rank's own time; every rank must come back with the slowest one
        got = bench.max_over_ranks(1.0 + 1.5 * rank, world)
        bench.barrier(world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_bench_timing_is_the_max_over_ranks():
    # The bench's multi-GPU timing (barrier, then the max over ranks of each rank's device
    # time), run over gloo on the CPU: both ranks get the slower rank's time.
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_timing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 2.5, 1: 2.5}
