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


def _split_worker(rank, world, port, n_total, c, q):
    """One rank of bench.py's --split sequence path, on the CPU, with the oracle standing
    in for the kernels: its own rows (halo included) drawn piece-wise from the shared seed,
    its shards compressed, the halo entry dropped, then the sampled cross-rank check."""
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from oracle import compressor as O

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        f64 = lambda x: x.double().numpy()

        def csa_fn(sl, Ba, Bb, out):
            r = O.csa_compress(f64(sl["Ca"]), f64(sl["Cb"]), f64(sl["Za"]), f64(sl["Zb"]), f64(Ba),
                               f64(Bb), bench.M_CSA, True)
            out.copy_(torch.from_numpy(r))

        def hca_fn(Cs, Zs, B, out):
            out.copy_(torch.from_numpy(O.hca_compress(f64(Cs), f64(Zs), f64(B), bench.M_HCA)))

        t, lo, pc, ph = bench.split_inputs(n_total, world, rank, c, "f32", "cpu")
        out_c = torch.empty((1, pc.entries + int(pc.drop_first), c), dtype=torch.float64)
        out_h = torch.empty((1, ph.entries, c), dtype=torch.float64)
        oc, oh = bench.split_compress(t, lo, pc, ph, csa_fn, hca_fn, out_c, out_h)
        assert oc.shape[1] == pc.entries and oh.shape[1] == ph.entries

        def single_csa(x, Ba, Bb, j):
            return O.csa_compress(f64(x["Ca"]), f64(x["Cb"]), f64(x["Za"]), f64(x["Zb"]), f64(Ba),
                                  f64(Bb), bench.M_CSA, True, entries=[(0, j)])[0]

        def single_hca(Cs, Zs, B):
            return O.hca_compress(f64(Cs), f64(Zs), f64(B), bench.M_HCA)[0, 0]

        check = bench.split_check(world, rank, pc, ph, oc, oh, c, "f32", "cpu", single_csa,
                                  single_hca)
        parts = [None] * world
        dist.all_gather_object(parts, (oc.numpy(), oh.numpy()))
        if rank == 0:
            full = bench.split_inputs(n_total, 1, 0, c, "f32", "cpu")[0]
            ref_c = O.csa_compress(f64(full["Ca"]), f64(full["Cb"]), f64(full["Za"]), f64(full["Zb"]),
                                   f64(full["Ba"]), f64(full["Bb"]), bench.M_CSA, True)
            ref_h = O.hca_compress(f64(full["Ca"]), f64(full["Za"]), f64(full["Bh"]), bench.M_HCA)
            got_c = np.concatenate([p[0] for p in parts], axis=1)
            got_h = np.concatenate([p[1] for p in parts], axis=1)
            q.put((bool(np.array_equal(got_c, ref_c) and np.array_equal(got_h, ref_h)), check))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n_total,world", [(2 * 128 * 9 + 4 * 3 + 1, 2), (3 * 128 * 5 + 7, 3)])
def test_split_sequence_ranks_match_single_process(n_total, world):
    """bench.py --split sequence on gloo ranks: the gathered shards equal the one-process
    result bit for bit, and the bench's sampled cross-rank check passes (it includes each
    rank's first entry, the one that reads the halo)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, n_total, 16, q))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs)
    exact, (checked, worst, ok) = q.get(timeout=5)
    assert exact
    # the sampled entries travel as float32: one fp32 rounding of the fp64 oracle values
    assert ok and checked >= world * 2 and worst <= 2.0 ** -23
