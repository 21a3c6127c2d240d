"""The multi-rank path on the CPU: world_size-2 `gloo` process groups.

Requests are independent, so bench.py gives every rank its own batch of requests (the same
shape, its own seeds: bench.rank_workload) with no collective on the data path; only the timing
is reduced (bench.max_over_ranks) and the job's value is every rank's units over the slowest
rank's time (bench.job_value). These tests run that rank logic in two gloo ranks, each decoding
its own batch with the oracle on the CPU, and check that every rank's result equals the
single-process decode of that rank's workload, that the ranks' batches differ, and the
max-over-ranks reduction and job value."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as tmp

import bench
import oracle
import workloads as wl

BASE = dict(R=2, P=16)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _decode_all(w):
    steps = wl.make_all_steps(w)
    par = wl.make_parents(w)
    prompt = wl.make_prompt(w, "cpu")
    f = lambda key: np.stack([oracle.as_f64(s[key]) for s in steps])
    S = np.zeros((w.R, w.H, w.d_v, w.d_k))
    for r in range(w.R):
        for h in range(w.H):
            S[r, h] = oracle.prefill(*(oracle.as_f64(prompt[x][r, :, h])
                                       for x in ("k", "v", "g", "beta")))
    return oracle.decode_batch(S, f("q"), f("k"), f("v"), f("g"), f("beta"), par)


def _worker(rank, world, port, result_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        w = bench.rank_workload(wl.WORKLOADS["tiny"].scaled(**BASE), rank)
        part = _decode_all(w)
        parts = [None] * world
        dist.all_gather_object(parts, (rank, w.seed, part))
        ms = float(rank + 1) * 1.5
        slowest = bench.max_over_ranks(ms, world)
        value = bench.job_value(world, w.R * w.H * w.B * w.T, 4, slowest)
        if rank == 0:
            result_q.put((parts, slowest, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_decode_their_own_batches_and_reduce_time():
    world = 2
    port = _free_port()
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    parts, slowest, value = q.get(timeout=240)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert slowest == 3.0
    base = wl.WORKLOADS["tiny"].scaled(**BASE)
    units = base.R * base.H * base.B * base.T
    assert value == pytest.approx(2 * units * 4 / 3.0e-3)
    parts = sorted(parts, key=lambda x: x[0])
    assert [p[0] for p in parts] == [0, 1]
    assert parts[0][1] != parts[1][1]                       # distinct seeds
    assert not np.allclose(parts[0][2], parts[1][2])         # distinct batches
    for rank, seed, o in parts:
        w = bench.rank_workload(base, rank)
        assert w.seed == seed
        np.testing.assert_array_equal(o, _decode_all(w))


def test_rank_workloads_are_distinct():
    base = wl.WORKLOADS["stress"]
    w0, w1 = bench.rank_workload(base, 0), bench.rank_workload(base, 1)
    assert w0.seed == base.seed and w1.seed != w0.seed
    assert (w0.R, w0.B, w0.T) == (w1.R, w1.B, w1.T)
    a = wl.make_step_inputs(w0.scaled(R=1), 0)["q"]
    b = wl.make_step_inputs(w1.scaled(R=1), 0)["q"]
    assert not torch.equal(a, b)


def test_algorithmic_bytes_counts_distinct_records():
    w = wl.WORKLOADS["tiny"].scaled(dtype="bf16", d_k=64, d_v=64, B=8, T=3)
    par = np.zeros((3, 1, 8), dtype=np.int32)          # every beam forks from beam 0
    b = bench.algorithmic_bytes_per_step(w, par)
    rec = 4 * 64 + 2 * 64 + 4
    base = w.H * (4 * 64 * 64 + 8 * ((2 * 64 + 64) * 2 + 8) + 4 * 8 * 64 + 8 * rec)
    assert b[0] == base + 4 * 8 * 2                   # step 1: no ancestors
    assert b[1] == base + w.H * 1 * rec + 4 * 8 * 3   # one distinct parent record
    assert b[2] == base + w.H * 2 * rec + 4 * 8 * 4   # its parent and grandparent
