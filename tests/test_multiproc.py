"""The multi-rank path on the CPU: world_size-2 `gloo` process groups.

Requests are independent, so ranks split them with no collective on the data path: each rank
decodes its own requests (here with the oracle, on the CPU) and only the timing is reduced
(max over ranks). These tests check the request sharding, that the per-rank results put
together equal the single-process decode, and the max-over-ranks reduction bench.py uses."""
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


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _decode_requests(w, lo, hi):
    steps = wl.make_all_steps(w)
    par = wl.make_parents(w)
    prompt = wl.make_prompt(w, "cpu")
    f = lambda key: np.stack([oracle.as_f64(s[key]) for s in steps])
    S = np.zeros((w.R, w.H, w.d_v, w.d_k))
    for r in range(lo, hi):
        for h in range(w.H):
            S[r, h] = oracle.prefill(*(oracle.as_f64(prompt[x][r, :, h])
                                       for x in ("k", "v", "g", "beta")))
    units = [(r, h) for r in range(lo, hi) for h in range(w.H)]
    o = oracle.decode_batch(S, f("q"), f("k"), f("v"), f("g"), f("beta"), par, units=units)
    return o[:, lo:hi]


def _worker(rank, world, port, result_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        w = wl.WORKLOADS["tiny"].scaled(R=5, P=16)
        lo, hi = wl.shard_requests(w.R, world, rank)
        part = _decode_requests(w, lo, hi)
        parts = [None] * world
        dist.all_gather_object(parts, (lo, hi, part))
        slowest = bench.max_over_ranks(float(rank + 1) * 1.5, world)
        if rank == 0:
            result_q.put((parts, slowest))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_requests_and_reduce_time():
    world = 2
    port = _free_port()
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    parts, slowest = q.get(timeout=240)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert slowest == 3.0
    parts = sorted(parts, key=lambda x: x[0])
    assert parts[0][0] == 0 and parts[-1][1] == 5
    assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
    joined = np.concatenate([p[2] for p in parts], axis=1)
    w = wl.WORKLOADS["tiny"].scaled(R=5, P=16)
    whole = _decode_requests(w, 0, w.R)
    np.testing.assert_array_equal(joined, whole)


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
