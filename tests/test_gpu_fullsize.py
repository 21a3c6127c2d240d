"""Parity at the full workload sizes, in the launch configuration bench.py times.

Inputs are generated on the device exactly as the bench does (same seeds), the shared state is
built by the library's prefill kernel, and every step runs through the C ABI. The oracle then
takes sampled (request, head) units whole (all beams, all steps), runs its own fp64 prefill
from the same prompt tokens and its full-state decode, and the GPU outputs of those units
must match within the path's tolerance; the ancestry table is compared in full, bit for bit.
"""
import os

import numpy as np
import pytest
import torch

import linear_attention_beam_gdn_b200 as ola
import oracle
import workloads as wl
from helpers import PATHS, tol_for

pytestmark = pytest.mark.gpu

N_SM = 148      # the persistent tensor-core kernels run one CTA per SM of a B200


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    from linear_attention_beam_gdn_b200 import build
    build.build()


@pytest.fixture(scope="module")
def pool():
    """Host processes for the oracle (spawned: no CUDA state is inherited)."""
    import multiprocessing as mp
    n = max(1, min(len(os.sched_getaffinity(0)), 32))
    p = mp.get_context("spawn").Pool(n)
    yield p
    p.close()
    p.join()


def _oracle_unit(args):
    prompt, steps, parents_r = args
    S_ref = oracle.prefill(*prompt)
    return oracle.full_state_decode(S_ref, *steps, parents_r)


def _run(w, paths, units, pool):
    dev = torch.device("cuda")
    prompt = wl.make_prompt(w, dev)
    S = ola.prefill(prompt["k"], prompt["v"], prompt["g"], prompt["beta"])
    host_prompt = {(r, h): tuple(oracle.as_f64(prompt[x][r, :, h]) for x in
                                 ("k", "v", "g", "beta")) for r, h in units}
    del prompt
    steps = [wl.make_step_inputs(w, t, dev) for t in range(w.T)]
    parents = wl.make_parents(w)
    par = [torch.from_numpy(parents[t]).to(dev) for t in range(w.T)]
    host_steps = {(r, h): tuple(np.stack([oracle.as_f64(s[x][r, :, h]) for s in steps])
                                for x in ("q", "k", "v", "g", "beta")) for r, h in units}
    anc_ref = oracle.ancestry_table(parents)
    jobs = pool.map_async(_oracle_unit, [(host_prompt[u], host_steps[u], parents[:, u[0]])
                                         for u in units])
    idx = torch.tensor([r * w.H + h for r, h in units], device=dev)
    got_all = {}
    for path in paths:
        p, m = PATHS[path]
        dec = ola.Decoder(S, B=w.B, T_max=w.T, in_dtype=w.torch_dtype, path=p, math=m)
        got = []
        out = torch.empty((w.R, w.B, w.H, w.d_v), device=dev)
        try:
            for t in range(w.T):
                s = steps[t]
                dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], par[t], out=out)
                # the sampled units' outputs: [n_units, B, d_v]
                flat = out.permute(0, 2, 1, 3).reshape(w.R * w.H, w.B, w.d_v)
                got.append(flat.index_select(0, idx).double().cpu())
            anc = dec.ancestry().cpu().numpy()
            assert dec.error() == ola.OLA_OK
        finally:
            dec.close()
            torch.cuda.empty_cache()
        assert np.array_equal(anc, anc_ref), path
        got_all[path] = torch.stack(got, 1).numpy()       # [n_units, T, B, d_v]
    refs = jobs.get(timeout=1800)
    for path in paths:
        worst = max(float(np.abs(got_all[path][i] - refs[i]).max()) for i in range(len(units)))
        print(f"{w.name} {path}: max-abs over {len(units)} units {worst:.3e}")
        assert np.isfinite(worst) and worst <= tol_for(path), (path, worst)


def _tail_units(w, n=N_SM):
    """The last n (request, head) units: one in every residue class modulo the CTA count, and
    the last unit each CTA of the persistent kernels walks (units are dealt round-robin)."""
    last = w.R * w.H
    return [(u // w.H, u % w.H) for u in range(max(0, last - n), last)]


def test_stress_full_size(pool):
    w = wl.WORKLOADS["stress"]
    units = [(0, 0), (0, 1), (1, 7), (37, 9)] + _tail_units(w)
    # the two comparison paths too (FullState holds 2 x 34 GB of per-beam states here)
    _run(w, ["replay_tensor", "replay_fp32", "fullstate", "replayssm"], units, pool)


def test_multi_request_full_size_all_paths(pool):
    w = wl.WORKLOADS["multi_request"]
    units = [(r, h) for r in range(w.R) for h in (0, 15)] + [(3, 5), (6, 9)]
    _run(w, ["replay_tensor", "replay_fp32", "fullstate", "replayssm"], units, pool)


@pytest.mark.parametrize("B", [64, 256, 512])
@pytest.mark.parametrize("d_v", [64, 128, 256])
@pytest.mark.parametrize("d_k", [64, 128, 256])
def test_sweep_full_size(d_k, d_v, B, pool):
    """Every workload of the geometry sweep (R = 16, H = 16, P = 1024, T = 4) at full size: the
    first unit, the last unit of the last CTA's walk, and one in between."""
    w = wl.WORKLOADS[f"sweep_dk{d_k}_dv{d_v}_B{B}"]
    _run(w, ["replay_tensor"], [(0, 0), (9, 4), (15, 15)], pool)
