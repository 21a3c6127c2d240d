"""Parity at the full workload sizes, in the launch configuration bench.py times.

Inputs are generated on the device exactly as the bench does (same seeds), the shared state is
built by the library's prefill kernel, and every step runs through the C ABI. The oracle then
takes sampled (request, head) units whole (all beams, all steps), runs its own fp64 prefill
from the same prompt tokens and its full-state decode, and the GPU outputs of those units
must match within the path's tolerance; the ancestry table is compared in full, bit for bit.
"""
import numpy as np
import pytest
import torch

import linear_attention_beam_gdn_b200 as ola
import oracle
import workloads as wl
from helpers import PATHS, tol_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    from linear_attention_beam_gdn_b200 import build
    build.build()


def _run(w, paths, units):
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
    refs = {}
    for (r, h) in units:
        S_ref = oracle.prefill(*host_prompt[(r, h)])
        refs[(r, h)] = oracle.full_state_decode(S_ref, *host_steps[(r, h)], parents[:, r])
    for path in paths:
        p, m = PATHS[path]
        dec = ola.Decoder(S, B=w.B, T_max=w.T, in_dtype=w.torch_dtype, path=p, math=m)
        got = {u: [] for u in units}
        out = torch.empty((w.R, w.B, w.H, w.d_v), device=dev)
        try:
            for t in range(w.T):
                s = steps[t]
                dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], par[t], out=out)
                for (r, h) in units:
                    got[(r, h)].append(out[r, :, h].double().cpu().numpy())
            anc = dec.ancestry().cpu().numpy()
            assert dec.error() == ola.OLA_OK
        finally:
            dec.close()
            torch.cuda.empty_cache()
        assert np.array_equal(anc, anc_ref), path
        worst = 0.0
        for u in units:
            worst = max(worst, float(np.abs(np.stack(got[u]) - refs[u]).max()))
        print(f"{w.name} {path}: max-abs over {len(units)} units {worst:.3e}")
        assert worst <= tol_for(path), (path, worst)


def test_stress_full_size():
    w = wl.WORKLOADS["stress"]
    _run(w, ["replay_tensor", "replay_fp32"], [(0, 0), (37, 9), (63, 15)])


def test_multi_request_full_size_all_paths():
    w = wl.WORKLOADS["multi_request"]
    _run(w, ["replay_tensor", "replay_fp32", "fullstate"], [(0, 3), (5, 0), (7, 15)])


@pytest.mark.parametrize("name", ["sweep_dk256_dv256_B512", "sweep_dk64_dv64_B512",
                                  "sweep_dk128_dv256_B256", "sweep_dk256_dv64_B64"])
def test_sweep_full_size(name):
    w = wl.WORKLOADS[name]
    _run(w, ["replay_tensor"], [(0, 0), (15, 15)])
