"""Host-side byte models and the operator-sweep grid of bench.py (no GPU)."""
import importlib.util
import os

import numpy as np

import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)


def test_sweep_grid_has_405_shapes():
    n = (len(bench.SWEEP_GEOMETRIES) * len(bench.SWEEP_REQUESTS) * len(bench.SWEEP_BEAMS) *
         len(bench.SWEEP_STEPS))
    assert n == 405
    assert len(set(bench.SWEEP_GEOMETRIES)) == 9


def test_fullstate_bytes_count_distinct_parents():
    w = wl.Workload("t", R=2, H=3, d_k=8, d_v=4, P=1, B=5, T=3, parent_law="uniform",
                    dtype="f32")
    par = np.zeros((3, 2, 5), dtype=np.int32)
    par[1, 0] = [0, 0, 1, 1, 4]      # request 0: 3 distinct parents
    par[1, 1] = [2, 2, 2, 2, 2]      # request 1: 1
    par[2, 0] = [0, 1, 2, 3, 4]      # 5
    par[2, 1] = [3, 3, 0, 0, 1]      # 3
    state = 4 * w.d_v * w.d_k
    per_beam = state + (2 * w.d_k + w.d_v) * 4 + 8 + 4 * w.d_v
    got = bench.fullstate_bytes_per_step(w, par)
    want = [w.R * w.H * (w.B * per_beam + n * state) for n in (1, (3 + 1) / 2, (5 + 3) / 2)]
    assert got == [int(x) for x in want]


def test_replay_bytes_grow_with_distinct_ancestors():
    w = wl.Workload("t", R=1, H=2, d_k=8, d_v=4, P=1, B=4, T=3, parent_law="uniform",
                    dtype="f32")
    same = np.zeros((3, 1, 4), dtype=np.int32)
    spread = same.copy()
    spread[1, 0] = [0, 1, 2, 3]
    spread[2, 0] = [0, 1, 2, 3]
    a, b = bench.algorithmic_bytes_per_step(w, same), bench.algorithmic_bytes_per_step(w, spread)
    rec = 4 * w.d_v + 4 * w.d_k + 4
    assert a[0] == b[0]
    # step 3: one ancestor per slot with a single parent line, four per slot when spread
    assert b[2] - a[2] == w.H * (8 - 2) * rec


def test_prefill_bytes_are_the_prompt_tensors_plus_the_state():
    """The prefill's byte model counts each prompt tensor once (as generated) and the fp32
    state once."""
    for name in ("tiny", "single_request"):
        w = wl.WORKLOADS[name].scaled(P=40)
        prompt = wl.make_prompt(w, "cpu")
        nbytes = sum(t.numel() * t.element_size() for t in prompt.values())
        assert bench.prefill_bytes(w) == nbytes + w.R * w.H * w.d_v * w.d_k * 4


def test_state_and_record_bytes_are_the_full_bytes_minus_the_io():
    """The narrower byte count differs from the full one by exactly the per-beam inputs and
    outputs and the parent and chain rows."""
    w = wl.WORKLOADS["single_request"].scaled(R=3, B=16, T=4)
    parents = wl.make_parents(w)
    full = bench.algorithmic_bytes_per_step(w, parents)
    lit = bench.state_and_record_bytes_per_step(w, parents)
    e = w.elem_bytes
    for t in range(w.T):
        io = w.R * w.H * w.B * ((2 * w.d_k + w.d_v) * e + 8 + 4 * w.d_v)
        rows = w.R * 4 * w.B * (t + 2)
        assert full[t] - lit[t] == io + rows


def test_flop_models_per_step():
    """Replay: the two shared-state contractions plus per-ancestor key products and
    accumulations, one ancestor more at each step; FullState: a fixed 8 d_v d_k per beam."""
    w = wl.Workload("t", R=2, H=3, d_k=16, d_v=8, P=1, B=5, T=4, parent_law="uniform")
    rep = bench.algorithmic_flops_per_step(w)
    n = w.R * w.H * w.B
    assert rep[0] == n * (4 * w.d_v * w.d_k + 8 * w.d_v)
    assert all(rep[t + 1] - rep[t] == n * 4 * (w.d_k + w.d_v) for t in range(w.T - 1))
    assert rep[0] - n * 8 * w.d_v == bench.tensor_flops_per_step(w)
    assert bench.fullstate_flops_per_step(w) == [n * 8 * w.d_v * w.d_k] * w.T
