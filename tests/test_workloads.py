"""Host-side checks of the seeded synthetic workloads (no GPU)."""
import numpy as np
import torch

import workloads as wl


def test_registry_shapes():
    assert len([n for n in wl.WORKLOADS if n.startswith("sweep_")]) == 27
    s = wl.WORKLOADS["stress"]
    assert (s.R, s.H, s.d_k, s.d_v, s.P, s.B, s.T, s.max_children) == (64, 16, 128, 128, 5120,
                                                                        512, 8, 32)


def test_parents_deterministic_and_valid():
    W = wl.WORKLOADS["multi_request"].scaled(R=3)
    p1, p2 = wl.make_parents(W), wl.make_parents(W)
    assert np.array_equal(p1, p2)
    assert p1.dtype == np.int32 and p1.shape == (W.T, W.R, W.B)
    assert np.all(p1[0] == 0)
    assert p1.min() >= 0 and p1.max() < W.B


def test_children_cap_respected():
    W = wl.WORKLOADS["stress"].scaled(R=2, T=4)
    par = wl.make_parents(W)
    for t in range(1, W.T):
        for r in range(W.R):
            assert np.bincount(par[t, r], minlength=W.B).max() <= W.max_children


def test_zipf_rank_frequencies():
    rng = np.random.default_rng(0)
    n = 64
    draws = wl.draw_parents(rng, n, 200000, "zipf", 1.0, None)
    freq = np.bincount(draws, minlength=n) / draws.size
    pmf = wl.zipf_pmf(n, 1.0)
    assert abs(freq[0] / freq[1] - 2.0) < 0.1      # P(0)/P(1) = 2 for s = 1
    np.testing.assert_allclose(freq[:8], pmf[:8], rtol=0.05)


def test_step_inputs_distributions():
    W = wl.WORKLOADS["single_request"]
    x = wl.make_step_inputs(W, 1)
    assert x["q"].dtype == torch.bfloat16 and x["q"].shape == (1, 128, 16, 128)
    n = torch.linalg.vector_norm(x["k"].float(), dim=-1)
    assert torch.allclose(n, torch.ones_like(n), atol=1e-2)
    assert (x["g"] < 0).all() and (x["beta"] > 0).all() and (x["beta"] < 1).all()
    y = wl.make_step_inputs(W, 1)
    assert all(torch.equal(x[k], y[k]) for k in x)
    z = wl.make_step_inputs(W, 2)
    assert not torch.equal(x["q"], z["q"])


def test_distinct_ancestor_counts_brute_force():
    W = wl.WORKLOADS["stress"].scaled(R=2, B=32, T=5, max_children=6)
    par = wl.make_parents(W)
    U = wl.distinct_ancestor_counts(par)
    for r in range(W.R):
        for t in range(W.T):
            recs = set()
            for b in range(W.B):
                cur = par[t, r, b]
                for s in range(t - 1, -1, -1):
                    recs.add((s, int(cur)))
                    cur = par[s, r, cur]
            assert U[t, r] == len(recs)
