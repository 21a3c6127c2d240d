"""Pins for the FP64 oracle: each check uses a fact fixed independently of the oracle's own
code (hand-worked values, the defining properties of the delta-rule write, the gradient of
the delta-rule loss by finite differences, brute force, invariants), chosen so that a
dropped term, a wrong sign, a transposed outer product or a wrong index fails one of them.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _rng(i=0):
    return np.random.default_rng(12345 + i)


def _unit(x):
    return x / np.linalg.norm(x)


def _rand_problem(T, B, d_k, d_v, seed, law="uniform"):
    rng = _rng(seed)
    S = rng.standard_normal((d_v, d_k)) * 0.3
    q = np.stack([[_unit(rng.standard_normal(d_k)) for _ in range(B)] for _ in range(T)])
    k = np.stack([[_unit(rng.standard_normal(d_k)) for _ in range(B)] for _ in range(T)])
    v = rng.standard_normal((T, B, d_v))
    g = -np.log1p(np.exp(rng.standard_normal((T, B))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, B))))
    par = np.zeros((T, B), dtype=np.int32)
    for t in range(1, T):
        par[t] = rng.integers(0, B, size=B)
    return S, q, k, v, g, beta, par


# ----------------------------------------------------------------------------- hand-worked values

def _frac(a):
    return np.array([[float(Fraction(x)) for x in row] for row in a])


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_hand_worked_examples(case):
    S_ctx = _frac(case["S_ctx"])
    steps = case["steps"]
    T, B = len(steps), len(steps[0]["parents"])
    q = np.stack([_frac(s["q"]) for s in steps])
    k = np.stack([_frac(s["k"]) for s in steps])
    v = np.stack([_frac(s["v"]) for s in steps])
    alpha = np.stack([[float(Fraction(a)) for a in s["alpha"]] for s in steps])
    beta = np.stack([[float(Fraction(a)) for a in s["beta"]] for s in steps])
    par = np.array([s["parents"] for s in steps], dtype=np.int32)
    expect = np.stack([_frac(s["o"]) for s in steps])
    g = np.log(alpha)
    o = oracle.full_state_decode(S_ctx, q, k, v, g, beta, par)
    np.testing.assert_allclose(o, expect, rtol=0, atol=1e-14)
    o2, _ = oracle.replay_decode(S_ctx, q, k, v, g, beta, par)
    np.testing.assert_allclose(o2, expect, rtol=0, atol=1e-14)
    assert oracle.chains(par)[-1] == case["chains"]


# ----------------------------------------------------------------------------- the transition

@pytest.mark.parametrize("d_k,d_v", [(4, 3), (16, 16), (8, 24)])
def test_transition_defining_properties(d_k, d_v):
    """For unit k the delta-rule write is the unique linear map with
    S'k = alpha (1 - beta) S k + beta v  and  S'x = alpha S x  for x orthogonal to k."""
    rng = _rng(d_k * 7 + d_v)
    for _ in range(5):
        S = rng.standard_normal((d_v, d_k))
        k = _unit(rng.standard_normal(d_k))
        v = rng.standard_normal(d_v)
        alpha, beta = rng.uniform(0.05, 1.0), rng.uniform(0.0, 1.0)
        S1 = oracle.gdn_transition(S, k, v, alpha, beta)
        np.testing.assert_allclose(S1 @ k, alpha * (1 - beta) * (S @ k) + beta * v,
                                   rtol=0, atol=1e-12)
        for _ in range(3):
            x = rng.standard_normal(d_k)
            x -= (x @ k) * k
            np.testing.assert_allclose(S1 @ x, alpha * (S @ x), rtol=0, atol=1e-12)


def test_transition_is_decay_then_one_sgd_step():
    """S' = A - beta * grad_A L(A), A = alpha S, L(A) = 1/2 |A k - v|^2 (any k, not only
    unit). The gradient is taken by central differences of the scalar loss, which are exact
    for a quadratic up to rounding."""
    rng = _rng(3)
    d_k, d_v = 5, 4
    S = rng.standard_normal((d_v, d_k))
    k = rng.standard_normal(d_k)          # deliberately not normalised
    v = rng.standard_normal(d_v)
    alpha, beta = 0.7, 0.35
    A = alpha * S

    def loss(M):
        r = M @ k - v
        return 0.5 * float(r @ r)

    grad = np.zeros_like(A)
    h = 1e-3
    for i in range(d_v):
        for j in range(d_k):
            E = np.zeros_like(A)
            E[i, j] = h
            grad[i, j] = (loss(A + E) - loss(A - E)) / (2 * h)
    np.testing.assert_allclose(oracle.gdn_transition(S, k, v, alpha, beta), A - beta * grad,
                               rtol=0, atol=1e-9)


def test_transition_explicit_matrix_form_agrees():
    rng = _rng(4)
    S = rng.standard_normal((6, 9))
    k, v = rng.standard_normal(9), rng.standard_normal(6)
    np.testing.assert_allclose(oracle.gdn_transition(S, k, v, 0.4, 0.8),
                               oracle.gdn_transition_explicit(S, k, v, 0.4, 0.8),
                               rtol=0, atol=1e-13)


def test_delta_overwrite_exact():
    """alpha = 1, beta = 1, k = e_i, q = k: the new state reads back exactly v."""
    rng = _rng(5)
    d = 8
    S = rng.standard_normal((d, d))
    for i in range(d):
        e = np.zeros(d)
        e[i] = 1.0
        v = rng.standard_normal(d)
        o = oracle.full_state_decode(S, e[None, None], e[None, None], v[None, None],
                                     np.zeros((1, 1)), np.ones((1, 1)), np.zeros((1, 1), np.int32))
        assert np.array_equal(o[0, 0], v)


def test_prefill_orthogonal_writes_store_values():
    """alpha = 1, beta = 1 and orthonormal keys e_1..e_P from S = 0: S = sum_p v_p e_p^T."""
    rng = _rng(6)
    d_k, d_v, P = 8, 5, 6
    K = np.eye(d_k)[:P]
    V = rng.standard_normal((P, d_v))
    S = oracle.prefill(K, V, np.zeros(P), np.ones(P))
    expect = np.zeros((d_v, d_k))
    expect[:, :P] = V.T
    np.testing.assert_allclose(S, expect, rtol=0, atol=1e-15)


def test_prefill_first_token_and_pure_decay():
    rng = _rng(7)
    k, v = _unit(rng.standard_normal((1, 6))[0])[None], rng.standard_normal((1, 4))
    S = oracle.prefill(k, v, np.array([-0.3]), np.array([0.6]))
    np.testing.assert_allclose(S, 0.6 * np.outer(v[0], k[0]), rtol=0, atol=1e-15)
    S0 = rng.standard_normal((4, 6))
    g = -rng.uniform(0, 1, size=5)
    S5 = oracle.prefill(rng.standard_normal((5, 6)), rng.standard_normal((5, 4)), g,
                        np.zeros(5), S0=S0)
    np.testing.assert_allclose(S5, np.exp(g.sum()) * S0, rtol=1e-13, atol=0)


# ----------------------------------------------------------------------------- decode special cases

def test_beta_zero_is_pure_decay_along_chain():
    """beta = 0 at every step: o_t(b) = (product of alpha along b's chain) S_ctx q_t(b)."""
    T, B, d = 4, 6, 8
    S, q, k, v, g, beta, par = _rand_problem(T, B, d, d, 8)
    beta[:] = 0.0
    o = oracle.full_state_decode(S, q, k, v, g, beta, par)
    ch = oracle.chains(par)
    for t in range(T):
        for b in range(B):
            decay = np.prod([np.exp(g[s, c]) for s, c in enumerate(ch[t][b])])
            np.testing.assert_allclose(o[t, b], decay * (S @ q[t, b]), rtol=1e-13, atol=1e-14)


def test_zero_context_first_step():
    """S_ctx = 0 and t = 1: o = beta (k . q) v."""
    T, B, d = 1, 5, 7
    S, q, k, v, g, beta, par = _rand_problem(T, B, d, d + 2, 9)
    o = oracle.full_state_decode(np.zeros_like(S), q, k, v, g, beta, par)
    for b in range(B):
        np.testing.assert_allclose(o[0, b], beta[0, b] * (k[0, b] @ q[0, b]) * v[0, b],
                                   rtol=1e-14, atol=1e-15)


def test_single_beam_is_sequential_decode():
    """B = 1 (all parents 0) is plain single-sequence decode: running the prompt recurrence
    over context + decode tokens gives the same final state."""
    T, d_k, d_v = 5, 6, 4
    S, q, k, v, g, beta, par = _rand_problem(T, 1, d_k, d_v, 10)
    o, states = oracle.full_state_decode_states(S, q, k, v, g, beta, par)
    S_seq = oracle.prefill(k[:, 0], v[:, 0], g[:, 0], beta[:, 0], S0=S)
    np.testing.assert_allclose(states[-1][0], S_seq, rtol=0, atol=1e-13)
    np.testing.assert_allclose(o[-1, 0], S_seq @ q[-1, 0], rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------- replay vs full state

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_replay_equals_full_state(seed):
    """Check (a): projection replay (shared state + records) equals the literal recurrence."""
    W = wl.WORKLOADS["tiny"]
    S, q, k, v, g, beta, par = _rand_problem(W.T, W.B, W.d_k, W.d_v, 20 + seed)
    o_full = oracle.full_state_decode(S, q, k, v, g, beta, par)
    o_rep, _ = oracle.replay_decode(S, q, k, v, g, beta, par)
    np.testing.assert_allclose(o_rep, o_full, rtol=0, atol=1e-12)


def test_closed_form_state_matches_literal_state():
    """Check (b): (prod alpha) S_ctx + sum_j (prod_{i>j} alpha_i) w_j k_j^T == S_t."""
    T, B, d_k, d_v = 4, 6, 8, 5
    S, q, k, v, g, beta, par = _rand_problem(T, B, d_k, d_v, 30)
    _, states = oracle.full_state_decode_states(S, q, k, v, g, beta, par)
    _, recs = oracle.replay_decode(S, q, k, v, g, beta, par)
    ch = oracle.chains(par)
    for t in range(T):
        for b in range(B):
            St = oracle.closed_form_state(S, recs, ch[t][b])
            np.testing.assert_allclose(St, states[t][b], rtol=0, atol=1e-12)
            # and the one-step form S_t = alpha S_{t-1} + w k^T
            w, kk, a = recs[t][b]
            prev = S if t == 0 else states[t - 1][par[t, b]]
            np.testing.assert_allclose(a * prev + np.outer(w, kk), states[t][b], rtol=0,
                                       atol=1e-12)


def test_identical_ancestry_gives_identical_outputs():
    """Check (c): two beams with the same parent and the same inputs agree bit for bit."""
    T, B, d = 3, 6, 8
    S, q, k, v, g, beta, par = _rand_problem(T, B, d, d, 40)
    for arr in (q, k, v, g, beta):
        arr[:, 4] = arr[:, 1]
    par[:, 4] = par[:, 1]
    o = oracle.full_state_decode(S, q, k, v, g, beta, par)
    assert np.array_equal(o[:, 4], o[:, 1])
    o2, _ = oracle.replay_decode(S, q, k, v, g, beta, par)
    assert np.array_equal(o2[:, 4], o2[:, 1])


def test_beam_permutation_equivariance():
    """Renumbering the beams of one step (inputs, parents, and the next step's parent indices)
    permutes that step's outputs and leaves the rest unchanged."""
    T, B, d = 3, 7, 6
    S, q, k, v, g, beta, par = _rand_problem(T, B, d, d, 50)
    o = oracle.full_state_decode(S, q, k, v, g, beta, par)
    perm = _rng(51).permutation(B)
    inv = np.argsort(perm)
    q2, k2, v2, g2, b2, p2 = (x.copy() for x in (q, k, v, g, beta, par))
    for x, x2 in ((q, q2), (k, k2), (v, v2), (g, g2), (beta, b2), (par, p2)):
        x2[1] = x[1][perm]
    p2[2] = inv[par[2]]
    o2 = oracle.full_state_decode(S, q2, k2, v2, g2, b2, p2)
    np.testing.assert_allclose(o2[1], o[1][perm], rtol=0, atol=1e-14)
    np.testing.assert_allclose(o2[2], o[2], rtol=0, atol=1e-14)
    np.testing.assert_allclose(o2[0], o[0], rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------- ancestry

def test_chains_by_walking_parent_pointers():
    W = wl.WORKLOADS["stress"].scaled(R=2, B=64, T=6, max_children=8)
    par = wl.make_parents(W)
    for r in range(W.R):
        ch = oracle.chains(par[:, r])
        for t in range(W.T):
            for b in range(W.B):
                # brute force: climb the parent pointers from (t, b) to the root
                walk, cur = [], b
                for s in range(t, -1, -1):
                    walk.append(cur)
                    cur = par[s, r, cur]
                assert ch[t][b] == walk[::-1]
                assert ch[t][b][t] == b
                if t > 0:
                    assert ch[t][b][:t] == ch[t - 1][par[t, r, b]]


def _walk_table(par):
    """[R, B, T] record beam index of every slot of every final beam, by climbing the parent
    pointers from (T-1, b) of each request to the root."""
    T, R, B = par.shape
    out = np.zeros((R, B, T), dtype=np.int64)
    for r in range(R):
        for b in range(B):
            cur = b
            for s in range(T - 1, -1, -1):
                out[r, b, s] = cur
                cur = par[s, r, cur]
    return out


def test_ancestry_table_by_walking_parent_pointers():
    """Every entry of the table, for every request: requests draw different parents (their
    own seeds), so a table built from one request's parents for all of them fails."""
    W = wl.WORKLOADS["stress"].scaled(R=3, B=48, T=5, max_children=6)
    par = wl.make_parents(W)
    assert not np.array_equal(par[:, 0], par[:, 1]) and not np.array_equal(par[:, 1], par[:, 2])
    table = oracle.ancestry_table(par)
    assert table.shape == (W.R, W.B, W.T)
    assert np.array_equal(table, _walk_table(par))
    # a hand-made two-request tree: request 0 keeps every beam, request 1 follows beam 1
    par2 = np.zeros((3, 2, 3), dtype=np.int32)
    par2[1, 0] = [0, 1, 2]
    par2[2, 0] = [2, 0, 1]
    par2[1, 1] = [1, 1, 0]
    par2[2, 1] = [1, 2, 2]
    # worked by hand: slot s of final beam b is the beam it descends from at step s
    exp = np.array([[[2, 2, 0], [0, 0, 1], [1, 1, 2]],
                    [[1, 1, 0], [0, 2, 1], [0, 2, 2]]])
    assert np.array_equal(oracle.ancestry_table(par2), exp)


def test_bad_parents_rejected():
    S, q, k, v, g, beta, par = _rand_problem(2, 3, 4, 4, 60)
    par[0, 1] = 1
    with pytest.raises(ValueError):
        oracle.full_state_decode(S, q, k, v, g, beta, par)
    par[0, 1] = 0
    par[1, 2] = 3
    with pytest.raises(ValueError):
        oracle.full_state_decode(S, q, k, v, g, beta, par)


def test_batch_layout_matches_units():
    """decode_batch over the library's [T,R,B,H,d] layout equals per-unit decodes."""
    W = wl.WORKLOADS["tiny"].scaled(R=2, H=2)
    steps = wl.make_all_steps(W)
    par = wl.make_parents(W)
    q = np.stack([oracle.as_f64(s["q"]) for s in steps])
    k = np.stack([oracle.as_f64(s["k"]) for s in steps])
    v = np.stack([oracle.as_f64(s["v"]) for s in steps])
    g = np.stack([oracle.as_f64(s["g"]) for s in steps])
    beta = np.stack([oracle.as_f64(s["beta"]) for s in steps])
    S = _rng(70).standard_normal((W.R, W.H, W.d_v, W.d_k))
    o = oracle.decode_batch(S, q, k, v, g, beta, par)
    for r in range(W.R):
        for h in range(W.H):
            ou, _ = oracle.replay_decode(S[r, h], q[:, r, :, h], k[:, r, :, h], v[:, r, :, h],
                                         g[:, r, :, h], beta[:, r, :, h], par[:, r])
            np.testing.assert_allclose(o[:, r, :, h], ou, rtol=0, atol=1e-12)
