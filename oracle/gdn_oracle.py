"""FP64 CPU oracle for beam-parallel Gated DeltaNet (GDN) decode.

TEST INFRASTRUCTURE ONLY. This module is the slow, plain definition that the
CUDA library is checked against. Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference leg may import it; the library's
product path never does. It shares no code with the CUDA path.

What it computes, and where that comes from
-------------------------------------------
"Scientific Impact Assessment: OneLA", §1 Core Contribution: hundreds of
beams start from one recurrent state derived from the shared prompt and
diverge through a few decode-time transitions; a GDN layer touches its prior
state only through two vector contractions (the key and query projections).
The OneLA listing's Abstract (arXiv) adds that the method is exact: it keeps
one shared state plus append-only records and never rebuilds per-beam states.

The transition is the gated delta rule of "Gated Delta Networks: Improving
Mamba2 with Delta Rule" (cited in the OneLA listing, "Builds on"): with the
state S in R^{d_v x d_k}, decay alpha = exp(g) and write strength beta,

    S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
    o_t = S_t q_t.

``full_state_decode`` runs that recurrence literally for every beam from the
shared state (the "materialise a full recurrent state for every beam"
strategy the Abstract names as the existing practice): this is the oracle.
``replay_decode`` is a second, independent fp64 routine that evaluates the
same outputs from the shared state plus per-step transition records (the
projection-replay closed form); tests pin one against the other.

Readings where the pages are silent (each is listed in the design notes):
* o_t uses the post-update state S_t.
* ``g`` is the log decay, alpha = exp(g); no query scaling, no output gate.
* Step 1 has one implicit root (the shared state); every parent is 0.
* Parents are shared across the heads of a request.
* Inputs (bf16 or fp32) are widened exactly to fp64.

parity pinned: every function here is checked by tests/test_oracle_pins.py
against closed forms, invariants or brute force that do not reuse it.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np


def as_f64(x) -> np.ndarray:
    """Widen a torch tensor (bf16 / fp32) or array to fp64 exactly."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------- one transition

def gdn_transition(S: np.ndarray, k: np.ndarray, v: np.ndarray, alpha: float, beta: float
                   ) -> np.ndarray:
    """S' = alpha * S (I - beta k k^T) + beta v k^T, written with S (k k^T) = (S k) k^T.

    Gated delta rule (Gated Delta Networks, cited in the OneLA listing).
    S: [d_v, d_k], k: [d_k], v: [d_v]."""
    u = S @ k
    return alpha * (S - beta * np.outer(u, k)) + beta * np.outer(v, k)


def gdn_transition_explicit(S: np.ndarray, k: np.ndarray, v: np.ndarray, alpha: float,
                            beta: float) -> np.ndarray:
    """The same transition with the d_k x d_k matrix (I - beta k k^T) built explicitly."""
    eye = np.eye(k.shape[0])
    return alpha * (S @ (eye - beta * np.outer(k, k))) + beta * np.outer(v, k)


def prefill(k: np.ndarray, v: np.ndarray, g: np.ndarray, beta: np.ndarray,
            S0: np.ndarray | None = None) -> np.ndarray:
    """Shared post-prefill state of one (request, head): the transition applied to every
    prompt token in order, from S = 0 (or S0).

    "Scientific Impact Assessment: OneLA", §1: all beams start from one prompt-derived
    state. k: [P, d_k], v: [P, d_v], g, beta: [P]."""
    P, d_k = k.shape
    d_v = v.shape[1]
    S = np.zeros((d_v, d_k)) if S0 is None else np.array(S0, dtype=np.float64)
    for p in range(P):
        S = gdn_transition(S, k[p], v[p], float(np.exp(g[p])), float(beta[p]))
    return S


# ----------------------------------------------------------------------------- ancestry

def chains(parents: np.ndarray) -> List[List[List[int]]]:
    """Beam ancestry by list concatenation, for one request.

    parents: [T, B] (step 0 parents must be 0: one root). Returns chain[t][b] = the record
    beam index at steps 0..t of new beam b of step t, i.e. chain[t-1][parent] + [b].
    "Scientific Impact Assessment: OneLA", §1: a lightweight ancestry index separates the
    logical beam history from where records are stored."""
    T, B = parents.shape
    prev: List[List[int]] = [[]]          # the root has no records
    out = []
    for t in range(T):
        cur = []
        for b in range(B):
            p = int(parents[t, b])
            cur.append(prev[p] + [b])
        out.append(cur)
        prev = cur
    return out


def check_parents(parents: np.ndarray, B: int) -> None:
    T = parents.shape[0]
    if np.any(parents[0] != 0):
        raise ValueError("step-0 parents must all be 0 (single post-prefill root)")
    if T > 1 and (np.any(parents[1:] < 0) or np.any(parents[1:] >= B)):
        raise ValueError("parent index out of range")


# ----------------------------------------------------------------------------- the oracle

def full_state_decode(S_ctx: np.ndarray, q: np.ndarray, k: np.ndarray, v: np.ndarray,
                      g: np.ndarray, beta: np.ndarray, parents: np.ndarray
                      ) -> np.ndarray:
    """Literal per-beam recurrence for one (request, head).

    S_ctx: [d_v, d_k]; q, k: [T, B, d_k]; v: [T, B, d_v]; g, beta: [T, B];
    parents: [T, B]. Returns o: [T, B, d_v] with o[t, b] = S_t(b) q[t, b], where
    S_t(b) = transition(S_{t-1}(parent[t, b]), k, v, alpha, beta)."""
    T, B, _ = q.shape
    d_v = v.shape[2]
    check_parents(parents, B)
    prev = [np.asarray(S_ctx, dtype=np.float64)]
    o = np.zeros((T, B, d_v))
    for t in range(T):
        cur = []
        for b in range(B):
            S = prev[int(parents[t, b])]
            Sb = gdn_transition(S, k[t, b], v[t, b], float(np.exp(g[t, b])), float(beta[t, b]))
            o[t, b] = Sb @ q[t, b]
            cur.append(Sb)
        prev = cur
    return o


def full_state_decode_states(S_ctx, q, k, v, g, beta, parents):
    """As full_state_decode, also returning every beam's state: states[t][b] = S_t(b)."""
    T, B, _ = q.shape
    check_parents(parents, B)
    prev = [np.asarray(S_ctx, dtype=np.float64)]
    o = np.zeros((T, B, v.shape[2]))
    states = []
    for t in range(T):
        cur = []
        for b in range(B):
            Sb = gdn_transition(prev[int(parents[t, b])], k[t, b], v[t, b],
                                float(np.exp(g[t, b])), float(beta[t, b]))
            o[t, b] = Sb @ q[t, b]
            cur.append(Sb)
        states.append(cur)
        prev = cur
    return o, states


# ----------------------------------------------------------------------------- replay (second routine)

def replay_decode(S_ctx: np.ndarray, q: np.ndarray, k: np.ndarray, v: np.ndarray,
                  g: np.ndarray, beta: np.ndarray, parents: np.ndarray
                  ) -> Tuple[np.ndarray, list]:
    """Projection replay in fp64: no per-beam state is ever formed.

    Each new beam appends one transition record (w, k, alpha) with
    u = S_{t-1} k, w = beta (v - alpha u), so that S_t = alpha S_{t-1} + w k^T.
    Unrolled along a beam's chain j = 1..t:
        S_t x = (prod_{i<=t} alpha_i) S_ctx x + sum_j (prod_{j<i<=t} alpha_i) w_j (k_j . x).
    The decay products are taken directly (not in log form).
    "Scientific Impact Assessment: OneLA", §1 (records of O(d_v + d_k) per beam; the
    projection-replay trick) and Additional Observations (only two projections of the
    state are ever needed).

    Returns (o [T, B, d_v], records) with records[t][b] = (w, k, alpha)."""
    T, B, _ = q.shape
    check_parents(parents, B)
    S_ctx = np.asarray(S_ctx, dtype=np.float64)
    ch = chains(parents)
    records: list = []
    o = np.zeros((T, B, v.shape[2]))

    def apply_state(chain_prev: Sequence[int], x: np.ndarray) -> np.ndarray:
        # S_{t-1} x for the state reached through records chain_prev[s] at steps s = 0..t-2
        alphas = [records[s][c][2] for s, c in enumerate(chain_prev)]
        y = float(np.prod(alphas)) * (S_ctx @ x)
        for j, c in enumerate(chain_prev):
            w_j, k_j, _ = records[j][c]
            y = y + float(np.prod(alphas[j + 1:])) * w_j * float(k_j @ x)
        return y

    for t in range(T):
        cur = []
        for b in range(B):
            chain_prev = ch[t][b][:-1]
            alpha = float(np.exp(g[t, b]))
            bt = float(beta[t, b])
            kt, qt = k[t, b], q[t, b]
            u = apply_state(chain_prev, kt)
            w = bt * (v[t, b] - alpha * u)
            o[t, b] = alpha * apply_state(chain_prev, qt) + w * float(kt @ qt)
            cur.append((w, kt.copy(), alpha))
        records.append(cur)
    return o, records


def closed_form_state(S_ctx: np.ndarray, records: list, chain: Sequence[int]) -> np.ndarray:
    """Materialise (prod alpha) S_ctx + sum_j (prod_{i>j} alpha_i) w_j k_j^T along a chain
    (chain[s] = record beam index at step s)."""
    alphas = [records[s][c][2] for s, c in enumerate(chain)]
    S = float(np.prod(alphas)) * np.asarray(S_ctx, dtype=np.float64)
    for j, c in enumerate(chain):
        w_j, k_j, _ = records[j][c]
        S = S + float(np.prod(alphas[j + 1:])) * np.outer(w_j, k_j)
    return S


# ----------------------------------------------------------------------------- batched layouts

def decode_batch(S_ctx: np.ndarray, q: np.ndarray, k: np.ndarray, v: np.ndarray, g: np.ndarray,
                 beta: np.ndarray, parents: np.ndarray, units=None) -> np.ndarray:
    """Oracle over the library's tensor layout.

    S_ctx: [R, H, d_v, d_k]; q, k: [T, R, B, H, d_k]; v: [T, R, B, H, d_v];
    g, beta: [T, R, B, H]; parents: [T, R, B]. Returns o [T, R, B, H, d_v]
    (NaN for (r, h) units not in `units`, when given)."""
    T, R, B, H, _ = q.shape
    d_v = v.shape[4]
    o = np.full((T, R, B, H, d_v), np.nan)
    todo = units if units is not None else [(r, h) for r in range(R) for h in range(H)]
    for (r, h) in todo:
        o[:, r, :, h, :] = full_state_decode(S_ctx[r, h], q[:, r, :, h], k[:, r, :, h],
                                             v[:, r, :, h], g[:, r, :, h], beta[:, r, :, h],
                                             parents[:, r])
    return o


def ancestry_table(parents: np.ndarray) -> np.ndarray:
    """Chain table for every request after the last step: [R, B, T] int32 (record beam
    index at each step), from `chains`."""
    T, R, B = parents.shape
    out = np.zeros((R, B, T), dtype=np.int32)
    for r in range(R):
        ch = chains(parents[:, r])
        out[r] = np.array(ch[T - 1], dtype=np.int32)
    return out
