"""Seeded synthetic workloads for beam-parallel Gated DeltaNet decode.

This module is shared by the CUDA library's callers (bench, tests) and by the
CPU oracle's tests. It holds the workload shapes and the random draws only:
no step of the recurrence, of projection replay or of the ancestry index is
computed here.

The pages describe the workload qualitatively: one long prompt shared by all
beams and a short decode suffix over a wide beam ("Scientific Impact
Assessment: OneLA", §3 Potential Impact and Additional Observations), prompts
of 1K and 5K tokens (§2 Methodological Rigor, Weaknesses) and a sweep over
request counts, beam widths, decode lengths and nine recurrent geometries
(§2). The industrial data is not released (§5 Strengths & Limitations), so
every input here is synthetic:

* q, k ~ N(0, 1) per component, L2-normalised along d_k, then (bf16 inputs)
  rounded to bfloat16 round-to-nearest-even; the rounded values are the
  canonical inputs that both sides read.
* v ~ N(0, 1) per component (rounded to bf16 for bf16 inputs).
* g = -softplus(N(0, 1)) (the log of the decay, alpha = exp(g)), fp32.
* beta = sigmoid(N(0, 1)), fp32.
* parents: step 1 has the single post-prefill root (every parent is 0); later
  steps draw each new beam's parent i.i.d. from a truncated Zipf law over the
  previous beams' score rank (beam 0 = best), P(i) ~ (i + 1) ** -s, or
  uniformly; an optional cap on children per parent resamples among parents
  that are not yet full.
* prompt tokens for the shared state use the same distributions.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one beam-decode workload (one GDN layer of R requests)."""

    name: str
    R: int            # requests in the batch
    H: int            # heads
    d_k: int          # key / query width
    d_v: int          # value width
    P: int            # prompt length that builds the shared state
    B: int            # beams per request
    T: int            # decode steps
    parent_law: str   # "zipf" or "uniform"
    zipf_s: float = 1.0
    max_children: Optional[int] = None
    dtype: str = "bf16"   # dtype of q, k, v: "bf16" or "f32"
    seed: int = 1000

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _sweep() -> Dict[str, Workload]:
    out = {}
    for dk in (64, 128, 256):
        for dv in (64, 128, 256):
            for B in (64, 256, 512):
                name = f"sweep_dk{dk}_dv{dv}_B{B}"
                out[name] = Workload(name, R=16, H=16, d_k=dk, d_v=dv, P=1024, B=B, T=4,
                                     parent_law="zipf", zipf_s=1.0, seed=1003)
    return out


#: The workloads the library is measured and checked on.
WORKLOADS: Dict[str, Workload] = {
    # tiny fp32 case the oracle finishes instantly
    "tiny": Workload("tiny", R=1, H=2, d_k=16, d_v=16, P=64, B=8, T=3,
                     parent_law="uniform", dtype="f32", seed=1000),
    # one request, 16 heads of 128x128, 128 beams, 1K prompt
    "single_request": Workload("single_request", R=1, H=16, d_k=128, d_v=128, P=1024, B=128,
                               T=4, parent_law="zipf", zipf_s=1.0, seed=1001),
    # 8 requests, 5K prompt, 256 beams, steep Zipf pruning
    "multi_request": Workload("multi_request", R=8, H=16, d_k=128, d_v=128, P=5120, B=256,
                              T=4, parent_law="zipf", zipf_s=1.2, seed=1002),
    # 64 requests, 5K prompt, 512 beams, 8 steps, fan-out capped at 32 children
    "stress": Workload("stress", R=64, H=16, d_k=128, d_v=128, P=5120, B=512, T=8,
                       parent_law="zipf", zipf_s=1.0, max_children=32, seed=1004),
}
WORKLOADS.update(_sweep())


# --------------------------------------------------------------------------- seeds

_ROLES = {"parents": 1, "decode": 2, "prompt": 3, "misc": 4}


def derive_seed(base: int, role: str, *idx: int) -> int:
    """A 63-bit seed for (workload seed, role, indices) via numpy's SeedSequence."""
    ss = np.random.SeedSequence([int(base), _ROLES[role], *[int(i) for i in idx]])
    return int(ss.generate_state(1, dtype=np.uint64)[0] >> np.uint64(1))


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


# --------------------------------------------------------------------------- parents

def zipf_pmf(n: int, s: float) -> np.ndarray:
    """Truncated Zipf law over ranks 0..n-1: P(i) proportional to (i + 1) ** -s."""
    p = (np.arange(1, n + 1, dtype=np.float64)) ** (-float(s))
    return p / p.sum()


def draw_parents(rng: np.random.Generator, n_prev: int, n_new: int, law: str, s: float,
                 max_children: Optional[int]) -> np.ndarray:
    """Parent index (rank among the previous beams) for each of n_new beams."""
    if law == "uniform":
        pmf = np.full(n_prev, 1.0 / n_prev)
    elif law == "zipf":
        pmf = zipf_pmf(n_prev, s)
    else:
        raise ValueError(law)
    if max_children is None:
        return rng.choice(n_prev, size=n_new, p=pmf).astype(np.int32)
    if max_children * n_prev < n_new:
        raise ValueError("children cap too small for the beam width")
    out = np.empty(n_new, dtype=np.int32)
    counts = np.zeros(n_prev, dtype=np.int64)
    for b in range(n_new):
        while True:
            p = int(rng.choice(n_prev, p=pmf))
            if counts[p] < max_children:
                break
            # the drawn parent is full: renormalise over the parents that are not
            pmf = pmf.copy()
            pmf[counts >= max_children] = 0.0
            pmf /= pmf.sum()
        counts[p] += 1
        out[b] = p
    return out


def make_parents(w: Workload) -> np.ndarray:
    """parent[t][r][b] (int32, shape [T, R, B]); step 0 (the first decode step) is all 0."""
    par = np.zeros((w.T, w.R, w.B), dtype=np.int32)
    for t in range(1, w.T):
        for r in range(w.R):
            rng = np.random.default_rng(derive_seed(w.seed, "parents", t, r))
            par[t, r] = draw_parents(rng, w.B, w.B, w.parent_law, w.zipf_s, w.max_children)
    return par


# --------------------------------------------------------------------------- tensors

def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def make_step_inputs(w: Workload, t: int, device="cpu", R: Optional[int] = None
                     ) -> Dict[str, torch.Tensor]:
    """Inputs of decode step t (0-based): q, k [R,B,H,d_k], v [R,B,H,d_v] in the workload
    dtype; g, beta [R,B,H] fp32; all contiguous on `device`."""
    R = w.R if R is None else R
    gen = _gen(device, derive_seed(w.seed, "decode", t))
    f32 = torch.float32
    q = _unit_rows(torch.randn((R, w.B, w.H, w.d_k), generator=gen, device=device, dtype=f32))
    k = _unit_rows(torch.randn((R, w.B, w.H, w.d_k), generator=gen, device=device, dtype=f32))
    v = torch.randn((R, w.B, w.H, w.d_v), generator=gen, device=device, dtype=f32)
    g = -torch.nn.functional.softplus(torch.randn((R, w.B, w.H), generator=gen, device=device,
                                                  dtype=f32))
    beta = torch.sigmoid(torch.randn((R, w.B, w.H), generator=gen, device=device, dtype=f32))
    dt = w.torch_dtype
    return {"q": q.to(dt).contiguous(), "k": k.to(dt).contiguous(), "v": v.to(dt).contiguous(),
            "g": g.contiguous(), "beta": beta.contiguous()}


def make_prompt(w: Workload, device="cpu", R: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Prompt tokens that build the shared state: k [R,P,H,d_k], v [R,P,H,d_v] in the workload
    dtype; g, beta [R,P,H] fp32."""
    R = w.R if R is None else R
    gen = _gen(device, derive_seed(w.seed, "prompt"))
    f32 = torch.float32
    dt = w.torch_dtype
    k = _unit_rows(torch.randn((R, w.P, w.H, w.d_k), generator=gen, device=device, dtype=f32)).to(dt)
    v = torch.randn((R, w.P, w.H, w.d_v), generator=gen, device=device, dtype=f32).to(dt)
    g = -torch.nn.functional.softplus(torch.randn((R, w.P, w.H), generator=gen, device=device,
                                                  dtype=f32))
    beta = torch.sigmoid(torch.randn((R, w.P, w.H), generator=gen, device=device, dtype=f32))
    return {"k": k.contiguous(), "v": v.contiguous(), "g": g.contiguous(),
            "beta": beta.contiguous()}


def make_all_steps(w: Workload, device="cpu") -> List[Dict[str, torch.Tensor]]:
    return [make_step_inputs(w, t, device) for t in range(w.T)]


def distinct_ancestor_counts(parents: np.ndarray) -> np.ndarray:
    """U[t][r]: number of distinct (step, beam) records at steps < t reachable from the beams
    of step t through the parent tables (pure bookkeeping on integer parent tables, used to
    count the bytes the replay must read).  parents: [T, R, B]."""
    T, R, B = parents.shape
    U = np.zeros((T, R), dtype=np.int64)
    for r in range(R):
        for t in range(1, T):
            live = np.unique(parents[t, r])
            total = 0
            for s in range(t - 1, -1, -1):
                total += live.size          # records of step s reachable
                if s == 0:
                    break
                live = np.unique(parents[s, r][live])
            U[t, r] = total
    return U
