"""Shared helpers for the parity tests: run the CUDA library through its C ABI on seeded
workloads and bring the same inputs to the oracle."""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

import linear_attention_beam_gdn_b200 as ola
import oracle
import workloads as wl

TOL_FP32 = 1e-4     # max-abs error on the fp32 paths
TOL_TENSOR = 2e-3   # max-abs error on the bf16-operand tensor-core path

PATHS = {
    "replay_fp32": (ola.OLA_PATH_REPLAY, ola.OLA_MATH_FP32),
    "replay_tensor": (ola.OLA_PATH_REPLAY, ola.OLA_MATH_TENSOR),
    "fullstate": (ola.OLA_PATH_FULLSTATE, ola.OLA_MATH_FP32),
    "replayssm": (ola.OLA_PATH_REPLAYSSM, ola.OLA_MATH_FP32),
}


def tol_for(path: str) -> float:
    return TOL_TENSOR if path == "replay_tensor" else TOL_FP32


def stack_f64(steps: Sequence[Dict[str, torch.Tensor]], key: str) -> np.ndarray:
    return np.stack([oracle.as_f64(s[key]) for s in steps])


def oracle_prefill_all(prompt: Dict[str, torch.Tensor], units=None) -> np.ndarray:
    """fp64 prefill of every (or the given) (r, h) unit; [R, H, d_v, d_k]."""
    k, v = oracle.as_f64(prompt["k"]), oracle.as_f64(prompt["v"])
    g, b = oracle.as_f64(prompt["g"]), oracle.as_f64(prompt["beta"])
    R, P, H, d_k = k.shape
    d_v = v.shape[3]
    S = np.full((R, H, d_v, d_k), np.nan)
    todo = units if units is not None else [(r, h) for r in range(R) for h in range(H)]
    for r, h in todo:
        S[r, h] = oracle.prefill(k[r, :, h], v[r, :, h], g[r, :, h], b[r, :, h])
    return S


def run_library(S_ctx: torch.Tensor, steps: List[Dict[str, torch.Tensor]], parents: np.ndarray,
                path: str, in_dtype: torch.dtype, T_max: Optional[int] = None,
                keep_on_device: bool = False):
    """Decode every step through the C ABI. Returns (o [T,R,B,H,d_v], ancestry [R,B,T],
    status of ola_get_error)."""
    p, m = PATHS[path]
    T, R, B = parents.shape
    dev = S_ctx.device
    dec = ola.Decoder(S_ctx, B=B, T_max=T_max or T, in_dtype=in_dtype, path=p, math=m)
    outs = []
    try:
        for t in range(T):
            s = steps[t]
            par = torch.from_numpy(parents[t]).to(dev)
            o = dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], par)
            outs.append(o if keep_on_device else o.cpu())
        anc = dec.ancestry().cpu().numpy()
        status = dec.error()
    finally:
        dec.close()
    o = torch.stack(outs)
    return (o if keep_on_device else o.double().numpy()), anc, status


def small_problem(w: wl.Workload, device="cuda"):
    """Inputs of a small workload on `device` plus the fp32 shared state made by the oracle's
    fp64 prefill (the same fp32 values go to both sides)."""
    prompt = wl.make_prompt(w, "cpu")
    S64 = oracle_prefill_all(prompt)
    S32 = torch.from_numpy(S64).float()
    steps = [wl.make_step_inputs(w, t, "cpu") for t in range(w.T)]
    parents = wl.make_parents(w)
    dev_steps = [{k: v.to(device) for k, v in s.items()} for s in steps]
    return S32, steps, dev_steps, parents


def oracle_outputs(S32: torch.Tensor, steps, parents, units=None) -> np.ndarray:
    return oracle.decode_batch(S32.double().numpy(), stack_f64(steps, "q"), stack_f64(steps, "k"),
                               stack_f64(steps, "v"), stack_f64(steps, "g"),
                               stack_f64(steps, "beta"), parents, units=units)


def max_abs(a: np.ndarray, b: np.ndarray) -> float:
    """Largest |a - b| over the positions where the reference b is defined (b holds NaN for
    units the oracle did not compute); a non-finite a at such a position is an infinite error,
    so unwritten (NaN-filled) or overflowed outputs never pass."""
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape, (a.shape, b.shape)
    mask = np.isfinite(b)
    if not np.all(np.isfinite(a[mask])):
        return float("inf")
    d = np.abs(a[mask] - b[mask])
    return float(d.max()) if d.size else 0.0
