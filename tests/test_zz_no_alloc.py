"""ola_decode_noalloc: the allocation-free whole-decode entry point, for callers that may not
allocate device memory while they decode (servers whose device memory an arena allocator has
reserved up front, plugins inside a host application that owns every allocation, loops that
cannot take an allocation's synchronisation). On two consecutive calls, which reuse its fixed
scratch array, it must give the FP64 oracle's outputs within the fp32 tolerance and the same
outputs as the handle-based entry points; it must refuse problems larger than that scratch and
bad pointers before anything is queued. Collected last on purpose (file name), so a failure
here comes after every other test has run."""
import ctypes

import numpy as np
import pytest
import torch

import linear_attention_beam_gdn_b200 as ola
import workloads as wl
from helpers import TOL_FP32, max_abs, oracle_outputs, run_library, small_problem


@pytest.fixture(scope="module")
def L():
    from linear_attention_beam_gdn_b200 import build
    build.build()
    return ola.lib()


def _stack(dev_steps, key):
    return torch.stack([s[key] for s in dev_steps]).contiguous()


def _geom(w):
    return ola.Geometry(w.R, w.H, w.d_k, w.d_v, w.B, w.T,
                        ola.OLA_BF16 if w.dtype == "bf16" else ola.OLA_F32,
                        ola.OLA_PATH_REPLAY, ola.OLA_MATH_FP32)


# ----------------------------------------------------------------------------- host-side checks

def test_noalloc_rejects_before_queueing_anything(L):
    """Host-side validation answers without a device: oversize problems, the tensor path, bad
    geometry and misaligned or NULL pointers (nothing is queued, so no GPU is needed)."""
    big = ola.Geometry(64, 16, 128, 128, 512, 8, ola.OLA_BF16, ola.OLA_PATH_REPLAY,
                       ola.OLA_MATH_FP32)
    assert ola.ola_noalloc_scratch_bytes(big) > ola.OLA_NOALLOC_SCRATCH_BYTES
    ok = [4096] * 8
    assert L.ola_decode_noalloc(ctypes.byref(big), *ok, None) == ola.OLA_ERR_SCRATCH_LIMIT
    tensor = ola.Geometry(1, 1, 128, 128, 8, 2, ola.OLA_BF16, ola.OLA_PATH_REPLAY,
                          ola.OLA_MATH_TENSOR)
    assert L.ola_decode_noalloc(ctypes.byref(tensor), *ok, None) == ola.OLA_ERR_UNSUPPORTED
    small = ola.Geometry(1, 2, 16, 16, 8, 3, ola.OLA_F32, ola.OLA_PATH_REPLAY, ola.OLA_MATH_FP32)
    for bad_geom, code in ((ola.Geometry(1, 2, 24, 16, 8, 3, ola.OLA_F32, ola.OLA_PATH_REPLAY,
                                         ola.OLA_MATH_FP32), ola.OLA_ERR_UNSUPPORTED),
                           (ola.Geometry(0, 2, 16, 16, 8, 3, ola.OLA_F32, ola.OLA_PATH_REPLAY,
                                         ola.OLA_MATH_FP32), ola.OLA_ERR_INVALID_ARG),
                           (ola.Geometry(1, 2, 16, 16, 8, 33, ola.OLA_F32, ola.OLA_PATH_REPLAY,
                                         ola.OLA_MATH_FP32), ola.OLA_ERR_UNSUPPORTED)):
        assert L.ola_decode_noalloc(ctypes.byref(bad_geom), *ok, None) == code
    assert L.ola_decode_noalloc(None, *ok, None) == ola.OLA_ERR_INVALID_ARG
    # argument i misaligned (S_ctx, q, k, v, out_o need 16 bytes; g, beta, parents 4)
    for i, off in ((0, 4), (1, 8), (2, 8), (3, 4), (4, 2), (5, 2), (6, 1), (7, 8)):
        args = list(ok)
        args[i] += off
        assert L.ola_decode_noalloc(ctypes.byref(small), *args, None) == \
            ola.OLA_ERR_INVALID_ARG, f"argument {i} misaligned by {off}"
        args[i] = None
        assert L.ola_decode_noalloc(ctypes.byref(small), *args, None) == \
            ola.OLA_ERR_INVALID_ARG, f"argument {i} NULL"


# ----------------------------------------------------------------------------- on the GPU

@pytest.mark.gpu
@pytest.mark.parametrize("name,kw", [
    ("single_request", dict(H=4, B=40, P=32, T=4)),
    ("tiny", dict(B=8, T=3)),
])
def test_noalloc_matches_oracle_twice(name, kw, L, cuda_ok):
    w = wl.WORKLOADS[name].scaled(**kw)
    S32, steps, dev_steps, parents = small_problem(w)
    ref = oracle_outputs(S32, steps, parents)
    S = S32.cuda()
    handle_o, _, st = run_library(S, dev_steps, parents, "replay_fp32", w.torch_dtype)
    assert st == ola.OLA_OK
    geom = _geom(w)
    assert 0 < ola.ola_noalloc_scratch_bytes(geom) <= ola.OLA_NOALLOC_SCRATCH_BYTES
    q, k, v = _stack(dev_steps, "q"), _stack(dev_steps, "k"), _stack(dev_steps, "v")
    g, beta = _stack(dev_steps, "g"), _stack(dev_steps, "beta")
    par = torch.from_numpy(parents).cuda().contiguous()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):                     # the second call reuses the scratch left behind
        out = torch.full((w.T, w.R, w.B, w.H, w.d_v), float("nan"), device="cuda")
        st = ola.ola_decode_noalloc(geom, S.data_ptr(), q.data_ptr(), k.data_ptr(),
                                    v.data_ptr(), g.data_ptr(), beta.data_ptr(),
                                    par.data_ptr(), out.data_ptr(), stream)
        assert st == ola.OLA_OK, ola.ola_strerror(st)
        got = out.double().cpu().numpy()
        assert max_abs(got, ref) <= TOL_FP32
        assert max_abs(got, handle_o) <= TOL_FP32


@pytest.mark.gpu
def test_noalloc_reports_bad_parent_then_recovers(L, cuda_ok):
    w = wl.WORKLOADS["tiny"].scaled(B=8, T=2)
    S32, steps, dev_steps, parents = small_problem(w)
    geom = _geom(w)
    bad = parents.copy()
    bad[1, 0, 3] = w.B                      # out of range at step 2
    S = S32.cuda()
    ins = [_stack(dev_steps, x) for x in ("q", "k", "v", "g", "beta")]
    out = torch.empty((w.T, w.R, w.B, w.H, w.d_v), device="cuda")
    stream = torch.cuda.current_stream().cuda_stream

    def call(par_np):
        par = torch.from_numpy(par_np).cuda().contiguous()
        return ola.ola_decode_noalloc(geom, S.data_ptr(), *[x.data_ptr() for x in ins],
                                      par.data_ptr(), out.data_ptr(), stream)

    assert call(bad) == ola.OLA_ERR_BAD_PARENT
    # the next call starts from a cleared error word
    assert call(parents) == ola.OLA_OK
    ref = oracle_outputs(S32, steps, parents)
    assert max_abs(out.double().cpu().numpy(), ref) <= TOL_FP32
