"""ola_decode_noalloc: the allocation-free whole-decode entry point, for callers that may not
allocate device memory while decoding (stream capture, arena-reserved memory, latency-critical
loops). It must give the same outputs as the handle-based entry points on the same inputs,
on consecutive calls that reuse its fixed scratch, and refuse problems larger than that
scratch. Collected last on purpose (file name), so a failure here comes after every other
test has run."""
import numpy as np
import pytest
import torch

import linear_attention_beam_gdn_b200 as ola
import workloads as wl
from helpers import TOL_FP32, max_abs, run_library, small_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    from linear_attention_beam_gdn_b200 import build
    build.build()


def _stack(dev_steps, key):
    return torch.stack([s[key] for s in dev_steps]).contiguous()


@pytest.mark.parametrize("name,kw", [
    ("single_request", dict(H=4, B=40, P=32, T=4)),
    ("tiny", dict(B=8, T=3)),
])
def test_noalloc_matches_handle_path_twice(name, kw):
    w = wl.WORKLOADS[name].scaled(**kw)
    S32, steps, dev_steps, parents = small_problem(w)
    S = S32.cuda()
    ref, _, st = run_library(S, dev_steps, parents, "replay_fp32", w.torch_dtype)
    assert st == ola.OLA_OK
    geom = ola.Geometry(w.R, w.H, w.d_k, w.d_v, w.B, w.T,
                        ola.OLA_BF16 if w.dtype == "bf16" else ola.OLA_F32,
                        ola.OLA_PATH_REPLAY, ola.OLA_MATH_FP32)
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
        assert max_abs(out.double().cpu().numpy(), ref) <= TOL_FP32


def test_noalloc_rejects_oversize_and_reports_bad_parent():
    big = ola.Geometry(64, 16, 128, 128, 512, 8, ola.OLA_BF16, ola.OLA_PATH_REPLAY,
                       ola.OLA_MATH_FP32)
    assert ola.ola_noalloc_scratch_bytes(big) > ola.OLA_NOALLOC_SCRATCH_BYTES
    assert ola.ola_decode_noalloc(big, 16, 16, 16, 16, 16, 16, 16, 16, None) == \
        ola.OLA_ERR_SCRATCH_LIMIT
    tensor = ola.Geometry(1, 1, 128, 128, 8, 2, ola.OLA_BF16, ola.OLA_PATH_REPLAY,
                          ola.OLA_MATH_TENSOR)
    assert ola.ola_decode_noalloc(tensor, 16, 16, 16, 16, 16, 16, 16, 16, None) == \
        ola.OLA_ERR_UNSUPPORTED

    w = wl.WORKLOADS["tiny"].scaled(B=8, T=2)
    S32, steps, dev_steps, parents = small_problem(w)
    geom = ola.Geometry(w.R, w.H, w.d_k, w.d_v, w.B, w.T, ola.OLA_F32, ola.OLA_PATH_REPLAY,
                        ola.OLA_MATH_FP32)
    bad = parents.copy()
    bad[1, 0, 3] = w.B                      # out of range at step 2
    par = torch.from_numpy(bad).cuda().contiguous()
    out = torch.empty((w.T, w.R, w.B, w.H, w.d_v), device="cuda")
    S = S32.cuda()
    st = ola.ola_decode_noalloc(geom, S.data_ptr(), _stack(dev_steps, "q").data_ptr(),
                                _stack(dev_steps, "k").data_ptr(),
                                _stack(dev_steps, "v").data_ptr(),
                                _stack(dev_steps, "g").data_ptr(),
                                _stack(dev_steps, "beta").data_ptr(), par.data_ptr(),
                                out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == ola.OLA_ERR_BAD_PARENT
    # the next call starts from a cleared error word
    par_ok = torch.from_numpy(parents).cuda().contiguous()
    st = ola.ola_decode_noalloc(geom, S.data_ptr(), _stack(dev_steps, "q").data_ptr(),
                                _stack(dev_steps, "k").data_ptr(),
                                _stack(dev_steps, "v").data_ptr(),
                                _stack(dev_steps, "g").data_ptr(),
                                _stack(dev_steps, "beta").data_ptr(), par_ok.data_ptr(),
                                out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == ola.OLA_OK
    assert np.isfinite(out.cpu().numpy()).all()
