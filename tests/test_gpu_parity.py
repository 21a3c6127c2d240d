"""Parity of the CUDA library (through its C ABI) with the FP64 oracle on seeded inputs.

Tolerances (max-abs over every step, request, beam, head and component of o):
1e-4 on the fp32 paths, 2e-3 on the bf16-operand tensor-core path; ancestry bit-exact."""
import numpy as np
import pytest
import torch

import linear_attention_beam_gdn_b200 as ola
import oracle
import workloads as wl
from helpers import (PATHS, max_abs, oracle_outputs, oracle_prefill_all, run_library,
                     small_problem, stack_f64, tol_for)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    from linear_attention_beam_gdn_b200 import build
    build.build()
    torch.cuda.init()


def _check(w, paths, S32, steps, dev_steps, parents, ref=None):
    ref = oracle_outputs(S32, steps, parents) if ref is None else ref
    anc_ref = oracle.ancestry_table(parents)
    for path in paths:
        o, anc, status = run_library(S32.cuda(), dev_steps, parents, path, w.torch_dtype)
        assert status == ola.OLA_OK, (path, status)
        err = max_abs(o, ref)
        print(f"{w.name} {path}: max-abs {err:.3e}")
        assert err <= tol_for(path), (path, err)
        assert np.array_equal(anc, anc_ref), path
    return ref


# ----------------------------------------------------------------------------- prefill

@pytest.mark.parametrize("name", ["tiny", "single_request"])
def test_prefill_matches_oracle(name):
    w = wl.WORKLOADS[name]
    if name == "single_request":
        w = w.scaled(H=4)
    prompt = wl.make_prompt(w, "cpu")
    S_ref = oracle_prefill_all(prompt)
    dp = {k: v.cuda() for k, v in prompt.items()}
    S = ola.prefill(dp["k"], dp["v"], dp["g"], dp["beta"])
    err = max_abs(S.double().cpu().numpy(), S_ref)
    print(f"prefill {name}: max-abs {err:.3e}")
    assert err <= 1e-4


@pytest.mark.parametrize("P", [1, 63, 64, 65, 1000])
def test_prefill_chunked_ragged_lengths(P):
    """d_k = d_v = 128 with a bf16 prompt runs the chunked tensor-core prefill (64 tokens per
    chunk): prompts that end inside, at and just past a chunk boundary, and one of many chunks
    with a ragged tail, against the fp64 token recurrence."""
    w = wl.WORKLOADS["single_request"].scaled(R=2, H=3, P=P)
    prompt = wl.make_prompt(w, "cpu")
    S_ref = oracle_prefill_all(prompt)
    dp = {k: v.cuda() for k, v in prompt.items()}
    S = ola.prefill(dp["k"], dp["v"], dp["g"], dp["beta"])
    assert bool(torch.isfinite(S).all())
    err = max_abs(S.double().cpu().numpy(), S_ref)
    print(f"chunked prefill P={P}: max-abs {err:.3e}")
    assert err <= 1e-4


def test_prefill_chunked_weak_decay():
    """alpha = exp(-0.01) on every token: the state keeps the contributions of all 32 chunks,
    where the rounding of the bf16 hi/lo operands (relative 2^-17 per product) accumulates the
    most instead of decaying away. Bound: 32 chunks x a few such roundings on entries of order 1,
    well inside 2e-3."""
    w = wl.WORKLOADS["single_request"].scaled(R=1, H=2, P=2048)
    prompt = wl.make_prompt(w, "cpu")
    prompt["g"] = torch.full_like(prompt["g"], -0.01)
    S_ref = oracle_prefill_all(prompt)
    dp = {k: v.cuda() for k, v in prompt.items()}
    S = ola.prefill(dp["k"], dp["v"], dp["g"], dp["beta"])
    assert bool(torch.isfinite(S).all())
    err = max_abs(S.double().cpu().numpy(), S_ref)
    print(f"chunked prefill, weak decay: max-abs {err:.3e}, max |S| {np.abs(S_ref).max():.2f}")
    assert err <= 2e-3


def test_prefill_chunked_repeated_call_is_deterministic():
    """Same prompt twice: bit-identical states (fixed reduction order in every kernel)."""
    w = wl.WORKLOADS["single_request"].scaled(R=1, H=4, P=300)
    dp = {k: v.cuda() for k, v in wl.make_prompt(w, "cpu").items()}
    S1 = ola.prefill(dp["k"], dp["v"], dp["g"], dp["beta"])
    S2 = ola.prefill(dp["k"], dp["v"], dp["g"], dp["beta"])
    assert torch.equal(S1, S2)


def test_prefill_zero_tokens_gives_zero_state():
    w = wl.WORKLOADS["tiny"].scaled(P=0)
    k = torch.empty((1, 0, 2, 16), device="cuda")
    S = ola.prefill(k, torch.empty((1, 0, 2, 16), device="cuda"),
                    torch.empty((1, 0, 2), device="cuda"), torch.empty((1, 0, 2), device="cuda"))
    assert torch.count_nonzero(S) == 0


# ----------------------------------------------------------------------------- whole workloads

def test_tiny_all_fp32_paths():
    w = wl.WORKLOADS["tiny"]
    S32, steps, dev_steps, parents = small_problem(w)
    _check(w, ["replay_fp32", "fullstate", "replayssm"], S32, steps, dev_steps, parents)


def test_single_request_all_paths():
    w = wl.WORKLOADS["single_request"]
    S32, steps, dev_steps, parents = small_problem(w)
    _check(w, ["replay_tensor", "replay_fp32", "fullstate", "replayssm"], S32, steps, dev_steps, parents)


@pytest.mark.parametrize("d_k", [64, 128, 256])
@pytest.mark.parametrize("d_v", [64, 128, 256])
def test_geometries_reduced(d_k, d_v):
    """The nine recurrent geometries at a size the oracle finishes in seconds, with a ragged
    beam count (not a multiple of any chunk) and several tiles."""
    w = wl.WORKLOADS[f"sweep_dk{d_k}_dv{d_v}_B64"].scaled(R=2, H=2, B=100, P=128, T=4)
    S32, steps, dev_steps, parents = small_problem(w)
    _check(w, ["replay_tensor", "replay_fp32", "fullstate", "replayssm"], S32, steps, dev_steps, parents)


@pytest.mark.parametrize("d_k,d_v", [(64, 64), (128, 64), (256, 128), (64, 256), (256, 256)])
def test_geometries_past_tensor_unit_limits(d_k, d_v):
    """T_max = 14 exceeds the chain depth of the unit-planned tensor-core kernel: these handles
    run the per-chunk tensor-core kernels (d_v = 64: position-major; a 256 in the shape: the
    d_v-major kernel)."""
    w = wl.WORKLOADS[f"sweep_dk{d_k}_dv{d_v}_B64"].scaled(R=1, H=2, B=40, P=64, T=14)
    S32, steps, dev_steps, parents = small_problem(w)
    _check(w, ["replay_tensor"], S32, steps, dev_steps, parents)


@pytest.mark.parametrize("B", [16, 17, 33, 64, 65, 200])
def test_ragged_beam_counts(B):
    w = wl.WORKLOADS["single_request"].scaled(H=2, B=B, P=64, T=3)
    S32, steps, dev_steps, parents = small_problem(w)
    _check(w, ["replay_tensor", "replay_fp32", "fullstate", "replayssm"], S32, steps, dev_steps, parents)


@pytest.mark.parametrize("B", [1, 5, 31, 32, 63])
def test_small_beam_counts_all_paths(B):
    w = wl.WORKLOADS["single_request"].scaled(H=2, B=B, P=32, T=4)
    S32, steps, dev_steps, parents = small_problem(w)
    _check(w, ["replay_tensor", "replay_fp32", "fullstate", "replayssm"], S32, steps, dev_steps, parents)


@pytest.mark.parametrize("B", [1, 3, 8])
def test_tiny_beam_counts_fp32(B):
    w = wl.WORKLOADS["tiny"].scaled(B=B, T=4)
    S32, steps, dev_steps, parents = small_problem(w)
    _check(w, ["replay_fp32", "fullstate", "replayssm"], S32, steps, dev_steps, parents)


def test_max_steps_32():
    """T_max = 32 (the largest a handle holds): chains as long as a warp."""
    w = wl.WORKLOADS["single_request"].scaled(H=1, B=24, P=16, T=32)
    S32, steps, dev_steps, parents = small_problem(w)
    _check(w, ["replay_tensor", "replay_fp32", "fullstate", "replayssm"], S32, steps, dev_steps, parents)


@pytest.mark.parametrize("d_k", [64, 128])
def test_deep_chains_tensor_units(d_k):
    """d_v = 128, chains of up to 11 records (T = 12, the deepest the tensor-core replay
    accumulation takes) under steep Zipf pruning with a fan-out cap: units are cut at 48
    distinct records, several per request."""
    w = wl.WORKLOADS["stress"].scaled(R=2, H=2, d_k=d_k, B=300, P=64, T=12)
    S32, steps, dev_steps, parents = small_problem(w)
    _check(w, ["replay_tensor"], S32, steps, dev_steps, parents)


@pytest.mark.parametrize("B", [1024, 1025])
def test_beam_count_limit_of_tensor_units(B):
    """B = 1024 is the widest beam the unit-planned tensor kernel takes; 1025 goes to the
    per-chunk kernel. Both must agree with the oracle."""
    w = wl.WORKLOADS["single_request"].scaled(H=1, B=B, P=16, T=3)
    S32, steps, dev_steps, parents = small_problem(w)
    _check(w, ["replay_tensor"], S32, steps, dev_steps, parents)


def test_bf16_inputs_small_widths_fp32_path():
    w = wl.WORKLOADS["tiny"].scaled(dtype="bf16", d_k=32, d_v=16, B=12)
    S32, steps, dev_steps, parents = small_problem(w)
    _check(w, ["replay_fp32", "fullstate", "replayssm"], S32, steps, dev_steps, parents)


# ----------------------------------------------------------------------------- properties

@pytest.mark.parametrize("path", list(PATHS))
def test_identical_ancestry_bit_identical(path):
    """Two beams with the same parent and the same inputs give bit-identical outputs, wherever
    they sit in the beam array (different chunks / CTAs)."""
    w = wl.WORKLOADS["single_request"].scaled(H=2, B=130, P=32, T=3)
    S32, steps, dev_steps, parents = small_problem(w)
    parents = parents.copy()
    for t in range(w.T):
        for key in ("q", "k", "v", "g", "beta"):
            dev_steps[t][key][:, 129] = dev_steps[t][key][:, 5]
            dev_steps[t][key][:, 70] = dev_steps[t][key][:, 5]
        parents[t, :, 129] = parents[t, :, 5]
        parents[t, :, 70] = parents[t, :, 5]
    o, _, st = run_library(S32.cuda(), dev_steps, parents, path, w.torch_dtype)
    assert st == ola.OLA_OK
    assert np.array_equal(o[:, :, 129], o[:, :, 5])
    assert np.array_equal(o[:, :, 70], o[:, :, 5])


@pytest.mark.parametrize("path", list(PATHS))
def test_deterministic(path):
    w = wl.WORKLOADS["single_request"].scaled(H=4, P=32)
    S32, steps, dev_steps, parents = small_problem(w)
    o1, a1, _ = run_library(S32.cuda(), dev_steps, parents, path, w.torch_dtype)
    o2, a2, _ = run_library(S32.cuda(), dev_steps, parents, path, w.torch_dtype)
    assert np.array_equal(o1, o2) and np.array_equal(a1, a2)


def test_replay_agrees_with_fullstate_on_gpu():
    w = wl.WORKLOADS["single_request"].scaled(H=4, P=256)
    S32, steps, dev_steps, parents = small_problem(w)
    o_fs, _, _ = run_library(S32.cuda(), dev_steps, parents, "fullstate", w.torch_dtype)
    o_rp, _, _ = run_library(S32.cuda(), dev_steps, parents, "replay_fp32", w.torch_dtype)
    assert np.isfinite(o_rp).all()
    assert max_abs(o_fs, o_rp) <= 1e-4


def test_step_host_matches_step():
    w = wl.WORKLOADS["single_request"].scaled(H=2, P=32, T=3)
    S32, steps, dev_steps, parents = small_problem(w)
    o_dev, _, _ = run_library(S32.cuda(), dev_steps, parents, "replay_tensor", w.torch_dtype)
    dec = ola.Decoder(S32.cuda(), B=w.B, T_max=w.T, in_dtype=w.torch_dtype)
    try:
        for t in range(w.T):
            s = {k: v.pin_memory() for k, v in steps[t].items()}
            out = torch.empty((w.R, w.B, w.H, w.d_v)).pin_memory()
            dec.step_host(s["q"], s["k"], s["v"], s["g"], s["beta"],
                          torch.from_numpy(parents[t]).pin_memory(), out)
            assert np.array_equal(out.double().numpy(), o_dev[t])
    finally:
        dec.close()


def test_step_host_async_matches_step():
    """The pipelined host-buffer entry point (two staging sets, copy-in and copy-out streams)
    gives the device path's outputs bit for bit, over two decodes and more steps than staging
    sets."""
    w = wl.WORKLOADS["single_request"].scaled(H=2, P=32, T=5)
    S32, steps, dev_steps, parents = small_problem(w)
    o_dev, _, _ = run_library(S32.cuda(), dev_steps, parents, "replay_tensor", w.torch_dtype)
    dec = ola.Decoder(S32.cuda(), B=w.B, T_max=w.T, in_dtype=w.torch_dtype)
    hs = [{k: v.pin_memory() for k, v in steps[t].items()} for t in range(w.T)]
    hp = [torch.from_numpy(parents[t]).pin_memory() for t in range(w.T)]
    try:
        for _ in range(2):
            dec.reset()
            outs = [torch.full((w.R, w.B, w.H, w.d_v), float("nan")).pin_memory()
                    for _ in range(w.T)]
            for t in range(w.T):
                s = hs[t]
                dec.step_host_async(s["q"], s["k"], s["v"], s["g"], s["beta"], hp[t], outs[t])
            dec.host_sync()
            for t in range(w.T):
                assert np.array_equal(outs[t].double().numpy(), o_dev[t]), t
    finally:
        dec.close()


# ----------------------------------------------------------------------------- errors

def test_bad_parent_is_sticky_and_reset_clears():
    w = wl.WORKLOADS["single_request"].scaled(H=2, B=32, P=8, T=3)
    S32, steps, dev_steps, parents = small_problem(w)
    for path in PATHS:
        p, m = PATHS[path]
        dec = ola.Decoder(S32.cuda(), B=w.B, T_max=3, in_dtype=w.torch_dtype, path=p, math=m)
        try:
            s = dev_steps[0]
            bad = torch.zeros((w.R, w.B), dtype=torch.int32, device="cuda")
            bad[0, 3] = 1                       # step 1 must have parent 0
            dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], bad)
            assert dec.error() == ola.OLA_ERR_BAD_PARENT
            with pytest.raises(ola.OlaError) as ei:
                dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], bad)
            assert ei.value.status == ola.OLA_ERR_BAD_PARENT
            dec.reset()
            assert dec.error() == ola.OLA_OK and dec.t == 0
            good = torch.zeros((w.R, w.B), dtype=torch.int32, device="cuda")
            dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], good)
            s1 = dev_steps[1]
            oob = torch.full((w.R, w.B), w.B, dtype=torch.int32, device="cuda")
            dec.step(s1["q"], s1["k"], s1["v"], s1["g"], s1["beta"], oob)
            assert dec.error() == ola.OLA_ERR_BAD_PARENT
        finally:
            dec.close()


def test_capacity_and_argument_errors():
    w = wl.WORKLOADS["single_request"].scaled(H=2, B=32, P=8, T=2)
    S32, steps, dev_steps, parents = small_problem(w)
    dec = ola.Decoder(S32.cuda(), B=w.B, T_max=2, in_dtype=w.torch_dtype)
    try:
        for t in range(2):
            s = dev_steps[t]
            dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"],
                     torch.from_numpy(parents[t]).cuda())
        with pytest.raises(ola.OlaError) as ei:
            dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"],
                     torch.from_numpy(parents[1]).cuda())
        assert ei.value.status == ola.OLA_ERR_CAPACITY
        assert dec.t == 2
        # misaligned q pointer: rejected on the host, nothing launched
        out = torch.empty((w.R, w.B, w.H, w.d_v), device="cuda")
        qbuf = torch.empty(s["q"].numel() + 8, dtype=s["q"].dtype, device="cuda")
        st = ola.ola_step(dec.handle, qbuf.data_ptr() + 2, s["k"].data_ptr(),
                          s["v"].data_ptr(), s["g"].data_ptr(), s["beta"].data_ptr(),
                          torch.from_numpy(parents[1]).cuda().data_ptr(), out.data_ptr(), None)
        assert st == ola.OLA_ERR_INVALID_ARG
        assert dec.error() == ola.OLA_OK
    finally:
        dec.close()


def test_shape_checks_in_binding():
    w = wl.WORKLOADS["single_request"].scaled(H=2, B=32, P=8, T=2)
    S32, steps, dev_steps, parents = small_problem(w)
    with ola.Decoder(S32.cuda(), B=w.B, T_max=2, in_dtype=w.torch_dtype) as dec:
        s = dev_steps[0]
        with pytest.raises(ValueError):
            dec.step(s["q"][:, :16], s["k"], s["v"], s["g"], s["beta"],
                     torch.zeros((w.R, w.B), dtype=torch.int32, device="cuda"))
        with pytest.raises(TypeError):
            dec.step(s["q"].float(), s["k"], s["v"], s["g"], s["beta"],
                     torch.zeros((w.R, w.B), dtype=torch.int32, device="cuda"))


# ----------------------------------------------------------------------------- reclamation

def _converging_parents(w, merge_steps):
    """Zipf parents, except that at each step in `merge_steps` (0-based) every new beam takes
    beam 0 as its parent: after such a step all chains share every earlier slot."""
    par = wl.make_parents(w)
    for t in merge_steps:
        par[t] = 0
    return par


@pytest.mark.parametrize("path", ["replay_tensor", "replay_fp32", "replayssm", "fullstate"])
def test_compact_decodes_past_t_max(path):
    """A decode of 8 steps on a handle of T_max = 4: ola_compact after steps 3 and 6 folds the
    chain slots every beam shares into S_ctx, and the outputs of every step still match the
    oracle's full-state decode (which has no capacity limit); the ancestry after the last step
    equals the oracle's chains without the folded slots."""
    w = wl.WORKLOADS["single_request"].scaled(H=2, B=40, P=64, T=8)
    S32, steps, dev_steps, _ = small_problem(w)
    parents = _converging_parents(w, merge_steps=[2, 5])
    ref = oracle_outputs(S32, steps, parents)
    p, m = PATHS[path]
    dev = torch.device("cuda")
    dec = ola.Decoder(S32.cuda(), B=w.B, T_max=4, in_dtype=w.torch_dtype, path=p, math=m)
    folded, outs = [], []
    try:
        for t in range(w.T):
            s = dev_steps[t]
            par = torch.from_numpy(parents[t]).to(dev)
            outs.append(dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], par).cpu())
            if t in (2, 5):
                folded.append(dec.compact())
        anc = dec.ancestry().cpu().numpy()
        assert dec.error() == ola.OLA_OK
        # after step 3 (1-based) every chain shares slots 0..1; after step 6 slots 0..2 of the
        # compacted chains (steps 3..5)
        assert folded == [2, 3]
        assert dec.t == 8 - 5
    finally:
        dec.close()
    o = torch.stack(outs).double().numpy()
    err = max_abs(o, ref)
    assert err <= tol_for(path), (path, err)
    assert np.array_equal(anc, oracle.ancestry_table(parents)[:, :, 5:])


def test_compact_without_shared_prefix_changes_nothing():
    """With no chain slot shared by every beam nothing is folded, and the next steps match the
    oracle as without the call."""
    w = wl.WORKLOADS["single_request"].scaled(H=2, B=40, P=64, T=4)
    S32, steps, dev_steps, parents = small_problem(w)
    assert len(np.unique(parents[1, 0])) > 1        # step 2 keeps several parents
    ref = oracle_outputs(S32, steps, parents)
    dev = torch.device("cuda")
    dec = ola.Decoder(S32.cuda(), B=w.B, T_max=4, in_dtype=w.torch_dtype,
                      path=ola.OLA_PATH_REPLAY, math=ola.OLA_MATH_TENSOR)
    outs = []
    try:
        for t in range(w.T):
            s = dev_steps[t]
            outs.append(dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"],
                                 torch.from_numpy(parents[t]).to(dev)).cpu())
            if t == 1:
                assert dec.compact() == 0
        assert dec.error() == ola.OLA_OK
    finally:
        dec.close()
    assert max_abs(torch.stack(outs).double().numpy(), ref) <= tol_for("replay_tensor")


def _shared_prefix(table):
    """Chain slots every beam of one request shares: the first slot whose record differs
    between two beams (table: [B, t] record beam index per slot)."""
    for s in range(table.shape[1]):
        if len(np.unique(table[:, s])) > 1:
            return s
    return table.shape[1]


@pytest.mark.parametrize("path", ["replay_tensor", "replay_fp32", "replayssm", "fullstate"])
def test_compact_requests_converging_at_different_steps(path):
    """Three requests whose beams converge at different steps (each request's own merges), a
    handle of T_max = 4 decoding 9 steps with ola_compact after every step: each call folds the
    slots every request shares (the smallest shared prefix over the requests, which the oracle's
    chains give), the decode runs past T_max, and every step matches the oracle."""
    w = wl.WORKLOADS["single_request"].scaled(R=3, H=2, B=24, P=64, T=9)
    S32, steps, dev_steps, _ = small_problem(w)
    parents = wl.make_parents(w)
    for r, merges in enumerate(([1, 3, 5, 7], [2, 4, 6], [1, 2, 4, 6, 7])):
        for t in merges:
            parents[t, r] = 0
    ref = oracle_outputs(S32, steps, parents)
    p, m = PATHS[path]
    dev = torch.device("cuda")
    dec = ola.Decoder(S32.cuda(), B=w.B, T_max=4, in_dtype=w.torch_dtype, path=p, math=m)
    outs, base = [], 0                  # base: slots folded so far
    try:
        for t in range(w.T):
            s = dev_steps[t]
            outs.append(dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"],
                                 torch.from_numpy(parents[t]).to(dev)).cpu())
            table = oracle.ancestry_table(parents[: t + 1])[:, :, base:]
            expect = min(min(_shared_prefix(table[r]) for r in range(w.R)), t - base)
            got = dec.compact()
            assert got == expect, (t, got, expect)
            base += got
            assert dec.t == t + 1 - base
        anc = dec.ancestry().cpu().numpy()
        assert dec.error() == ola.OLA_OK
    finally:
        dec.close()
    assert base >= w.T - 4
    o = torch.stack(outs).double().numpy()
    err = max_abs(o, ref)
    assert err <= tol_for(path), (path, err)
    assert np.array_equal(anc, oracle.ancestry_table(parents)[:, :, base:])


@pytest.mark.parametrize("R,H,d_v", [(37, 4, 128), (149, 1, 128), (3, 16, 256), (5, 61, 64)])
def test_walk_item_counts(R, H, d_v):
    """The tensor-core replay deals its (request, head, row block) items to the 148 CTAs in
    round-robin rounds and splits the units of a last, partial round into contiguous ranges:
    exactly one round (148 items), one round plus one item (149), row-blocked items (d_v = 256:
    96 items, all in the split tail) and 305 items (two rounds plus a tail). Sampled units
    include the last items of the walk; ancestry is compared in full."""
    w = wl.WORKLOADS["single_request"].scaled(R=R, H=H, d_k=64, d_v=d_v, B=130, P=16, T=3)
    S32, steps, dev_steps, parents = small_problem(w)
    n = R * H
    units = sorted({(u // H, u % H) for u in [0, 1, n // 2, n - 3, n - 2, n - 1]})
    ref = oracle_outputs(S32, steps, parents, units=units)
    o, anc, status = run_library(S32.cuda(), dev_steps, parents, "replay_tensor", w.torch_dtype)
    assert status == ola.OLA_OK
    err = max_abs(o, ref)
    print(f"walk R={R} H={H} d_v={d_v}: max-abs {err:.3e}")
    assert err <= tol_for("replay_tensor")
    assert np.array_equal(anc, oracle.ancestry_table(parents))
