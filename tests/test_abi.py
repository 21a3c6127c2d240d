"""The C-ABI library builds, loads and exports every entry point the header declares; host-side
validation answers without a GPU (no compute calls here)."""
import ctypes

import pytest

import linear_attention_beam_gdn_b200 as ola
from linear_attention_beam_gdn_b200 import build as olabuild


@pytest.fixture(scope="module")
def L():
    olabuild.build()
    return ola.lib()


def test_every_declared_symbol_is_exported(L):
    names = ola.declared_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ola.h but not exported"


def test_version_and_strerror(L):
    assert ola.ola_version() >> 16 == 1
    for code in range(9):
        assert ola.ola_strerror(code)
    assert "unknown" in ola.ola_strerror(99)


def _geom(**kw):
    base = dict(R=1, H=2, d_k=16, d_v=16, B=8, T_max=3, in_dtype=ola.OLA_F32,
                path=ola.OLA_PATH_REPLAY, math=ola.OLA_MATH_FP32)
    base.update(kw)
    return ola.Geometry(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(R=0), ola.OLA_ERR_INVALID_ARG),
    (dict(B=0), ola.OLA_ERR_INVALID_ARG),
    (dict(in_dtype=7), ola.OLA_ERR_INVALID_ARG),
    (dict(path=5), ola.OLA_ERR_INVALID_ARG),
    (dict(d_k=48), ola.OLA_ERR_UNSUPPORTED),
    (dict(d_v=512), ola.OLA_ERR_UNSUPPORTED),
    (dict(T_max=33), ola.OLA_ERR_UNSUPPORTED),
    (dict(B=5000), ola.OLA_ERR_UNSUPPORTED),
    (dict(math=ola.OLA_MATH_TENSOR), ola.OLA_ERR_UNSUPPORTED),                 # fp32 inputs
    (dict(math=ola.OLA_MATH_TENSOR, in_dtype=ola.OLA_BF16), ola.OLA_ERR_UNSUPPORTED),  # d=16
    (dict(math=ola.OLA_MATH_TENSOR, in_dtype=ola.OLA_BF16, d_k=128, d_v=128, B=4096, R=8192,
          H=2, T_max=32), ola.OLA_ERR_UNSUPPORTED),                             # 32-bit rows
    (dict(math=ola.OLA_MATH_TENSOR, in_dtype=ola.OLA_BF16, d_k=128, d_v=128, B=16,
          path=ola.OLA_PATH_FULLSTATE), ola.OLA_ERR_UNSUPPORTED),
])
def test_geometry_validation(L, kw, code):
    out = ctypes.c_uint64(0)
    assert L.ola_workspace_bytes(ctypes.byref(_geom(**kw)), ctypes.byref(out)) == code
    h = ctypes.c_void_p(123)
    assert L.ola_create(ctypes.byref(_geom(**kw)), 4096, None, ctypes.byref(h)) == code
    assert h.value is None


def test_workspace_bytes_formula(L):
    g = _geom(R=2, H=3, d_k=64, d_v=128, B=40, T_max=5, in_dtype=ola.OLA_BF16)
    R, H, dk, dv, B, T = 2, 3, 64, 128, 40, 5
    expect = (R * H * dv * dk * 4 + T * R * H * B * dv * 4 + T * R * H * B * dk * 2 +
              T * R * H * B * 4 + T * R * B * T * 4 + 16 + R * 4)
    assert ola.ola_workspace_bytes(g) == expect
    gf = _geom(R=2, H=3, d_k=64, d_v=128, B=40, T_max=5, path=ola.OLA_PATH_FULLSTATE)
    expect_fs = R * H * dv * dk * 4 + 2 * R * H * B * dv * dk * 4 + T * R * B * T * 4 + 16 + R * 4
    assert ola.ola_workspace_bytes(gf) == expect_fs
    # history-replay path: the raw tokens of every record (k, v in the input dtype, alpha,
    # beta), no w records and no per-beam state
    gr = _geom(R=2, H=3, d_k=64, d_v=128, B=40, T_max=5, in_dtype=ola.OLA_BF16,
               path=ola.OLA_PATH_REPLAYSSM)
    expect_rs = (R * H * dv * dk * 4 + T * R * H * B * dk * 2 + T * R * H * B * 4 +
                 T * R * H * B * dv * 2 + T * R * H * B * 4 + T * R * B * T * 4 + 16 + R * 4)
    assert ola.ola_workspace_bytes(gr) == expect_rs
    # the tensor math is for the record replay path only
    assert L.ola_workspace_bytes(ctypes.byref(_geom(path=ola.OLA_PATH_REPLAYSSM,
                                                    in_dtype=ola.OLA_BF16, d_k=128, d_v=128,
                                                    math=ola.OLA_MATH_TENSOR)),
                                 ctypes.byref(ctypes.c_uint64(0))) == ola.OLA_ERR_UNSUPPORTED
    # tensor path, d_v = 128: unit plan buffers (counts, prefix, unit records, per-position
    # record indices, a counter) instead of the parent-chain table
    gt = _geom(R=2, H=3, d_k=64, d_v=128, B=40, T_max=5, in_dtype=ola.OLA_BF16,
               math=ola.OLA_MATH_TENSOR)
    split = 2 * R * H * 128 * dk * 2
    units = R * 4 + (R + 1) * 4 + R * B * 96 * 4 + R * B * 16 + 16
    assert ola.ola_workspace_bytes(gt) == (expect + split + 2 * R * B * 4 + 2 * R * B * 4 +
                                           units)
    # tensor path, d_v = 64: the same unit plan buffers
    dv2 = 64
    g2 = _geom(R=2, H=3, d_k=64, d_v=dv2, B=40, T_max=5, in_dtype=ola.OLA_BF16,
               math=ola.OLA_MATH_TENSOR)
    expect2 = (R * H * dv2 * dk * 4 + T * R * H * B * dv2 * 4 + T * R * H * B * dk * 2 +
               T * R * H * B * 4 + T * R * B * T * 4 + 16 + R * 4)
    assert ola.ola_workspace_bytes(g2) == (expect2 + 2 * R * H * 128 * dk * 2 + 2 * R * B * 4 +
                                           2 * R * B * 4 + units)
    # tensor path past the unit-planned kernel's chain depth (T_max > 12): the parent-chain
    # table instead of the unit plan
    T3 = 13
    g3 = _geom(R=2, H=3, d_k=64, d_v=dv2, B=40, T_max=T3, in_dtype=ola.OLA_BF16,
               math=ola.OLA_MATH_TENSOR)
    expect3 = (R * H * dv2 * dk * 4 + T3 * R * H * B * dv2 * 4 + T3 * R * H * B * dk * 2 +
               T3 * R * H * B * 4 + T3 * R * B * T3 * 4 + 16 + R * 4)
    assert ola.ola_workspace_bytes(g3) == (expect3 + 2 * R * H * 128 * dk * 2 + 2 * R * B * 4 +
                                           2 * R * B * 4 + R * B * T3 * 4)


def test_null_arguments(L):
    assert L.ola_create(None, 4096, None, ctypes.byref(ctypes.c_void_p())) == \
        ola.OLA_ERR_INVALID_ARG
    assert L.ola_create(ctypes.byref(_geom()), 4096, None, None) == ola.OLA_ERR_INVALID_ARG
    # NULL / misaligned shared state
    assert L.ola_create(ctypes.byref(_geom()), None, None, ctypes.byref(ctypes.c_void_p())) == \
        ola.OLA_ERR_INVALID_ARG
    assert L.ola_create(ctypes.byref(_geom()), 4100, None, ctypes.byref(ctypes.c_void_p())) == \
        ola.OLA_ERR_INVALID_ARG
    for fn in ("ola_reset", "ola_get_error"):
        assert getattr(L, fn)(None) == ola.OLA_ERR_INVALID_ARG
    assert L.ola_destroy(None) == ola.OLA_OK
    assert L.ola_current_step(None) == -1
    assert L.ola_step(None, 16, 16, 16, 16, 16, 16, 16, None) == ola.OLA_ERR_INVALID_ARG
    assert L.ola_get_ancestry(None, 16, None) == ola.OLA_ERR_INVALID_ARG
    assert L.ola_compact(None, None, None) == ola.OLA_ERR_INVALID_ARG
    assert L.ola_step_host_async(None, 16, 16, 16, 16, 16, 16, 16, None) == \
        ola.OLA_ERR_INVALID_ARG
    assert L.ola_host_sync(None) == ola.OLA_ERR_INVALID_ARG


def test_prefill_validation(L):
    assert L.ola_prefill(0, 1, 16, 16, 4, 0, 16, 16, 16, 16, 16, None) == \
        ola.OLA_ERR_INVALID_ARG
    assert L.ola_prefill(1, 1, 24, 16, 4, 0, 16, 16, 16, 16, 16, None) == \
        ola.OLA_ERR_UNSUPPORTED
    assert L.ola_prefill(1, 1, 16, 16, 4, 0, None, 16, 16, 16, 16, None) == \
        ola.OLA_ERR_INVALID_ARG
    assert L.ola_prefill(1, 1, 16, 16, 4, 0, 16, 16, 16, 16, 12, None) == \
        ola.OLA_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(ola, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(ola, "_LIB", None)
    with pytest.raises(ola.LibraryMissing):
        ola.lib()
