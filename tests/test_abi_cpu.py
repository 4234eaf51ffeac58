"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every entry point
that include/kta.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kta():
    from hybrid_linear_temporal_kta_b200 import build
    build.build()
    from hybrid_linear_temporal_kta_b200 import kta as mod
    return mod


def declared_entry_points():
    text = open(os.path.join(ROOT, "include", "kta.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kta_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_operator_entry_points():
    names = declared_entry_points()
    for n in ("kta_swa_fwd", "kta_dswa_fwd", "kta_gla_chunk_fwd", "kta_gla_delta_fwd",
              "kta_gla_gdn_fwd", "kta_hybrid_fwd", "kta_hybrid_fwd_window", "kta_state_affine",
              "kta_stream_create", "kta_stream_step", "kta_stream_reset",
              "kta_stream_state_bytes", "kta_stream_save", "kta_stream_load",
              "kta_stream_destroy", "kta_status_str", "kta_proj_fwd", "kta_softmax_fwd_lse",
              "kta_softmax_bwd_bf16", "kta_swa_bwd", "kta_dswa_bwd", "kta_gla_bwd",
              "kta_gla_delta_bwd"):
        assert n in names


def test_library_exports_every_declared_symbol(kta):
    lib = ctypes.CDLL(kta._LIB_PATH)
    missing = [n for n in declared_entry_points() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(kta.EXPORTED) == set(declared_entry_points())


def test_status_strings_and_version(kta):
    assert kta.version() == 1
    assert kta._lib.kta_status_str(0) == b"KTA_OK"
    assert kta._lib.kta_status_str(5) == b"KTA_ERR_TIMEOUT"


def _shape(kta, B=1, F=2, P=16, d=64, dt=0):
    return kta.Shape(B, F, P, d, dt)


def test_argument_errors_are_reported_before_any_launch(kta):
    good = ctypes.c_void_p(0x10000)      # never dereferenced: validation fails first
    null = ctypes.c_void_p(0)
    st = ctypes.c_void_p(0)
    s = _shape(kta)
    # null pointer
    assert kta.raw_call("kta_swa_fwd", null, good, good, good, s, 1, 1, 2, 0.1, st) == 1
    # head dim not supported
    assert kta.raw_call("kta_swa_fwd", good, good, good, good, _shape(kta, d=96), 1, 1, 2, 0.1,
                        st) == 2
    # bf16 softmax needs d >= 64
    assert kta.raw_call("kta_swa_fwd", good, good, good, good, _shape(kta, d=32), 1, 1, 2, 0.1,
                        st) == 2
    # misaligned pointer
    assert kta.raw_call("kta_swa_fwd", ctypes.c_void_p(0x10002), good, good, good, s, 1, 1, 2, 0.1,
                        st) == 3
    # W < 1, dil < 1, H > ld_heads, non-positive sizes, bad scale
    assert kta.raw_call("kta_swa_fwd", good, good, good, good, s, 1, 1, 0, 0.1, st) == 1
    assert kta.raw_call("kta_dswa_fwd", good, good, good, good, s, 1, 1, 2, 0, 0.1, st) == 1
    assert kta.raw_call("kta_swa_fwd", good, good, good, good, s, 3, 2, 2, 0.1, st) == 1
    assert kta.raw_call("kta_swa_fwd", good, good, good, good, _shape(kta, P=0), 1, 1, 2, 0.1,
                        st) == 1
    assert kta.raw_call("kta_swa_fwd", good, good, good, good, s, 1, 1, 2, -1.0, st) == 1
    assert "scale" in kta.last_error()
    # GLA: bad chunk, null gates
    assert kta.raw_call("kta_gla_chunk_fwd", good, good, good, good, null, null, good, s, 1, 1, 48,
                        1.0, st) == 1
    assert kta.raw_call("kta_gla_delta_fwd", good, good, good, good, null, null, null, good, s, 1,
                        1, 64, 1.0, st) == 1
    # row stride not a multiple of 16 bytes: fp32, d = 32, ... is fine; bf16 d=64 fine; use H=1,
    # ld_heads=1 with d=32 bf16 -> 64 B ok; cannot make it odd with supported d, so check that a
    # valid stride passes validation up to the pointer check
    assert kta.raw_call("kta_swa_fwd", null, good, good, good, _shape(kta, d=128), 1, 3, 2, 0.1,
                        st) == 1


def test_hybrid_and_stream_validation(kta):
    import torch
    st = ctypes.c_void_p(0)
    good = ctypes.c_void_p(0x10000)
    cfg = kta.hybrid_cfg(B=1, F=2, P=16, d=64, n_swa=1, n_dswa=1, n_gla=1)
    bad = kta.hybrid_cfg(B=1, F=2, P=16, d=64, n_swa=0, n_dswa=0, n_gla=0)
    assert kta.raw_call("kta_hybrid_fwd", ctypes.byref(bad), good, good, good, good, None, good,
                        st) == 1
    bad = kta.hybrid_cfg(B=1, F=2, P=16, d=64, n_swa=1, n_dswa=1, n_gla=1, chunk=8)
    assert kta.raw_call("kta_hybrid_fwd", ctypes.byref(bad), good, good, good, good, None, good,
                        st) == 1
    bad = kta.hybrid_cfg(B=1, F=2, P=16, d=64, n_swa=1, n_dswa=1, n_gla=1, dil=0)
    assert kta.raw_call("kta_hybrid_fwd", ctypes.byref(bad), good, good, good, good, None, good,
                        st) == 1
    # GLA heads need alpha; delta needs beta too
    assert kta.raw_call("kta_hybrid_fwd", ctypes.byref(cfg), good, good, good, None, None, good,
                        st) == 1
    dcfg = kta.hybrid_cfg(B=1, F=2, P=16, d=64, n_swa=0, n_dswa=0, n_gla=1, gla_delta=True)
    assert kta.raw_call("kta_hybrid_fwd", ctypes.byref(dcfg), good, good, good, good, None, good,
                        st) == 1
    # stream handle misuse
    h = ctypes.c_void_p(0x1234)
    assert kta.raw_call("kta_stream_step", h, good, good, good, good, None, good, st) == 6
    assert kta.raw_call("kta_stream_destroy", h) == 6
    assert kta.raw_call("kta_stream_frame", h) == -1
    out = ctypes.c_void_p()
    bad = kta.hybrid_cfg(B=1, F=2, P=16, d=64, n_swa=1, n_dswa=0, n_gla=0, W_swa=0)
    assert kta.raw_call("kta_stream_create", ctypes.byref(bad), ctypes.byref(out)) == 1
    assert out.value is None
    assert torch is not None


def test_selftest_budget_is_validated(kta):
    assert kta.raw_call("kta_selftest_wait_timeout", ctypes.c_longlong(0), ctypes.c_void_p(0)) == 1
    assert kta.raw_call("kta_selftest_wait_timeout", ctypes.c_longlong(1 << 40),
                        ctypes.c_void_p(0)) == 1


def test_new_entry_points_validate_before_any_launch(kta):
    """Projection, reverse-mode and sequence-split entry points: argument errors come back before
    any CUDA call (fake pointers are never dereferenced)."""
    good = ctypes.c_void_p(0x10000)
    null = ctypes.c_void_p(0)
    st = ctypes.c_void_p(0)
    seg = (kta.ProjSeg * 2)()
    seg[0] = kta.ProjSeg(0, 8, 0x10000, 8, kta.PROJ_BF16, None)
    seg[1] = kta.ProjSeg(8, 16, 0x20000, 8, kta.PROJ_SIGMOID_F32, None)
    assert kta.raw_call("kta_proj_fwd", null, good, 4, 16, 64, seg, 2, st) == 1      # null x
    assert kta.raw_call("kta_proj_fwd", ctypes.c_void_p(0x10004), good, 4, 16, 64, seg, 2, st) == 3
    assert kta.raw_call("kta_proj_fwd", good, good, 4, 16, 12, seg, 2, st) == 3       # K % 8
    assert kta.raw_call("kta_proj_fwd", good, good, 4, 16, 64, seg, 0, st) == 1       # no ranges
    assert kta.raw_call("kta_proj_fwd", good, good, 4, 12, 64, seg, 2, st) == 1       # past N
    over = (kta.ProjSeg * 2)()
    over[0] = kta.ProjSeg(0, 8, 0x10000, 8, kta.PROJ_BF16, None)
    over[1] = kta.ProjSeg(4, 12, 0x20000, 8, kta.PROJ_F32, None)
    assert kta.raw_call("kta_proj_fwd", good, good, 4, 16, 64, over, 2, st) == 1      # overlap
    over[1] = kta.ProjSeg(8, 16, 0x20000, 8, 7, None)
    assert kta.raw_call("kta_proj_fwd", good, good, 4, 16, 64, over, 2, st) == 1      # bad mode
    over[1] = kta.ProjSeg(8, 16, 0x20000, 4, kta.PROJ_F32, None)
    assert kta.raw_call("kta_proj_fwd", good, good, 4, 16, 64, over, 2, st) == 1      # ld < width

    s_bf = _shape(kta)
    s_f32 = _shape(kta, dt=1)
    # bf16 reverse mode and its forward: bf16 and d in {64, 128} only; lse required
    assert kta.raw_call("kta_softmax_fwd_lse", good, good, good, good, good, s_f32, 1, 1, 2, 1,
                        0.1, st) == 2
    assert kta.raw_call("kta_softmax_fwd_lse", good, good, good, good, null, s_bf, 1, 1, 2, 1,
                        0.1, st) == 1
    assert kta.raw_call("kta_softmax_bwd_bf16", good, good, good, good, good, good, good, good,
                        good, s_f32, 1, 1, 2, 1, 0.1, st) == 2
    assert kta.raw_call("kta_softmax_bwd_bf16", good, good, good, good, null, good, good, good,
                        good, s_bf, 1, 1, 2, 1, 0.1, st) == 1
    assert kta.raw_call("kta_softmax_bwd_bf16", good, good, good, good, good, good, good, good,
                        good, s_bf, 1, 1, 0, 1, 0.1, st) == 1
    # fp32 reverse mode refuses bf16; GLA gates required
    assert kta.raw_call("kta_swa_bwd", good, good, good, good, good, good, good, s_bf, 1, 1, 2,
                        0.1, st) == 2
    assert kta.raw_call("kta_gla_bwd", good, good, good, null, null, good, good, good, good, good,
                        null, s_f32, 1, 1, 1.0, st) == 1
    # windowed hybrid: f0 range, one sequence for f0 > 0, aligned states
    cfg = kta.hybrid_cfg(B=2, F=3, P=16, d=64, n_swa=1, n_dswa=0, n_gla=0)
    assert kta.raw_call("kta_hybrid_fwd_window", ctypes.byref(cfg), 3, good, good, good, None,
                        None, None, None, good, st) == 1
    assert kta.raw_call("kta_hybrid_fwd_window", ctypes.byref(cfg), 1, good, good, good, None,
                        None, None, None, good, st) == 2
    assert kta.raw_call("kta_hybrid_fwd_window", ctypes.byref(cfg), 0, good, good, good, None,
                        None, ctypes.c_void_p(0x10004), None, good, st) == 3
    # state composition: sizes and aliasing
    assert kta.raw_call("kta_state_affine", good, good, None, good, 0, 8, st) == 1
    assert kta.raw_call("kta_state_affine", good, ctypes.c_void_p(0x20000), None, good, 1, 8,
                        st) == 1
