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
