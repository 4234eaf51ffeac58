"""GPU test of kta_gla_chunk_fwd_noalloc, the GLA entry point that allocates no device memory.

It exists for callers that cannot allocate device memory while they run (a real-time rollout loop
that forbids allocation once started, or a process whose device memory belongs to another
allocator's pool): it runs the chunked GLA kernels with their segment workspace in a fixed
device array instead of memory obtained with cudaMalloc. This file is named to be collected last,
so that a run stopping at the first failure has run every other test first; it also passes on its
own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from hybrid_linear_temporal_kta_b200 import synth

pytestmark = pytest.mark.gpu

BF16_TOL = 1e-2


@pytest.fixture(scope="module")
def kta():
    from hybrid_linear_temporal_kta_b200 import build
    build.build()
    from hybrid_linear_temporal_kta_b200 import kta as mod
    return mod


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _noalloc(kta, q, k, v, alpha, S0, S_out, o, chunk):
    B, N, H, d = q.shape
    shape = kta.Shape(B, 1, N, d, kta.BF16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return kta.raw_call("kta_gla_chunk_fwd_noalloc", _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                        _ptr(S0), _ptr(S_out), _ptr(o), shape, H, H, chunk, ctypes.c_float(1.0),
                        stream)


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_noalloc_matches_allocating_entry_point_on_two_calls(kta):
    """Same kernels and segment plan as kta_gla_chunk_fwd, so the results are bit-identical; two
    calls in a row (the second finds the first call's scratch contents), and each is also checked
    against the oracle."""
    import oracle

    cases = [
        # (B, N, H, d, chunk): both use many segments, so the scratch array is in use
        (1, 20000, 2, 128, 64),
        (2, 9000, 1, 64, 32),
    ]
    for i, (B, N, H, d, chunk) in enumerate(cases):
        w = synth.HYBRID_BF16.replace(d=d, n_swa=0, n_dswa=0, n_gla=H, chunk=chunk)
        x = synth.make_inputs(w, N=N, B=B, seed_base=7000 + 10 * i)
        q, k, v, a = (x[n].cuda() for n in ("q", "k", "v", "alpha"))
        S0 = torch.randn(B, H, d, d, device="cuda", dtype=torch.float32)
        o_ref, S_ref = kta.gla_chunk_fwd(q, k, v, a, chunk=chunk, S0=S0, return_state=True)
        o = torch.full_like(q, float("nan"))
        S_out = torch.full_like(S_ref, float("nan"))
        st = _noalloc(kta, q, k, v, a, S0, S_out, o, chunk)
        assert st == 0, kta.last_error()
        torch.cuda.synchronize()
        kta.device_status()
        assert torch.equal(o, o_ref)
        assert torch.equal(S_out, S_ref)
        ref, Sref = oracle.gla(x["q"], x["k"], x["v"], x["alpha"], S0=S0.cpu())
        assert _rel(o, torch.from_numpy(ref)) <= BF16_TOL
        assert _rel(S_out, torch.from_numpy(Sref)) <= BF16_TOL


def test_noalloc_largest_segment_workspace_fits_and_matches(kta):
    # The segment planner aims at one wave of three CTAs per SM: 221 sequence-heads of d = 128
    # get two segments each, the largest workspace any plan asks for (221 x 2 x (128^2 + 128) x 4
    # bytes = 29.2 MB), which fits the 32 MiB array, so the refusal path is a guard that current
    # plans do not reach.
    B, N, H, d = 13, 128, 17, 128
    w = synth.HYBRID_BF16.replace(d=d, n_swa=0, n_dswa=0, n_gla=H, chunk=64)
    x = synth.make_inputs(w, N=N, B=B, seed_base=7100)
    q, k, v, a = (x[n].cuda() for n in ("q", "k", "v", "alpha"))
    o_ref = kta.gla_chunk_fwd(q, k, v, a, chunk=64)
    o = torch.full_like(q, float("nan"))
    st = _noalloc(kta, q, k, v, a, None, None, o, 64)
    assert st == 0, kta.last_error()
    torch.cuda.synchronize()
    kta.device_status()
    assert torch.equal(o, o_ref)


def test_noalloc_allocates_no_device_memory_after_warm_up(kta):
    """The property the entry point exists for: once a warm-up call has run, a call with a
    shape and stream the allocating path has never seen leaves the device's free memory
    unchanged (the allocating entry point would grow its per-stream workspace here)."""
    B, N, H, d = 1, 30000, 3, 128
    w = synth.HYBRID_BF16.replace(d=d, n_swa=0, n_dswa=0, n_gla=H, chunk=64)
    x = synth.make_inputs(w, N=N, B=B, seed_base=7200)
    q, k, v, a = (x[n].cuda() for n in ("q", "k", "v", "alpha"))
    o = torch.empty_like(q)
    st = _noalloc(kta, q[:, :640], k[:, :640], v[:, :640], a[:, :640], None, None, o[:, :640],
                  64)  # warm-up on a small shape
    assert st == 0, kta.last_error()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    free0, _ = torch.cuda.mem_get_info()
    with torch.cuda.stream(side):
        st = _noalloc(kta, q, k, v, a, None, None, o, 64)
    assert st == 0, kta.last_error()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    kta.device_status()
    assert free1 == free0
