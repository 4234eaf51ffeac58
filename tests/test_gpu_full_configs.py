"""Parity at the full sizes of the streaming workload (240 frames of 880 tokens, one frame per
call) and of the largest length-sweep point (256 frames of 1024 tokens, 262,144 tokens, plus the
full frame-causal baseline), in the launch configurations bench.py times.

The inputs are drawn on the device (synth.make_inputs_device, the same recipe). Checks:
- the rollout equals the full-sequence forward on every head (a property that holds at any
  size: the softmax heads bit for bit, the linear heads within the bf16 bound);
- the fp64 oracle on whole GLA heads (their state depends on every earlier token);
- the oracle on sampled softmax rows, each evaluated on the slice of frames its window can
  see (frames f - (W-1) dil .. f): the window predicate depends only on frame gaps, so the slice
  gives the same result as the whole sequence.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from hybrid_linear_temporal_kta_b200 import synth

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

BF16_TOL = 1e-2


@pytest.fixture(scope="module")
def kta():
    from hybrid_linear_temporal_kta_b200 import build
    build.build()
    from hybrid_linear_temporal_kta_b200 import kta as mod
    return mod


def rel(got, ref):
    got = np.asarray(got, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def head_cpu(t, h):
    """[1, N, H, d] device tensor -> [1, N, 1, d] float32 host array of head h."""
    return t[:, :, h:h + 1].float().cpu().numpy()


def check_softmax_rows(o, q, k, v, w, h, frames, W, dil, dilated, rows_per_frame=6, seed=0):
    """Oracle on sampled rows of head h for the given query frames, on window slices."""
    P = w.P
    rng = np.random.default_rng(seed)
    span = (W - 1) * dil
    for f in frames:
        lo = max(0, f - span)
        sl = slice(lo * P, (f + 1) * P)
        qs, ks, vs = (head_cpu(t[:, sl], h) for t in (q, k, v))
        local = np.unique(np.concatenate([[0, P - 1], rng.integers(0, P, rows_per_frame)]))
        rows = (f - lo) * P + local
        if dilated:
            ref = oracle.dswa(qs, ks, vs, P, W, dil, w.scale_softmax, rows=rows)
        else:
            ref = oracle.swa(qs, ks, vs, P, W, w.scale_softmax, rows=rows)
        got = o[0, f * P + local, h].float().cpu().numpy()
        e = rel(got, ref[0, rows, 0])
        assert e <= BF16_TOL, f"head {h} frame {f}: relative L2 error {e:.3e}"


def check_gla_head(o, x, h, hg, chunk_tol=BF16_TOL):
    """Whole GLA head h (gate index hg) against the fp64 recurrence."""
    q, k, v = (head_cpu(x[n], h) for n in ("q", "k", "v"))
    a = x["alpha"][:, :, hg:hg + 1].cpu().numpy()
    ref, _ = oracle.gla(q, k, v, a)
    e = rel(o[:, :, h:h + 1].float().cpu().numpy(), ref)
    assert e <= chunk_tol, f"GLA head {h}: relative L2 error {e:.3e}"


def test_stream_rollout_full_size(kta):
    w = synth.STREAM_BF16
    x = synth.make_inputs_device(w, seed=w.seed_base)
    cfg = kta.cfg_from_workload(w)
    full = kta.hybrid_fwd(cfg, x["q"], x["k"], x["v"], x["alpha"])
    st = kta.Stream(cfg)
    roll = torch.empty_like(full)
    P = w.P
    for f in range(w.F):
        sl = slice(f * P, (f + 1) * P)
        st.step(x["q"][:, sl], x["k"][:, sl], x["v"][:, sl], x["alpha"][:, sl], out=roll[:, sl])
    torch.cuda.synchronize()
    kta.device_status()
    assert st.frame == w.F
    st.close()
    ns = w.n_swa + w.n_dswa
    # softmax heads: a one-frame launch splits each query tile's key range over the CTA's two
    # accumulators, the full pass pairs query tiles instead, so the two agree to bf16 rounding;
    # the last (ragged) tile of every frame is split in both, so its rows are bit-identical
    for h in range(ns):
        e = rel(roll[:, :, h].float().cpu().numpy(), full[:, :, h].float().cpu().numpy())
        assert e <= BF16_TOL, f"stream vs full, softmax head {h}: {e:.3e}"
    last = (P - 1) // 128 * 128
    r_roll = roll[:, :, :ns].reshape(roll.shape[0], w.F, P, ns, -1)[:, :, last:]
    r_full = full[:, :, :ns].reshape(full.shape[0], w.F, P, ns, -1)[:, :, last:]
    assert torch.equal(r_roll, r_full)
    for h in range(ns, w.H):
        e = rel(roll[:, :, h].float().cpu().numpy(), full[:, :, h].float().cpu().numpy())
        assert e <= BF16_TOL, f"stream vs full, head {h}: {e:.3e}"
    # oracle: two whole GLA heads, sampled rows of one SWA and one DSWA head
    for h in (ns, w.H - 1):
        check_gla_head(roll, x, h, h - ns)
    frames = [0, 1, 2, 9, 120, w.F - 1]
    check_softmax_rows(roll, x["q"], x["k"], x["v"], w, 0, frames, w.W_swa, 1, dilated=False)
    check_softmax_rows(roll, x["q"], x["k"], x["v"], w, w.n_swa, frames, w.W_dswa, w.dil,
                       dilated=True, seed=1)


def test_sweep_largest_point_and_full_causal_baseline(kta):
    w = synth.sweep_workload(256)
    x = synth.make_inputs_device(w, seed=w.seed_base + 256)
    cfg = kta.cfg_from_workload(w)
    o = kta.hybrid_fwd(cfg, x["q"], x["k"], x["v"], x["alpha"])
    torch.cuda.synchronize()
    kta.device_status()
    ns = w.n_swa + w.n_dswa
    frames = [0, 3, 100, w.F - 1]
    check_softmax_rows(o, x["q"], x["k"], x["v"], w, 1, frames, w.W_swa, 1, dilated=False)
    check_softmax_rows(o, x["q"], x["k"], x["v"], w, w.n_swa + 2, frames, w.W_dswa, w.dil,
                       dilated=True, seed=2)
    check_gla_head(o, x, ns + 3, 3)
    # the full frame-causal baseline (window = every earlier frame) on one head
    full = kta.swa_fwd(x["q"], x["k"], x["v"], P=w.P, W=w.F, heads=(5, 6))
    torch.cuda.synchronize()
    kta.device_status()
    for f in (0, 37, w.F - 1):
        check_softmax_rows(full, x["q"], x["k"], x["v"], w, 5, [f], w.F, 1, dilated=False,
                           rows_per_frame=3, seed=3 + f)
    assert math.isfinite(float(full[:, :, 5].float().abs().max()))
