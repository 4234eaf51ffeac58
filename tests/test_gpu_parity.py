"""GPU parity: every C-ABI entry point against the fp64 CPU oracle on the same seeded inputs.

Tolerances (relative L2 error per output tensor, per head): 1e-2 for the bf16 path, 1e-4 for
the fp32 reference mode. Masks are checked bit-exactly with probe inputs. Sizes span several
query/key tiles and chunks with ragged tails; the full-size workloads are checked on sampled
rows (softmax heads) and on sampled heads (delta rule).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from hybrid_linear_temporal_kta_b200 import synth

pytestmark = pytest.mark.gpu

BF16_TOL = 1e-2
F32_TOL = 1e-4


@pytest.fixture(scope="module")
def kta():
    from hybrid_linear_temporal_kta_b200 import build
    build.build()
    from hybrid_linear_temporal_kta_b200 import kta as mod
    return mod


def dev(x):
    return None if x is None else x.cuda()


def rel(got, ref):
    got = np.asarray(got, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def assert_heads_close(got, ref, heads, tol, rows=None, what=""):
    g = got.float().cpu().numpy().astype(np.float64)
    for h in heads:
        a, b = (g[:, :, h], ref[:, :, h]) if rows is None else (g[:, rows, h], ref[:, rows, h])
        e = rel(a, b)
        assert e <= tol, f"{what} head {h}: relative L2 error {e:.3e} > {tol}"


# --------------------------------------------------------------------------- fp32 reference mode


def test_tiny_f32_hybrid_matches_oracle(kta):
    w = synth.TINY_F32
    x = synth.make_inputs(w)
    o = kta.hybrid_fwd(kta.cfg_from_workload(w), dev(x["q"]), dev(x["k"]), dev(x["v"]),
                       dev(x["alpha"]))
    kta.device_status()
    ref, _ = oracle.hybrid(x["q"], x["k"], x["v"], x["alpha"], None, P=w.P, n_swa=w.n_swa,
                           n_dswa=w.n_dswa, n_gla=w.n_gla, W_swa=w.W_swa, W_dswa=w.W_dswa,
                           dil=w.dil, scale_softmax=w.scale_softmax)
    assert_heads_close(o, ref, range(w.H), F32_TOL, what="tiny f32 hybrid")


@pytest.mark.parametrize("d", [32, 64, 128])
def test_f32_linear_branches_with_state(kta, d):
    B, N, H = 2, 77, 2
    w = synth.TINY_F32.replace(d=d, n_swa=0, n_dswa=0, n_gla=H)
    x = synth.make_inputs(w, N=N, B=B)
    S0 = torch.from_numpy(np.random.default_rng(7).standard_normal((B, H, d, d)).astype(np.float32))
    o, S = kta.gla_chunk_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["alpha"]), scale=0.5,
                             S0=dev(S0), return_state=True)
    ref, Sref = oracle.gla(x["q"], x["k"], x["v"], x["alpha"], scale=0.5, S0=S0)
    assert_heads_close(o, ref, range(H), F32_TOL, what="f32 gla")
    assert rel(S.cpu().numpy(), Sref) < F32_TOL
    wd = w.replace(gla_delta=True)
    xd = synth.make_inputs(wd, N=N, B=B)
    o, S = kta.gla_delta_fwd(dev(xd["q"]), dev(xd["k"]), dev(xd["v"]), dev(xd["alpha"]),
                             dev(xd["beta"]), S0=dev(S0), return_state=True)
    ref, Sref = oracle.delta(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], S0=S0)
    assert_heads_close(o, ref, range(H), F32_TOL, what="f32 delta")
    assert rel(S.cpu().numpy(), Sref) < F32_TOL
    o, S = kta.gla_delta_fwd(dev(xd["q"]), dev(xd["k"]), dev(xd["v"]), dev(xd["alpha"]),
                             dev(xd["beta"]), S0=dev(S0), return_state=True, erase_decayed=True)
    ref, Sref = oracle.delta(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], S0=S0,
                             erase_decayed=True)
    assert_heads_close(o, ref, range(H), F32_TOL, what="f32 decayed-erase delta")
    assert rel(S.cpu().numpy(), Sref) < F32_TOL


@pytest.mark.parametrize("W,dil", [(1, 1), (2, 1), (3, 2), (9, 1)])
def test_f32_softmax_branches(kta, W, dil):
    w = synth.TINY_F32.replace(F=7, P=19, n_swa=0, n_dswa=2, n_gla=0)
    x = synth.make_inputs(w, B=2)
    q, k, v = dev(x["q"]), dev(x["k"]), dev(x["v"])
    o = kta.dswa_fwd(q, k, v, P=w.P, W=W, dil=dil, scale=0.3)
    ref = oracle.dswa(x["q"], x["k"], x["v"], w.P, W, dil, 0.3)
    assert_heads_close(o, ref, range(2), F32_TOL, what="f32 dswa")


# --------------------------------------------------------------------------- bf16 softmax


SOFTMAX_CASES = [
    # d, B, F, P, W, dil      (P = 200: one full 128-row tile and a 72-row tail per frame)
    (128, 2, 6, 200, 3, 1),
    (128, 1, 9, 200, 4, 3),
    (64, 2, 5, 128, 2, 2),
    (128, 1, 4, 33, 20, 1),   # W >= F: full frame-causal attention
    (64, 1, 7, 300, 1, 1),    # own frame only
    (128, 1, 13, 96, 3, 5),   # dilation larger than the window
    # frames shorter than a key tile: a packed dilated window puts many frames in one tile
    (128, 1, 12, 8, 4, 2),
    (64, 2, 10, 16, 5, 2),
    (128, 1, 30, 104, 8, 2),  # some packed tiles cross three frames
    (128, 1, 6, 1, 3, 2),     # one-token frames (not packed: P is not a multiple of 8)
]


@pytest.mark.parametrize("d,B,F,P,W,dil", SOFTMAX_CASES)
def test_bf16_softmax_matches_oracle(kta, d, B, F, P, W, dil):
    w = synth.HYBRID_BF16.replace(F=F, P=P, d=d, n_swa=0, n_dswa=3, n_gla=0)
    x = synth.make_inputs(w, B=B)
    q, k, v = dev(x["q"]), dev(x["k"]), dev(x["v"])
    scale = 1 / math.sqrt(d)
    if dil == 1:
        o = kta.swa_fwd(q, k, v, P=P, W=W)
        ref = oracle.swa(x["q"], x["k"], x["v"], P, W, scale)
    else:
        o = kta.dswa_fwd(q, k, v, P=P, W=W, dil=dil)
        ref = oracle.dswa(x["q"], x["k"], x["v"], P, W, dil, scale)
    kta.device_status()
    assert_heads_close(o, ref, range(3), BF16_TOL, what=f"softmax d={d} P={P} W={W} dil={dil}")


def test_bf16_softmax_head_range_leaves_other_heads(kta):
    w = synth.HYBRID_BF16.replace(F=3, P=150, n_swa=0, n_dswa=4, n_gla=0)
    x = synth.make_inputs(w)
    q, k, v = dev(x["q"]), dev(x["k"]), dev(x["v"])
    out = torch.full_like(q, 7.0)
    kta.dswa_fwd(q, k, v, P=w.P, W=2, dil=1, heads=(1, 3), out=out)
    ref = oracle.swa(x["q"], x["k"], x["v"], w.P, 2, w.scale_softmax)
    assert_heads_close(out, ref, (1, 2), BF16_TOL)
    assert torch.all(out[:, :, 0] == 7.0) and torch.all(out[:, :, 3] == 7.0)


@pytest.mark.parametrize("W,dil,code", [(3, 1, "frame"), (4, 3, "frame"), (2, 1, "token"),
                                        (3, 2, "token")])
def test_bf16_mask_probe_is_bit_exact(kta, W, dil, code):
    """q = k = 0 gives equal weight to every visible key; v = one-hot(code of key) makes the zero
    pattern of o exactly the set of codes among visible keys."""
    F, P, d = 11, 200, 128
    N = F * P
    q = torch.zeros(1, N, 1, d, dtype=torch.bfloat16)
    v = torch.zeros(1, N, 1, d, dtype=torch.bfloat16)
    s = np.arange(N)
    col = (s // P) if code == "frame" else (s % P) % d
    v[0, torch.from_numpy(s), 0, torch.from_numpy(col)] = 1.0
    o = kta.dswa_fwd(dev(q), dev(q), dev(v), P=P, W=W, dil=dil)
    got = o[0, :, 0].float().cpu().numpy()
    ref = oracle.dswa(q, q, v, P, W, dil, 1.0)[0, :, 0]
    assert np.array_equal(got != 0, ref != 0)
    assert np.max(np.abs(got - ref)) <= 2.0 ** -8 * np.max(np.abs(ref)) + 1e-6


def test_bf16_dswa_equals_swa_on_page_reshape(kta):
    """Page identity: when dil divides F, DSWA equals SWA on the reshape (B, F*L, D) ->
    (B*dil, F/dil*L, D) with frame f in group f mod dil. Both sides run on the GPU."""
    B, F, P, dil, W = 1, 12, 160, 3, 3
    w = synth.HYBRID_BF16.replace(F=F, P=P, n_swa=0, n_dswa=2, n_gla=0)
    x = synth.make_inputs(w, B=B)
    q, k, v = dev(x["q"]), dev(x["k"]), dev(x["v"])
    o = kta.dswa_fwd(q, k, v, P=P, W=W, dil=dil)

    def fwd(t):
        H, d = t.shape[2], t.shape[3]
        return t.reshape(B, F // dil, dil, P, H, d).transpose(1, 2).reshape(B * dil, F // dil * P,
                                                                              H, d).contiguous()

    og = kta.swa_fwd(fwd(q), fwd(k), fwd(v), P=P, W=W)
    back = og.reshape(B, dil, F // dil, P, 2, 128).transpose(1, 2).reshape(B, F * P, 2, 128)
    # the two sides tile the keys differently (per frame vs one span), so they agree to rounding
    for h in range(2):
        assert rel(back[:, :, h].float().cpu().numpy(), o[:, :, h].float().cpu().numpy()) < 2e-3


# --------------------------------------------------------------------------- bf16 linear branches


@pytest.mark.parametrize("d,chunk,N,B,H", [(128, 64, 1000, 2, 2), (128, 32, 777, 1, 3),
                                           (64, 16, 333, 2, 1), (128, 64, 20000, 1, 1),
                                           (64, 64, 64, 1, 2),
                                           # 40 sequence-heads: three segments, folded by the
                                           # output pass itself (no carry launch)
                                           (128, 64, 700, 2, 20),
                                           # one token; one chunk and one token; a partial chunk
                                           (128, 64, 1, 1, 2), (128, 64, 65, 2, 1),
                                           (64, 32, 33, 1, 2), (128, 16, 15, 1, 1)])
def test_bf16_gla_matches_oracle(kta, d, chunk, N, B, H):
    w = synth.HYBRID_BF16.replace(d=d, n_swa=0, n_dswa=0, n_gla=H, chunk=chunk)
    x = synth.make_inputs(w, N=N, B=B)
    S0 = torch.from_numpy(np.random.default_rng(3).standard_normal((B, H, d, d)).astype(np.float32))
    o, S = kta.gla_chunk_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["alpha"]), chunk=chunk,
                             S0=dev(S0), return_state=True)
    kta.device_status()
    ref, Sref = oracle.gla(x["q"], x["k"], x["v"], x["alpha"], S0=S0)
    assert_heads_close(o, ref, range(H), BF16_TOL, what=f"gla d={d} C={chunk} N={N}")
    assert rel(S.cpu().numpy(), Sref) < BF16_TOL


@pytest.mark.parametrize("d,chunk,N,B,H", [(128, 64, 1000, 2, 2), (128, 64, 50, 1, 3),
                                           (128, 64, 9000, 1, 2), (64, 32, 777, 2, 1),
                                           (128, 16, 300, 1, 2), (128, 64, 1, 1, 2)])
def test_bf16_gla_end_state_only_matches_full_forward(kta, d, chunk, N, B, H):
    """kta_gla_chunk_state (state pass + segment fold, no outputs) against the full forward's
    S_out and the oracle, with a start state; one segment (N = 50) and many (N = 9000)."""
    w = synth.HYBRID_BF16.replace(d=d, n_swa=0, n_dswa=0, n_gla=H, chunk=chunk)
    x = synth.make_inputs(w, N=N, B=B)
    S0 = torch.from_numpy(np.random.default_rng(4).standard_normal((B, H, d, d)).astype(np.float32))
    q, k, v, a = dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["alpha"])
    S = kta.gla_chunk_state(k, v, a, chunk=chunk, S0=dev(S0))
    _, S_full = kta.gla_chunk_fwd(q, k, v, a, chunk=chunk, S0=dev(S0), return_state=True)
    kta.device_status()
    assert torch.isfinite(S).all()
    assert rel(S.cpu().numpy(), S_full.cpu().numpy()) < 1e-5
    _, Sref = oracle.gla(x["q"], x["k"], x["v"], x["alpha"], S0=S0)
    assert rel(S.cpu().numpy(), Sref) < BF16_TOL


def small_gates(kind, shape, seed):
    """Forget gates far below the usual range (all valid: alpha in [0, 1))."""
    rng = np.random.default_rng(seed)
    if kind == "sigmoid(N(-3,1))":
        a = 1.0 / (1.0 + np.exp(-(rng.standard_normal(shape) - 3.0)))
    elif kind == "uniform[1e-4,0.1]":
        a = rng.uniform(1e-4, 0.1, size=shape)
    else:  # ordinary gates with exact zeros, 1e-30 and 1e-12 sprinkled in
        a = rng.uniform(0.3, 0.999, size=shape)
        flat = a.reshape(-1)
        idx = rng.choice(flat.size, size=flat.size // 20, replace=False)
        flat[idx[0::3]], flat[idx[1::3]], flat[idx[2::3]] = 0.0, 1e-30, 1e-12
    return torch.from_numpy(a.astype(np.float32))


@pytest.mark.parametrize("kind", ["sigmoid(N(-3,1))", "uniform[1e-4,0.1]", "zeros-and-tiny"])
@pytest.mark.parametrize("d,chunk,N", [(128, 64, 5 * 64 + 7), (128, 32, 4 * 32 + 19),
                                       (128, 16, 4 * 16 + 5), (64, 64, 4 * 64 + 33),
                                       (64, 32, 6 * 32), (64, 16, 5 * 16 + 1),
                                       (128, 64, 9000)])
def test_bf16_gla_small_gates_match_oracle(kta, kind, d, chunk, N):
    """Gates near 0 (the GLA paragraph's forget gate ranges over (0, 1)): every output finite and
    within the bf16 bound of the oracle, with a start state, several chunks, a ragged tail and
    (N = 9000) several segments joined by the carry pass."""
    B, H = 2, 2
    w = synth.HYBRID_BF16.replace(d=d, n_swa=0, n_dswa=0, n_gla=H, chunk=chunk)
    x = synth.make_inputs(w, N=N, B=B)
    alpha = small_gates(kind, (B, N, H, d), seed=7 * d + chunk)
    S0 = torch.from_numpy(np.random.default_rng(5).standard_normal((B, H, d, d)).astype(np.float32))
    o, S = kta.gla_chunk_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(alpha), chunk=chunk,
                             S0=dev(S0), return_state=True)
    kta.device_status()
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    ref, Sref = oracle.gla(x["q"], x["k"], x["v"], alpha, S0=S0)
    assert_heads_close(o, ref, range(H), BF16_TOL, what=f"gla {kind} d={d} C={chunk} N={N}")
    assert rel(S.cpu().numpy(), Sref) < BF16_TOL


@pytest.mark.parametrize("d,N,B,H,with_s0", [(128, 300, 2, 2, True), (64, 1000, 1, 3, False),
                                             (128, 4096, 1, 1, True), (128, 50, 3, 1, True),
                                             (64, 640, 2, 5, True),
                                             # one token; a chunk less one; a chunk and one
                                             (128, 1, 1, 1, True), (128, 63, 2, 1, True),
                                             (64, 65, 1, 2, False)])
def test_bf16_delta_matches_oracle(kta, d, N, B, H, with_s0):
    w = synth.DELTA_BF16.replace(d=d, n_gla=H)
    x = synth.make_inputs(w, N=N, B=B)
    S0 = (torch.from_numpy(np.random.default_rng(5).standard_normal((B, H, d, d)).astype(np.float32))
          * 0.1 if with_s0 else None)
    o, S = kta.gla_delta_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["alpha"]),
                             dev(x["beta"]), S0=dev(S0), return_state=True)
    kta.device_status()
    ref, Sref = oracle.delta(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S0=S0)
    assert_heads_close(o, ref, range(H), BF16_TOL, what=f"delta d={d} N={N}")
    assert rel(S.cpu().numpy(), Sref) < BF16_TOL


@pytest.mark.parametrize("d,N,B,H,with_s0", [(128, 300, 2, 2, True), (64, 1000, 1, 3, False),
                                             (128, 50, 1, 1, True), (128, 4096, 1, 1, False)])
def test_bf16_decayed_erase_delta_matches_oracle(kta, d, N, B, H, with_s0):
    w = synth.DELTA_BF16.replace(d=d, n_gla=H)
    x = synth.make_inputs(w, N=N, B=B)
    S0 = (torch.from_numpy(np.random.default_rng(6).standard_normal((B, H, d, d)).astype(np.float32))
          * 0.1 if with_s0 else None)
    o, S = kta.gla_delta_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["alpha"]),
                             dev(x["beta"]), S0=dev(S0), return_state=True, erase_decayed=True)
    kta.device_status()
    ref, Sref = oracle.delta(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S0=S0,
                             erase_decayed=True)
    assert_heads_close(o, ref, range(H), BF16_TOL, what=f"decayed-erase delta d={d} N={N}")
    assert rel(S.cpu().numpy(), Sref) < BF16_TOL


# --------------------------------------------------------------------------- hybrid


def test_bf16_hybrid_small_matches_oracle(kta):
    w = synth.HYBRID_BF16.replace(F=6, P=260, n_swa=2, n_dswa=2, n_gla=2, W_swa=2, W_dswa=3, dil=2)
    x = synth.make_inputs(w, B=2)
    o = kta.hybrid_fwd(kta.cfg_from_workload(w, B=2), dev(x["q"]), dev(x["k"]), dev(x["v"]),
                       dev(x["alpha"]))
    kta.device_status()
    ref, _ = oracle.hybrid(x["q"], x["k"], x["v"], x["alpha"], None, P=w.P, n_swa=2, n_dswa=2,
                           n_gla=2, W_swa=2, W_dswa=3, dil=2, scale_softmax=w.scale_softmax)
    assert_heads_close(o, ref, range(w.H), BF16_TOL, what="hybrid small")


def test_bf16_hybrid_delta_heads(kta):
    w = synth.HYBRID_BF16.replace(F=4, P=200, n_swa=1, n_dswa=1, n_gla=2, gla_delta=True)
    x = synth.make_inputs(w)
    o = kta.hybrid_fwd(kta.cfg_from_workload(w), dev(x["q"]), dev(x["k"]), dev(x["v"]),
                       dev(x["alpha"]), dev(x["beta"]))
    ref, _ = oracle.hybrid(x["q"], x["k"], x["v"], x["alpha"], x["beta"], P=w.P, n_swa=1,
                           n_dswa=1, n_gla=2, W_swa=w.W_swa, W_dswa=w.W_dswa, dil=w.dil,
                           gla_delta=True, scale_softmax=w.scale_softmax)
    assert_heads_close(o, ref, range(w.H), BF16_TOL, what="hybrid delta")


def test_bf16_hybrid_decayed_erase_delta_heads(kta):
    w = synth.HYBRID_BF16.replace(F=5, P=180, n_swa=1, n_dswa=1, n_gla=2, gla_delta=2)
    x = synth.make_inputs(w)
    o = kta.hybrid_fwd(kta.cfg_from_workload(w), dev(x["q"]), dev(x["k"]), dev(x["v"]),
                       dev(x["alpha"]), dev(x["beta"]))
    ref, _ = oracle.hybrid(x["q"], x["k"], x["v"], x["alpha"], x["beta"], P=w.P, n_swa=1,
                           n_dswa=1, n_gla=2, W_swa=w.W_swa, W_dswa=w.W_dswa, dil=w.dil,
                           gla_delta=2, scale_softmax=w.scale_softmax)
    assert_heads_close(o, ref, range(w.H), BF16_TOL, what="hybrid decayed-erase delta")


@pytest.mark.slow
def test_hybrid_full_size_sampled(kta):
    """The 32,760-token bf16 hybrid layer (24 heads: 8 SWA, 8 DSWA, 8 GLA) in the launch
    configuration the benchmark times: GLA heads checked in full, softmax heads on sampled rows
    (every frame's first and last row, tile edges, and a seeded 1% of rows)."""
    w = synth.HYBRID_BF16
    x = synth.make_inputs(w)
    o = kta.hybrid_fwd(kta.cfg_from_workload(w), dev(x["q"]), dev(x["k"]), dev(x["v"]),
                       dev(x["alpha"]))
    kta.device_status()
    rows = synth.sample_rows(w.N, w.P, 0.01, seed=11)
    ref, _ = oracle.hybrid(x["q"], x["k"], x["v"], x["alpha"], None, P=w.P, n_swa=w.n_swa,
                           n_dswa=w.n_dswa, n_gla=w.n_gla, W_swa=w.W_swa, W_dswa=w.W_dswa,
                           dil=w.dil, scale_softmax=w.scale_softmax, rows=rows)
    assert_heads_close(o, ref, range(16), BF16_TOL, rows=rows, what="full hybrid softmax")
    assert_heads_close(o, ref, range(16, 24), BF16_TOL, what="full hybrid gla")


@pytest.mark.slow
def test_delta_full_size_sampled_heads(kta):
    """The two-sequence, 65,536-token, 16-head gated delta-rule workload; the oracle checks the
    first two heads of both sequences."""
    w = synth.DELTA_BF16
    x = synth.make_inputs(w)
    o = kta.gla_delta_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["alpha"]), dev(x["beta"]))
    kta.device_status()
    hs = 2
    ref, _ = oracle.delta(x["q"][:, :, :hs], x["k"][:, :, :hs], x["v"][:, :, :hs],
                          x["alpha"][:, :, :hs], x["beta"][:, :, :hs])
    assert_heads_close(o[:, :, :hs], ref, range(hs), BF16_TOL, what="full delta")
    assert torch.isfinite(o.float()).all()


# --------------------------------------------------------------------------- streaming


def _stream_case(dtype="bf16"):
    w = synth.STREAM_BF16.replace(F=9, P=200, n_swa=2, n_dswa=2, n_gla=2, dtype=dtype,
                                  d=128 if dtype == "bf16" else 64)
    return w, synth.make_inputs(w, B=2)


@pytest.mark.parametrize("gla_delta", [1, 2])
def test_stream_rollout_with_delta_heads(kta, gla_delta):
    w = synth.STREAM_BF16.replace(F=7, P=150, n_swa=1, n_dswa=1, n_gla=2, gla_delta=gla_delta)
    x = synth.make_inputs(w, B=2)
    cfg = kta.cfg_from_workload(w, B=2)
    q, k, v, a, be = (dev(x[n]) for n in ("q", "k", "v", "alpha", "beta"))
    full = kta.hybrid_fwd(cfg, q, k, v, a, be)
    st = kta.Stream(cfg)
    outs = []
    for f in range(w.F):
        sl = slice(f * w.P, (f + 1) * w.P)
        outs.append(st.step(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(),
                            a[:, sl].contiguous(), be[:, sl].contiguous()))
    kta.device_status()
    roll = torch.cat(outs, dim=1)
    assert_heads_close(roll, full.float().cpu().numpy().astype(np.float64), range(w.H), BF16_TOL,
                       what="delta stream vs full")
    ref, _ = oracle.hybrid(x["q"], x["k"], x["v"], x["alpha"], x["beta"], P=w.P, n_swa=1,
                           n_dswa=1, n_gla=2, W_swa=w.W_swa, W_dswa=w.W_dswa, dil=w.dil,
                           gla_delta=gla_delta, scale_softmax=w.scale_softmax)
    assert_heads_close(roll, ref, range(w.H), BF16_TOL, what="delta stream vs oracle")
    st.close()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_stream_rollout_matches_full_forward(kta, dtype):
    w, x = _stream_case(dtype)
    cfg = kta.cfg_from_workload(w, B=2)
    q, k, v, a = dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["alpha"])
    full = kta.hybrid_fwd(cfg, q, k, v, a)
    st = kta.Stream(cfg)
    outs = []
    for f in range(w.F):
        sl = slice(f * w.P, (f + 1) * w.P)
        outs.append(st.step(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(),
                            a[:, sl].contiguous()))
    kta.device_status()
    roll = torch.cat(outs, dim=1)
    assert st.frame == w.F
    tol = BF16_TOL if dtype == "bf16" else F32_TOL
    fr = full.float().cpu().numpy().astype(np.float64)
    assert_heads_close(roll, fr, range(w.H), tol, what="stream vs full")
    # softmax heads read identical key tiles in the same order: bit-identical to the full pass
    assert torch.equal(roll[:, :, :4], full[:, :, :4])
    ref, _ = oracle.hybrid(x["q"], x["k"], x["v"], x["alpha"], None, P=w.P, n_swa=2, n_dswa=2,
                           n_gla=2, W_swa=w.W_swa, W_dswa=w.W_dswa, dil=w.dil,
                           scale_softmax=w.scale_softmax)
    assert_heads_close(roll, ref, range(w.H), tol, what="stream vs oracle")
    st.close()


@pytest.mark.parametrize("P", [1, 7, 16, 40, 104])
def test_stream_short_frames_match_full_forward(kta, P):
    """Frames shorter than a key tile: the streamed SWA window is a ring of W slots, so its packed
    tiles (and the dilated window's) span several frames. DSWA heads equal the full forward bit
    for bit; so do SWA heads when P is a multiple of 8 (the ring's frames are then packed into the
    full forward's tiles; otherwise each frame is its own span and the two agree within rounding).
    Every head is within the bf16 bound of the oracle."""
    w = synth.STREAM_BF16.replace(F=14, P=P, n_swa=2, n_dswa=2, n_gla=2, W_swa=5, W_dswa=4, dil=2)
    x = synth.make_inputs(w, B=2)
    cfg = kta.cfg_from_workload(w, B=2)
    q, k, v, a = dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["alpha"])
    full = kta.hybrid_fwd(cfg, q, k, v, a)
    st = kta.Stream(cfg)
    outs = []
    for f in range(w.F):
        sl = slice(f * w.P, (f + 1) * w.P)
        outs.append(st.step(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(),
                            a[:, sl].contiguous()))
    kta.device_status()
    roll = torch.cat(outs, dim=1)
    assert torch.equal(roll[:, :, 2:4], full[:, :, 2:4])
    if P % 8 == 0:
        assert torch.equal(roll[:, :, :2], full[:, :, :2])
    else:
        assert_heads_close(roll, full.float().cpu().numpy().astype(np.float64), range(2), BF16_TOL,
                           what=f"short-frame stream P={P} vs full")
    ref, _ = oracle.hybrid(x["q"], x["k"], x["v"], x["alpha"], None, P=w.P, n_swa=2, n_dswa=2,
                           n_gla=2, W_swa=w.W_swa, W_dswa=w.W_dswa, dil=w.dil,
                           scale_softmax=w.scale_softmax)
    assert_heads_close(roll, ref, range(w.H), BF16_TOL, what=f"short-frame stream P={P}")
    st.close()


def test_stream_save_load_resumes_bit_identically(kta):
    w, x = _stream_case()
    cfg = kta.cfg_from_workload(w, B=2)
    q, k, v, a = dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["alpha"])
    frame = lambda t, f: t[:, f * w.P:(f + 1) * w.P].contiguous()  # noqa: E731
    s1 = kta.Stream(cfg)
    ref = [s1.step(frame(q, f), frame(k, f), frame(v, f), frame(a, f)) for f in range(w.F)]
    s2 = kta.Stream(cfg)
    split = 5
    for f in range(split):
        s2.step(frame(q, f), frame(k, f), frame(v, f), frame(a, f))
    blob = s2.save()
    s2.close()
    s3 = kta.Stream(cfg)
    s3.load(blob)
    assert s3.frame == split
    for f in range(split, w.F):
        o = s3.step(frame(q, f), frame(k, f), frame(v, f), frame(a, f))
        assert torch.equal(o, ref[f])
    s3.reset()
    assert s3.frame == 0
    o0 = s3.step(frame(q, 0), frame(k, 0), frame(v, 0), frame(a, 0))
    assert torch.equal(o0, ref[0])
    with pytest.raises(kta.KtaError):
        bad = kta.Stream(kta.cfg_from_workload(w.replace(W_swa=2), B=2))
        bad.load(blob)
    s1.close()
    s3.close()


# --------------------------------------------------------------------------- health


def test_bounded_wait_timeout_is_reported(kta):
    kta.selftest_wait_timeout(1_000_000)      # ~0.5 ms: a barrier nobody arrives at
    with pytest.raises(kta.KtaError) as e:
        kta.device_status()
    assert e.value.status == 5
    kta.device_status()                       # cleared; the context is still usable
    w = synth.HYBRID_BF16.replace(F=2, P=128, n_swa=1, n_dswa=0, n_gla=0)
    x = synth.make_inputs(w)
    o = kta.swa_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), P=128, W=2)
    kta.device_status()
    assert torch.isfinite(o.float()).all()


def test_repeat_runs_are_bit_identical(kta):
    w = synth.HYBRID_BF16.replace(F=5, P=200, n_swa=1, n_dswa=1, n_gla=1)
    x = synth.make_inputs(w)
    cfg = kta.cfg_from_workload(w)
    args = [dev(x[n]) for n in ("q", "k", "v", "alpha")]
    o1 = kta.hybrid_fwd(cfg, *args)
    o2 = kta.hybrid_fwd(cfg, *args)
    assert torch.equal(o1, o2)


def test_hybrid_and_stream_replay_as_cuda_graphs(kta):
    """The hybrid call (its fork onto two internal streams and join) and a streamed rollout
    (ring gather, one-frame softmax, GLA beside it) captured with torch.cuda.graph and replayed:
    bit-identical to the eager calls."""
    w = synth.STREAM_BF16.replace(F=6, P=200, n_swa=2, n_dswa=2, n_gla=2)
    x = synth.make_inputs(w, B=2)
    cfg = kta.cfg_from_workload(w, B=2)
    q, k, v, a = dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["alpha"])
    ref = kta.hybrid_fwd(cfg, q, k, v, a)
    st = kta.Stream(cfg)
    P = w.P
    frames = [tuple(t[:, f * P:(f + 1) * P].contiguous() for t in (q, k, v, a)) for f in range(w.F)]
    outs = [torch.empty_like(fr[0]) for fr in frames]

    def rollout():
        st.reset()
        for (qf, kf, vf, af), of in zip(frames, outs):
            st.step(qf, kf, vf, af, out=of)

    rollout()  # eager: allocates the library's workspaces and side streams before capture
    torch.cuda.synchronize()
    eager = [o.clone() for o in outs]
    o_graph = torch.empty_like(ref)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        kta.hybrid_fwd(cfg, q, k, v, a, out=o_graph)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g1, g2 = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1):
        kta.hybrid_fwd(cfg, q, k, v, a, out=o_graph)
    with torch.cuda.graph(g2):
        rollout()
    for o in outs:
        o.zero_()
    o_graph.zero_()
    g1.replay()
    g2.replay()
    torch.cuda.synchronize()
    kta.device_status()
    assert torch.equal(o_graph, ref)
    for o, e in zip(outs, eager):
        assert torch.equal(o, e)
    assert st.frame == w.F
    del g1, g2
    st.close()
