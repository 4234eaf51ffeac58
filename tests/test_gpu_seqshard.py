"""The sequence-sharded hybrid forward on one GPU: its ranks emulated one after another in one
process (seqshard.emulate_ranks; no rank waits on another), with the library's kernels.
- At the full 21-frame x 1,560-token layer split over 3 and 4 ranks: softmax heads bit-identical
  to the single-call forward (same key tiles in the same order), GLA heads against the fp64 oracle
  over the whole sequence.
- A small case of every GLA form (vector, delta, decayed-erase delta) against the oracle.
- kta_hybrid_fwd_window's argument checks."""
import numpy as np
import pytest
import torch

import oracle
from hybrid_linear_temporal_kta_b200 import seqshard, synth

pytestmark = pytest.mark.gpu

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


def shard_cfg(w, gla_delta=0):
    return seqshard.ShardCfg(F=w.F, P=w.P, d=w.d, n_swa=w.n_swa, n_dswa=w.n_dswa, n_gla=w.n_gla,
                             W_swa=w.W_swa, W_dswa=w.W_dswa, dil=w.dil, gla_delta=gla_delta,
                             chunk=w.chunk)


@pytest.mark.parametrize("R", [3, 4])
def test_full_layer_split_over_ranks(kta, R):
    w = synth.HYBRID_BF16
    x = synth.make_inputs_device(w, seed=w.seed_base + 50)
    full = kta.hybrid_fwd(kta.cfg_from_workload(w), x["q"], x["k"], x["v"], x["alpha"])
    o = seqshard.emulate_ranks(shard_cfg(w), R, x["q"], x["k"], x["v"], x["alpha"],
                               ops=seqshard.KtaOps())
    torch.cuda.synchronize()
    kta.device_status()
    ns = w.n_swa + w.n_dswa
    assert torch.equal(o[:, :, :ns], full[:, :, :ns])
    for h in (ns, w.H - 1):
        q, k, v = (x[n][:, :, h:h + 1].float().cpu().numpy() for n in ("q", "k", "v"))
        a = x["alpha"][:, :, h - ns:h - ns + 1].cpu().numpy()
        ref, _ = oracle.gla(q, k, v, a)
        assert rel(o[:, :, h:h + 1].float().cpu().numpy(), ref) <= BF16_TOL


@pytest.mark.parametrize("gla_delta", [0, 1, 2])
def test_small_case_every_gla_form(kta, gla_delta):
    w = synth.HYBRID_BF16.replace(name="shard_small", F=9, P=150, n_swa=1, n_dswa=1, n_gla=2,
                                  W_swa=2, W_dswa=3, dil=2, gla_delta=bool(gla_delta))
    x = synth.make_inputs(w, seed_base=77 + gla_delta)
    dev = {n: (None if t is None else t.cuda()) for n, t in x.items()}
    c = shard_cfg(w, gla_delta)
    o = seqshard.emulate_ranks(c, 4, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"],
                               ops=seqshard.KtaOps())
    torch.cuda.synchronize()
    kta.device_status()
    ref, _ = oracle.hybrid(x["q"], x["k"], x["v"], x["alpha"], x["beta"], P=w.P, n_swa=w.n_swa,
                           n_dswa=w.n_dswa, n_gla=w.n_gla, W_swa=w.W_swa, W_dswa=w.W_dswa,
                           dil=w.dil, gla_delta=gla_delta, scale_softmax=w.scale_softmax)
    got = o.float().cpu().numpy()
    for h in range(w.H):
        assert rel(got[:, :, h], ref[:, :, h]) <= BF16_TOL, f"head {h}"


def test_window_argument_checks(kta):
    cfg = kta.hybrid_cfg(B=2, F=3, P=16, d=64, n_swa=1, n_dswa=0, n_gla=0)
    q = torch.zeros((2, 32, 1, 64), device="cuda", dtype=torch.bfloat16)
    kv = torch.zeros((2, 48, 1, 64), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(kta.KtaError):      # f0 > 0 needs one sequence
        kta.hybrid_fwd_window(cfg, 1, q, kv, kv)
    cfg1 = kta.hybrid_cfg(B=1, F=3, P=16, d=64, n_swa=1, n_dswa=0, n_gla=0)
    with pytest.raises(kta.KtaError):      # f0 must be < F
        kta.hybrid_fwd_window(cfg1, 3, q[:1], kv[:1], kv[:1])
    A = torch.eye(8, device="cuda").expand(3, 8, 8).contiguous()
    X = torch.randn((3, 8, 8), device="cuda")
    Y = kta.state_affine(A, X, X)
    torch.cuda.synchronize()
    assert torch.allclose(Y, 2 * X)


def test_ranks_with_one_frame_and_fp32(kta):
    """More ranks than the halo's worth of frames per rank (every rank holds one or two frames,
    halos span up to four predecessors), in the fp32 reference mode."""
    w = synth.TINY_F32.replace(name="shard_f32", F=7, P=20, d=32, n_swa=1, n_dswa=1, n_gla=1,
                               W_swa=2, W_dswa=3, dil=2)
    x = synth.make_inputs(w, seed_base=5)
    dev = {n: (None if t is None else t.cuda()) for n, t in x.items()}
    c = shard_cfg(w)
    c.chunk = w.chunk
    o = seqshard.emulate_ranks(c, 5, dev["q"], dev["k"], dev["v"], dev["alpha"],
                               ops=seqshard.KtaOps())
    torch.cuda.synchronize()
    kta.device_status()
    ref, _ = oracle.hybrid(x["q"], x["k"], x["v"], x["alpha"], None, P=w.P, n_swa=1, n_dswa=1,
                           n_gla=1, W_swa=2, W_dswa=3, dil=2, scale_softmax=w.scale_softmax)
    got = o.float().cpu().numpy()
    for h in range(w.H):
        assert rel(got[:, :, h], ref[:, :, h]) <= 1e-4, f"head {h}"


@pytest.mark.parametrize("d,N", [(128, 3000), (64, 777), (32, 1)])
def test_gla_transition_equals_state_map_from_identity(kta, d, N):
    """kta_gla_transition (the diagonal of gate products) equals the oracle's transition of the
    run: its end state from the identity with v = 0; exact zeros in the gates give 0."""
    import numpy as np

    import oracle
    rng = np.random.default_rng(11)
    B, H = 2, 3
    a = rng.uniform(0.97, 0.9999, size=(B, N, H, d)).astype(np.float32)
    a[0, N // 2, 1, :5] = 0.0
    q = np.zeros((B, N, H, d), dtype=np.float32)
    eye = np.broadcast_to(np.eye(d), (B, H, d, d)).copy()
    _, Tref = oracle.gla(q, q, q, a, S0=eye)
    T = kta.gla_transition(torch.from_numpy(a).cuda())
    torch.cuda.synchronize()
    kta.device_status()
    got = T.double().cpu().numpy()
    assert np.all(got[0, 1, np.arange(5), np.arange(5)] == 0.0)
    off = ~np.eye(d, dtype=bool)
    assert np.all(got[..., off] == 0.0)
    err = np.abs(got - Tref).max() / np.abs(Tref).max()
    assert err < 1e-4, err
