"""GPU parity of the bf16 tensor-core backward of the softmax heads (kta_softmax_fwd_lse +
kta_softmax_bwd_bf16) against the fp64 oracle's reverse mode: dq, dk, dv within the bf16 bound
(relative L2 <= 1e-2 per head), on ragged 128-row tiles, SWA and DSWA windows, head ranges of a
wider tensor, both head dims; the forward's row log-sum-exp against a direct fp64 evaluation."""
import numpy as np
import pytest
import torch

import oracle

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


def bf16(rng, shape):
    t = torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(torch.bfloat16)
    return t, t.float().numpy()


@pytest.mark.parametrize("d,F,P,W,dil,heads,Htot", [
    (128, 5, 200, 2, 1, (1, 3), 3),     # SWA, ragged second tile
    (64, 7, 130, 3, 2, (0, 2), 2),      # DSWA, 2-row tail tile
    (128, 4, 96, 8, 1, (0, 1), 1),      # one partial tile per frame, window past the start
    (128, 9, 256, 2, 3, (2, 4), 4),     # DSWA, whole tiles
    (128, 12, 16, 4, 2, (0, 2), 2),     # frames shorter than a tile: the forward packs several
    (64, 10, 8, 3, 1, (1, 2), 2),       # frames into one key tile
])
def test_bf16_backward_matches_oracle(kta, d, F, P, W, dil, heads, Htot):
    rng = np.random.default_rng(d + F + P + W)
    B, N = 2, F * P
    (q, qh), (k, kh), (v, vh), (do, doh) = (bf16(rng, (B, N, Htot, d)) for _ in range(4))
    q, k, v, do = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    scale = d ** -0.5
    o, lse = kta.softmax_fwd_lse(q, k, v, P=P, W=W, dil=dil, heads=heads)
    dq, dk, dv = kta.softmax_bwd_bf16(q, k, v, o, lse, do, P=P, W=W, dil=dil, heads=heads)
    torch.cuda.synchronize()
    kta.device_status()
    ref = oracle.softmax_bwd(qh, kh, vh, doh, P, W, scale, dil=dil, dilated=dil > 1, heads=heads)
    h0, h1 = heads
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        gg = g.float().cpu().numpy()
        for h in range(h0, h1):
            e = rel(gg[:, :, h], r[:, :, h])
            assert e <= BF16_TOL, f"{name} head {h}: relative L2 error {e:.3e}"
        assert np.all(gg[:, :, :h0] == 0) and np.all(gg[:, :, h1:] == 0)


def test_forward_lse_matches_direct_evaluation(kta):
    rng = np.random.default_rng(3)
    B, F, P, H, d, W, dil = 1, 6, 150, 2, 64, 3, 2
    N = F * P
    (q, qh), (k, kh), (v, _) = (bf16(rng, (B, N, H, d)) for _ in range(3))
    o, lse = kta.softmax_fwd_lse(q.cuda(), k.cuda(), v.cuda(), P=P, W=W, dil=dil)
    torch.cuda.synchronize()
    kta.device_status()
    got = lse.cpu().numpy()
    t = np.arange(N)
    c = (d ** -0.5) / np.log(2.0)
    for h in range(H):
        for row in (0, P - 1, P, 2 * P + 77, N - 1):
            vis = oracle.visible(np.full(N, row), t, P, W, dil, dilated=True)
            x = (qh[0, row, h].astype(np.float64) @ kh[0, vis, h].T.astype(np.float64)) * c
            mx = x.max()
            exp = mx + np.log2(np.exp2(x - mx).sum())
            assert abs(got[0, h, row] - exp) < 1e-3, (h, row)
    # the output of this entry point equals the plain forward's
    o2 = kta.dswa_fwd(q.cuda(), k.cuda(), v.cuda(), P=P, W=W, dil=dil)
    torch.cuda.synchronize()
    assert torch.equal(o, o2)


def test_bf16_backward_argument_checks(kta):
    q = torch.zeros((1, 64, 1, 32), device="cuda", dtype=torch.bfloat16)   # d = 32: unsupported
    lse = torch.zeros((1, 1, 64), device="cuda")
    with pytest.raises(kta.KtaError):
        kta.softmax_bwd_bf16(q, q, q, q, lse, q, P=16, W=2)
