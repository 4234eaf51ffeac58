"""GPU parity of the reverse mode (fp32 CUDA-core kernels) against the fp64 oracle's backward.

Every gradient is compared element by element (relative L2 <= 1e-4, the fp32 bound) on seeded
inputs that span several key tiles, checkpoint chunks and a ragged tail; head ranges inside a
wider tensor check that other heads stay untouched.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

F32_TOL = 1e-4


@pytest.fixture(scope="module")
def kta():
    from hybrid_linear_temporal_kta_b200 import build
    build.build()
    from hybrid_linear_temporal_kta_b200 import kta as mod
    return mod


def rel(got, ref):
    got = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def qkv(rng, B, N, H, d, unit_keys=False):
    q = rng.standard_normal((B, N, H, d)).astype(np.float32)
    k = rng.standard_normal((B, N, H, d)).astype(np.float32)
    v = rng.standard_normal((B, N, H, d)).astype(np.float32)
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    return q, k, v


@pytest.mark.parametrize("d,F,P,W,dil,dilated,heads,Htot", [
    (64, 5, 37, 2, 1, False, (0, 2), 2),
    (128, 7, 33, 3, 2, True, (1, 3), 4),
    (32, 4, 96, 4, 1, False, (2, 3), 3),
    (64, 9, 20, 2, 3, True, (0, 1), 2),
    (64, 3, 50, 8, 1, False, (0, 2), 2),   # window wider than the sequence: frame-causal
])
def test_softmax_backward_parity(kta, d, F, P, W, dil, dilated, heads, Htot):
    rng = np.random.default_rng(100 + d + F + P)
    B, N = 2, F * P
    q, k, v = qkv(rng, B, N, Htot, d)
    do = rng.standard_normal((B, N, Htot, d)).astype(np.float32)
    scale = d ** -0.5
    ref = oracle.softmax_bwd(q, k, v, do, P, W, scale, dil=dil, dilated=dilated, heads=heads)
    if dilated:
        got = kta.dswa_bwd(dev(q), dev(k), dev(v), dev(do), P=P, W=W, dil=dil, scale=scale,
                           heads=heads)
    else:
        got = kta.swa_bwd(dev(q), dev(k), dev(v), dev(do), P=P, W=W, scale=scale, heads=heads)
    torch.cuda.synchronize()
    kta.device_status()
    h0, h1 = heads
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        e = rel(g[:, :, h0:h1], r[:, :, h0:h1])
        assert e <= F32_TOL, f"{name}: relative L2 error {e:.3e}"
        gn = g.cpu().numpy()
        assert np.all(gn[:, :, :h0] == 0) and np.all(gn[:, :, h1:] == 0), f"{name} outside heads"


# B * H < 148 splits each sequence into segments (about one CTA per SM, 32-token multiples,
# ragged last segment); the last case has B * H >= 148 and runs one segment per sequence.
@pytest.mark.parametrize("d,N,with_s0,B,Htot,heads", [
    (32, 45, False, 2, 3, (1, 3)), (64, 100, True, 2, 3, (1, 3)), (128, 161, True, 2, 3, (1, 3)),
    (128, 1000, False, 2, 3, (1, 3)), (128, 1000, True, 1, 1, (0, 1)),
    (32, 40, True, 1, 150, (0, 150))])
def test_gla_backward_parity(kta, d, N, with_s0, B, Htot, heads):
    rng = np.random.default_rng(200 + d + N + Htot)
    H = heads[1] - heads[0]
    q, k, v = qkv(rng, B, N, Htot, d)
    k *= d ** -0.5
    alpha = (1.0 / (1.0 + np.exp(-(rng.standard_normal((B, N, H, d)) + 3.0)))).astype(np.float32)
    do = rng.standard_normal((B, N, Htot, d)).astype(np.float32)
    S0 = rng.standard_normal((B, H, d, d)).astype(np.float32) * 0.1 if with_s0 else None
    scale = 0.5
    ref = oracle.gla_bwd(q, k, v, alpha, do, scale=scale, S0=S0, heads=heads)
    got = kta.gla_bwd(dev(q), dev(k), dev(v), dev(alpha), dev(do), scale=scale,
                      S0=None if S0 is None else dev(S0), heads=heads)
    torch.cuda.synchronize()
    kta.device_status()
    h0, h1 = heads
    names = ("dq", "dk", "dv", "dalpha", "dS0")
    for i, (name, g, r) in enumerate(zip(names, got, ref)):
        if i < 3:
            g, r = g[:, :, h0:h1], r[:, :, h0:h1]
        e = rel(g, r)
        assert e <= F32_TOL, f"{name}: relative L2 error {e:.3e}"
    assert torch.all(got[0][:, :, :h0] == 0)


@pytest.mark.parametrize("erase_decayed", [False, True])
@pytest.mark.parametrize("d,N,with_s0", [(32, 70, True), (64, 129, False), (128, 300, True),
                                         (128, 1000, True)])
def test_delta_backward_parity(kta, d, N, with_s0, erase_decayed):
    rng = np.random.default_rng(300 + d + N + int(erase_decayed))
    B, Htot, heads = 2, 2, (0, 2)
    H = 2
    q, k, v = qkv(rng, B, N, Htot, d, unit_keys=True)
    alpha = rng.uniform(0.85, 0.999, (B, N, H)).astype(np.float32)
    beta = rng.uniform(0.05, 0.95, (B, N, H)).astype(np.float32)
    do = rng.standard_normal((B, N, Htot, d)).astype(np.float32)
    S0 = rng.standard_normal((B, H, d, d)).astype(np.float32) * 0.1 if with_s0 else None
    scale = d ** -0.5
    ref = oracle.delta_bwd(q, k, v, alpha, beta, do, scale=scale, S0=S0, heads=heads,
                           erase_decayed=erase_decayed)
    got = kta.gla_delta_bwd(dev(q), dev(k), dev(v), dev(alpha), dev(beta), dev(do), scale=scale,
                            S0=None if S0 is None else dev(S0), heads=heads,
                            erase_decayed=erase_decayed)
    torch.cuda.synchronize()
    kta.device_status()
    for name, g, r in zip(("dq", "dk", "dv", "dalpha", "dbeta", "dS0"), got, ref):
        e = rel(g, r)
        assert e <= F32_TOL, f"{name}: relative L2 error {e:.3e}"


def test_backward_rejects_bf16(kta):
    q = torch.zeros(1, 8, 1, 64, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        kta.swa_bwd(q, q, q, q, P=4, W=2)
    s = kta.Shape(1, 2, 4, 64, 0)
    z = torch.zeros(1, 8, 1, 64, device="cuda", dtype=torch.float32)
    p = z.data_ptr()
    st = kta.raw_call("kta_swa_bwd", p, p, p, p, p, p, p, s, 1, 1, 2, 1.0, None)
    assert st != 0 and "KTA_F32" in kta.last_error()
