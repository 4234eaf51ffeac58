"""GPU parity of the tensor-core projections (kta_proj_fwd) against the fp64 oracle: ragged row,
column and K tails, every epilogue mode, routed column ranges, the stacked q/k/v/gate weight of
the hybrid layer, and sampled rows at the full 32,760-token layer size."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

BF16_TOL = 1e-2
F32_TOL = 1e-4


@pytest.fixture(scope="module")
def kta():
    from hybrid_linear_temporal_kta_b200 import build
    build.build()
    from hybrid_linear_temporal_kta_b200 import kta as mod
    return mod


def rel(got, ref):
    got = np.asarray(got, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def bf16_pair(rng, shape, scale=1.0):
    """A bf16 device tensor and the same values as float32 on the host."""
    t = (torch.from_numpy(rng.standard_normal(shape).astype(np.float32)) * scale).to(torch.bfloat16)
    return t.cuda(), t.float().numpy()


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 600, 192), (1000, 1040, 200),
                                   (77, 40, 8), (4096, 512, 1024)])
def test_linear_parity(kta, M, N, K):
    rng = np.random.default_rng(M + N + K)
    x, xh = bf16_pair(rng, (M, K))
    w, wh = bf16_pair(rng, (N, K), K ** -0.5)
    y = kta.linear(x, w)
    torch.cuda.synchronize()
    kta.device_status()
    ref = oracle.proj(xh, wh)
    assert rel(y.float().cpu().numpy(), ref) <= BF16_TOL


def test_modes_and_routing(kta):
    rng = np.random.default_rng(7)
    M, K, N = 333, 256, 700
    x, xh = bf16_pair(rng, (M, K))
    w, wh = bf16_pair(rng, (N, K), K ** -0.5)
    a = torch.empty((M, 256), device="cuda", dtype=torch.bfloat16)
    b = torch.empty((M, 200), device="cuda", dtype=torch.float32)
    c = torch.full((M, 3, 37), -7.0, device="cuda", dtype=torch.float32)  # odd ld: scalar path
    segs = [(0, 256, a, kta.PROJ_BF16), (256, 456, b, kta.PROJ_SIGMOID_F32),
            (600, 700, c[:, :, :].reshape(M, 111)[:, :100], kta.PROJ_F32)]
    with pytest.raises(ValueError):   # a non-contiguous dst is refused
        kta.proj_fwd(x, w, segs)
    c2 = torch.full((M, 111), -7.0, device="cuda", dtype=torch.float32)
    segs[2] = (600, 700, c2, kta.PROJ_F32)
    kta.proj_fwd(x, w, segs)
    torch.cuda.synchronize()
    kta.device_status()
    raw = oracle.proj(xh, wh)
    sig = oracle.proj(xh, wh, sigmoid_cols=(256, 456))
    assert rel(a.float().cpu().numpy(), raw[:, :256]) <= BF16_TOL
    assert rel(b.cpu().numpy(), sig[:, 256:456]) <= F32_TOL
    cc = c2.cpu().numpy()
    assert rel(cc[:, :100], raw[:, 600:700]) <= F32_TOL
    assert np.all(cc[:, 100:] == -7.0)   # columns past the range untouched


def test_invalid_arguments_are_refused(kta):
    x = torch.zeros((4, 12), device="cuda", dtype=torch.bfloat16)   # K = 12: not a multiple of 8
    w = torch.zeros((8, 12), device="cuda", dtype=torch.bfloat16)
    y = torch.empty((4, 8), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(kta.KtaError):
        kta.proj_fwd(x, w, [(0, 8, y, kta.PROJ_BF16)])
    x = torch.zeros((4, 16), device="cuda", dtype=torch.bfloat16)
    w = torch.zeros((8, 16), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(kta.KtaError):   # overlapping ranges
        kta.proj_fwd(x, w, [(0, 8, y, kta.PROJ_BF16), (4, 8, y, kta.PROJ_BF16)])


@pytest.mark.parametrize("gla_delta", [False, True])
def test_stacked_qkv_gate_projection(kta, gla_delta):
    rng = np.random.default_rng(11 + int(gla_delta))
    B, N, C, H, d, n_gla = 2, 200, 384, 3, 64, 1
    x, xh = bf16_pair(rng, (B, N, C))
    rows = 3 * H * d + (2 * n_gla if gla_delta else n_gla * d)
    w, wh = bf16_pair(rng, (rows, C), C ** -0.5)
    ga = n_gla if gla_delta else n_gla * d
    gb = (3.0 + 0.5 * rng.standard_normal(ga)).astype(np.float32)   # forget gates near 1
    q, k, v, a, be = kta.qkv_gate_proj(x, w, H=H, d=d, n_gla=n_gla, gla_delta=gla_delta,
                                       gate_bias=torch.from_numpy(gb).cuda())
    torch.cuda.synchronize()
    kta.device_status()
    hd = 3 * H * d
    bias = np.zeros(rows, dtype=np.float32)
    bias[hd:hd + ga] = gb
    ref = oracle.proj(xh, wh, sigmoid_cols=(hd, rows), bias=bias)
    for i, t in enumerate((q, k, v)):
        got = t.float().cpu().numpy().reshape(B * N, H * d)
        assert rel(got, ref[:, i * H * d:(i + 1) * H * d]) <= BF16_TOL
    assert rel(a.cpu().numpy().reshape(B * N, ga), ref[:, hd:hd + ga]) <= F32_TOL
    if gla_delta:
        assert rel(be.cpu().numpy().reshape(B * N, ga), ref[:, hd + ga:]) <= F32_TOL
    else:
        assert be is None


def test_full_layer_size_sampled_rows(kta):
    """The hybrid layer's projection at full size (32,760 tokens, C = 3072, 24 heads of 128,
    8 vector-GLA heads): 10,240 output columns, checked on sampled rows (first and last rows of
    the tile grid, a ragged last tile, a seeded set)."""
    g = torch.Generator(device="cuda")
    g.manual_seed(99)
    B, N, C, H, d, n_gla = 1, 32760, 3072, 24, 128, 8
    x = torch.randn((B, N, C), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((3 * H * d + n_gla * d, C), generator=g, device="cuda") * C ** -0.5).to(
        torch.bfloat16)
    q, k, v, a, _ = kta.qkv_gate_proj(x, w, H=H, d=d, n_gla=n_gla)
    torch.cuda.synchronize()
    kta.device_status()
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 121, N - 1], rng.integers(0, N, 40)]))
    xs = x[0, rows].float().cpu().numpy()
    wh = w.float().cpu().numpy()
    hd = 3 * H * d
    ref = oracle.proj(xs, wh, sigmoid_cols=(hd, hd + n_gla * d))
    got = torch.cat([t[0, rows].reshape(len(rows), -1).float() for t in (q, k, v)], 1)
    assert rel(got.cpu().numpy(), ref[:, :hd]) <= BF16_TOL
    assert rel(a[0, rows].reshape(len(rows), -1).cpu().numpy(), ref[:, hd:]) <= F32_TOL


@pytest.mark.parametrize("M,N,K", [(1, 1, 8), (1, 300, 16), (129, 257, 72)])
def test_degenerate_and_odd_shapes(kta, M, N, K):
    """One row, one column, K below one 64-wide step, and tile edges plus one."""
    rng = np.random.default_rng(M * 7 + N + K)
    x, xh = bf16_pair(rng, (M, K))
    w, wh = bf16_pair(rng, (N, K))
    y = torch.empty((M, N), device="cuda", dtype=torch.float32)
    kta.proj_fwd(x, w, [(0, N, y, kta.PROJ_F32)])
    torch.cuda.synchronize()
    kta.device_status()
    assert rel(y.cpu().numpy(), oracle.proj(xh, wh)) <= F32_TOL
