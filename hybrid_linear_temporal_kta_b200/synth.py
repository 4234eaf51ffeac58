"""Seeded synthetic inputs for the hybrid temporal attention operator.

This module holds the input recipe only and none of the operator's arithmetic; the tests feed
the same tensors to the CUDA path and to the CPU oracle. Workload shapes follow the pages'
video setting: latent frames of P tokens in raster order, F frames in time order (81-frame
clips give 21 latent frames; frames of 30x52 or 22x40 latent tokens).

Recipe (stated once, used everywhere):
  - q, k, v ~ N(0, 1) drawn in float64 by numpy's PCG64 generator, rounded once to the storage
    dtype (bf16 round-to-nearest-even, or fp32);
  - vector GLA gate alpha = sigmoid(N(mu, 1)) per token, head and key dimension (fp32);
  - delta-rule gates alpha = sigmoid(N(mu, 1)), beta = sigmoid(N(0, 1)) per token and head;
  - for the delta rule, k is L2-normalised per token and head in float64 before rounding;
  - seed of tensor j of workload c = 1000 * c + j (q = 0, k = 1, v = 2, alpha = 3, beta = 4).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

TENSOR_ID = {"q": 0, "k": 1, "v": 2, "alpha": 3, "beta": 4}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One operator configuration. Heads are split SWA | DSWA | GLA in that order."""
    name: str
    B: int
    F: int
    P: int
    d: int
    n_swa: int
    n_dswa: int
    n_gla: int
    W_swa: int = 3
    W_dswa: int = 4
    dil: int = 3
    chunk: int = 64
    gla_delta: bool = False
    dtype: str = "bf16"          # storage / compute type of q, k, v, o
    alpha_mu: float = 3.0
    seed_base: int = 0

    @property
    def N(self) -> int:
        return self.F * self.P

    @property
    def H(self) -> int:
        return self.n_swa + self.n_dswa + self.n_gla

    @property
    def scale_softmax(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The named workloads (sizes as the operator's configurations give them).
TINY_F32 = Workload("tiny_f32_hybrid", B=1, F=8, P=16, d=32, n_swa=1, n_dswa=1, n_gla=1,
                    W_swa=2, W_dswa=2, dil=2, chunk=16, dtype="f32", alpha_mu=2.0,
                    seed_base=1000)
HYBRID_BF16 = Workload("hybrid_bf16_F21_P1560", B=1, F=21, P=1560, d=128, n_swa=8, n_dswa=8,
                       n_gla=8, W_swa=3, W_dswa=4, dil=3, chunk=64, seed_base=2000)
DELTA_BF16 = Workload("gated_delta_bf16_B2_L65536", B=2, F=64, P=1024, d=128, n_swa=0,
                      n_dswa=0, n_gla=16, chunk=64, gla_delta=True, seed_base=3000)
HYBRID_BWD_F32 = Workload("hybrid_bwd_f32_F21_P1560", B=1, F=21, P=1560, d=128, n_swa=8,
                          n_dswa=8, n_gla=8, W_swa=3, W_dswa=4, dil=3, chunk=64, dtype="f32",
                          seed_base=6000)
STREAM_BF16 = Workload("stream_bf16_P880_F240", B=1, F=240, P=880, d=128, n_swa=8, n_dswa=8,
                       n_gla=8, W_swa=3, W_dswa=4, dil=3, chunk=64, seed_base=4000)


def sweep_workload(F: int) -> Workload:
    """Length sweep of the hybrid layer: P = 1024 tokens per frame, F frames."""
    return HYBRID_BF16.replace(name=f"sweep_bf16_P1024_F{F}", F=F, P=1024, seed_base=5000)


WORKLOADS = {w.name: w for w in (TINY_F32, HYBRID_BF16, DELTA_BF16, STREAM_BF16,
                                  HYBRID_BWD_F32)}


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal(shape, seed: int, mu: float = 0.0) -> np.ndarray:
    """N(mu, 1) in float64, seeded."""
    return _rng(seed).standard_normal(size=shape, dtype=np.float64) + mu


def sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def to_storage(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Round float64 values once to the storage dtype (CPU tensor)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch_dtype(dtype)) if dtype != "f32" else t


def make_inputs(w: Workload, *, seed_base: int | None = None, B: int | None = None,
                N: int | None = None) -> dict:
    """Build q, k, v, alpha, beta (CPU tensors) for workload w.

    q, k, v: [B, N, H, d] in w.dtype. alpha: [B, N, n_gla, d] fp32 (vector gate) or
    [B, N, n_gla] fp32 (delta rule). beta: [B, N, n_gla] fp32 for the delta rule, else None.
    """
    sb = w.seed_base if seed_base is None else seed_base
    B = w.B if B is None else B
    N = w.N if N is None else N
    H, d = w.H, w.d
    out = {}
    for name in ("q", "k", "v"):
        x = normal((B, N, H, d), sb + TENSOR_ID[name])
        if name == "k" and w.gla_delta and w.n_gla:
            g = slice(w.n_swa + w.n_dswa, H)
            kg = x[:, :, g, :]
            x[:, :, g, :] = kg / np.linalg.norm(kg, axis=-1, keepdims=True)
        out[name] = to_storage(x, w.dtype)
    if w.n_gla:
        if w.gla_delta:
            a = sigmoid(normal((B, N, w.n_gla), sb + TENSOR_ID["alpha"], w.alpha_mu))
            be = sigmoid(normal((B, N, w.n_gla), sb + TENSOR_ID["beta"], 0.0))
            out["alpha"] = torch.from_numpy(a.astype(np.float32))
            out["beta"] = torch.from_numpy(be.astype(np.float32))
        else:
            a = sigmoid(normal((B, N, w.n_gla, d), sb + TENSOR_ID["alpha"], w.alpha_mu))
            out["alpha"] = torch.from_numpy(a.astype(np.float32))
            out["beta"] = None
    else:
        out["alpha"] = None
        out["beta"] = None
    return out


def make_inputs_device(w: Workload, *, seed: int, device="cuda", B: int | None = None,
                       N: int | None = None) -> dict:
    """The make_inputs recipe drawn on the device with torch's seeded generator (for timing-only
    workloads whose inputs are too large to draw on the host): same shapes, distributions and
    dtypes, different random numbers."""
    B = w.B if B is None else B
    N = w.N if N is None else N
    H, d = w.H, w.d
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    dt = torch_dtype(w.dtype)
    out = {}
    for name in ("q", "k", "v"):
        x = torch.randn((B, N, H, d), generator=g, device=device, dtype=torch.float32)
        if name == "k" and w.gla_delta and w.n_gla:
            kg = x[:, :, w.n_swa + w.n_dswa:, :]
            kg /= kg.norm(dim=-1, keepdim=True)
        out[name] = x.to(dt)
        del x
    out["alpha"] = out["beta"] = None
    if w.n_gla:
        shp = (B, N, w.n_gla) if w.gla_delta else (B, N, w.n_gla, d)
        out["alpha"] = torch.sigmoid(torch.randn(shp, generator=g, device=device) + w.alpha_mu)
        if w.gla_delta:
            out["beta"] = torch.sigmoid(torch.randn(shp, generator=g, device=device))
    return out


def sample_rows(N: int, P: int, frac: float, seed: int) -> np.ndarray:
    """Query rows for sampled parity at full size: every frame's first and last row, the rows
    at multiples of 128 around them (tile edges), plus a seeded random fraction."""
    rows = set()
    F = (N + P - 1) // P
    for f in range(F):
        lo, hi = f * P, min((f + 1) * P, N) - 1
        rows.update((lo, hi))
        for off in (127, 128):
            if lo + off <= hi:
                rows.add(lo + off)
    r = _rng(seed).choice(N, size=max(1, int(frac * N)), replace=False)
    rows.update(int(x) for x in r)
    return np.array(sorted(rows), dtype=np.int64)
