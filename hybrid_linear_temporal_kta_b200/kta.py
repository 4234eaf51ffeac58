"""ctypes binding of libkta.so (C ABI in include/kta.h).

Argument marshalling only: every step of the operator runs in the library's CUDA kernels. Tensors
are torch CUDA tensors in the operator's layout [B, N, H, d] (token-major, heads interleaved);
calls are enqueued on torch's current CUDA stream. Importing this module loads the library and
raises if it is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

from . import build as _build

_LIB_PATH = _build.LIB
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libkta.so not built ({_LIB_PATH}); run hybrid_linear_temporal_kta_b200.build")
_lib = ctypes.CDLL(_LIB_PATH)

BF16, F32 = 0, 1
_DT = {torch.bfloat16: BF16, torch.float32: F32}
_STATUS = {0: "KTA_OK", 1: "KTA_ERR_INVALID_ARG", 2: "KTA_ERR_UNSUPPORTED", 3: "KTA_ERR_ALIGNMENT",
           4: "KTA_ERR_CUDA", 5: "KTA_ERR_TIMEOUT", 6: "KTA_ERR_STATE"}


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("F", ctypes.c_int), ("P", ctypes.c_int), ("d", ctypes.c_int),
                ("dtype", ctypes.c_int)]


class ProjSeg(ctypes.Structure):
    _fields_ = [("col_begin", ctypes.c_int), ("col_end", ctypes.c_int), ("dst", ctypes.c_void_p),
                ("ld", ctypes.c_longlong), ("mode", ctypes.c_int), ("bias", ctypes.c_void_p)]


PROJ_BF16, PROJ_SIGMOID_F32, PROJ_F32 = 0, 1, 2


class HybridCfg(ctypes.Structure):
    _fields_ = [("s", Shape), ("n_swa", ctypes.c_int), ("n_dswa", ctypes.c_int),
                ("n_gla", ctypes.c_int), ("W_swa", ctypes.c_int), ("W_dswa", ctypes.c_int),
                ("dil", ctypes.c_int), ("chunk", ctypes.c_int), ("gla_delta", ctypes.c_int),
                ("scale_softmax", ctypes.c_float), ("scale_gla", ctypes.c_float)]


_vp, _i, _f, _st = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_int
_fp = ctypes.c_void_p

_SIGS = {
    "kta_status_str": ([_st], ctypes.c_char_p),
    "kta_last_error": ([], ctypes.c_char_p),
    "kta_version": ([], _i),
    "kta_swa_fwd": ([_vp, _vp, _vp, _vp, Shape, _i, _i, _i, _f, _vp], _st),
    "kta_dswa_fwd": ([_vp, _vp, _vp, _vp, Shape, _i, _i, _i, _i, _f, _vp], _st),
    "kta_gla_chunk_fwd": ([_vp, _vp, _vp, _fp, _fp, _fp, _vp, Shape, _i, _i, _i, _f, _vp], _st),
    "kta_gla_delta_fwd": ([_vp, _vp, _vp, _fp, _fp, _fp, _fp, _vp, Shape, _i, _i, _i, _f, _vp],
                          _st),
    "kta_gla_gdn_fwd": ([_vp, _vp, _vp, _fp, _fp, _fp, _fp, _vp, Shape, _i, _i, _i, _f, _vp],
                        _st),
    "kta_gla_chunk_state": ([_vp, _vp, _fp, _fp, _fp, Shape, _i, _i, _i, _vp], _st),
    "kta_gla_chunk_fwd_noalloc": ([_vp, _vp, _vp, _fp, _fp, _fp, _vp, Shape, _i, _i, _i, _f, _vp],
                                  _st),
    "kta_hybrid_fwd": ([ctypes.POINTER(HybridCfg), _vp, _vp, _vp, _fp, _fp, _vp, _vp], _st),
    "kta_proj_fwd": ([_vp, _vp, _i, _i, _i, ctypes.POINTER(ProjSeg), _i, _vp], _st),
    "kta_softmax_fwd_lse": ([_vp, _vp, _vp, _vp, _fp, Shape, _i, _i, _i, _i, _f, _vp], _st),
    "kta_softmax_bwd_bf16": ([_vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _vp, Shape, _i, _i, _i, _i,
                              _f, _vp], _st),
    "kta_swa_bwd": ([_vp] * 7 + [Shape, _i, _i, _i, _f, _vp], _st),
    "kta_dswa_bwd": ([_vp] * 7 + [Shape, _i, _i, _i, _i, _f, _vp], _st),
    "kta_gla_bwd": ([_vp, _vp, _vp, _fp, _fp, _vp, _vp, _vp, _vp, _fp, _fp, Shape, _i, _i, _f,
                     _vp], _st),
    "kta_gla_delta_bwd": ([_vp, _vp, _vp, _fp, _fp, _fp, _vp, _vp, _vp, _vp, _fp, _fp, _fp, Shape,
                           _i, _i, _f, _i, _vp], _st),
    "kta_hybrid_fwd_window": ([ctypes.POINTER(HybridCfg), _i, _vp, _vp, _vp, _fp, _fp, _fp, _fp,
                               _vp, _vp], _st),
    "kta_state_affine": ([_fp, _fp, _fp, _fp, _i, _i, _vp], _st),
    "kta_gla_transition": ([_fp, _fp, _i, _i, _i, _i, _vp], _st),
    "kta_stream_create": ([ctypes.POINTER(HybridCfg), ctypes.POINTER(_vp)], _st),
    "kta_stream_step": ([_vp, _vp, _vp, _vp, _fp, _fp, _vp, _vp], _st),
    "kta_stream_reset": ([_vp, _vp], _st),
    "kta_stream_frame": ([_vp], ctypes.c_int64),
    "kta_stream_state_bytes": ([_vp], ctypes.c_size_t),
    "kta_stream_save": ([_vp, _vp, _vp], _st),
    "kta_stream_load": ([_vp, _vp, _vp], _st),
    "kta_stream_destroy": ([_vp], _st),
    "kta_device_status": ([_vp], _st),
    "kta_selftest_wait_timeout": ([ctypes.c_longlong, _vp], _st),
    "kta_trace_begin": ([], _st),
    "kta_trace_end": ([ctypes.POINTER(_i), ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(_i),
                       ctypes.POINTER(ctypes.c_double), _i], _st),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = tuple(_SIGS)


class KtaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.kta_last_error().decode()
        super().__init__(f"{where}: {_STATUS.get(status, status)}: {msg}")


def _check(status: int, where: str):
    if status != 0:
        raise KtaError(status, where)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t, off_elems: int = 0):
    return None if t is None else ctypes.c_void_p(t.data_ptr() + off_elems * t.element_size())


def _need(t, name, dtype=None):
    if not (t.is_cuda and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")


def _shape(q: torch.Tensor, P: int) -> Shape:
    B, N, _, d = q.shape
    if N % P:
        raise ValueError(f"N = {N} is not a whole number of frames of P = {P}")
    if q.dtype not in _DT:
        raise ValueError("q, k, v must be bf16 or fp32")
    return Shape(B, N // P, P, d, _DT[q.dtype])


def version() -> int:
    return _lib.kta_version()


def _softmax(fn, q, k, v, P, W, dil, scale, heads, out, stream):
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, q.dtype)
    Htot, d = q.shape[2], q.shape[3]
    h0, h1 = heads if heads is not None else (0, Htot)
    o = torch.empty_like(q) if out is None else out
    _need(o, "out", q.dtype)
    s = _shape(q, P)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    args = [_ptr(q, h0 * d), _ptr(k, h0 * d), _ptr(v, h0 * d), _ptr(o, h0 * d), s, h1 - h0, Htot, W]
    if dil is not None:
        args.append(dil)
    _check(fn(*args, scale, _stream(stream)), fn.__name__)
    return o


def swa_fwd(q, k, v, *, P: int, W: int, scale: float | None = None, heads=None, out=None,
            stream=None):
    """Frame-block-causal sliding-window attention over W frames of P tokens."""
    return _softmax(_lib.kta_swa_fwd, q, k, v, P, W, None, scale, heads, out, stream)


def dswa_fwd(q, k, v, *, P: int, W: int, dil: int, scale: float | None = None, heads=None,
             out=None, stream=None):
    """Dilated sliding-window attention: key frames f, f-dil, ..., f-(W-1)*dil."""
    return _softmax(_lib.kta_dswa_fwd, q, k, v, P, W, dil, scale, heads, out, stream)


def _linear(delta, q, k, v, alpha, beta, chunk, scale, S0, return_state, heads, out, stream,
            erase_decayed=False):
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, q.dtype)
    _need(alpha, "alpha", torch.float32)
    if delta:
        _need(beta, "beta", torch.float32)
    B, N, Htot, d = q.shape
    h0, h1 = heads if heads is not None else (0, Htot)
    H = h1 - h0
    o = torch.empty_like(q) if out is None else out
    _need(o, "out", q.dtype)
    if S0 is not None:
        _need(S0, "S0", torch.float32)
    S_out = torch.empty((B, H, d, d), device=q.device, dtype=torch.float32) if return_state else None
    s = Shape(B, 1, N, d, _DT[q.dtype])  # one frame of N tokens: the linear branches ignore frames
    if delta:
        fn = _lib.kta_gla_gdn_fwd if erase_decayed else _lib.kta_gla_delta_fwd
        st = fn(_ptr(q, h0 * d), _ptr(k, h0 * d), _ptr(v, h0 * d), _ptr(alpha), _ptr(beta),
                _ptr(S0), _ptr(S_out), _ptr(o, h0 * d), s, H, Htot, chunk, scale, _stream(stream))
    else:
        st = _lib.kta_gla_chunk_fwd(_ptr(q, h0 * d), _ptr(k, h0 * d), _ptr(v, h0 * d), _ptr(alpha),
                                    _ptr(S0), _ptr(S_out), _ptr(o, h0 * d), s, H, Htot, chunk,
                                    scale, _stream(stream))
    _check(st, "kta_gla_delta_fwd" if delta else "kta_gla_chunk_fwd")
    return (o, S_out) if return_state else o


def gla_chunk_fwd(q, k, v, alpha, *, chunk: int = 64, scale: float = 1.0, S0=None,
                  return_state: bool = False, heads=None, out=None, stream=None):
    """Vector-gated GLA; alpha [B, N, H, d] fp32. Returns o (and the final state)."""
    return _linear(False, q, k, v, alpha, None, chunk, scale, S0, return_state, heads, out, stream)


def gla_chunk_state(k, v, alpha, *, chunk: int = 64, S0=None, heads=None, stream=None):
    """End state [B, H, d, d] fp32 of a vector-gated GLA run (no outputs); k, v bf16."""
    for n, t in (("k", k), ("v", v)):
        _need(t, n, torch.bfloat16)
    _need(alpha, "alpha", torch.float32)
    B, N, Htot, d = k.shape
    h0, h1 = heads if heads is not None else (0, Htot)
    H = h1 - h0
    if S0 is not None:
        _need(S0, "S0", torch.float32)
    S_out = torch.empty((B, H, d, d), device=k.device, dtype=torch.float32)
    s = Shape(B, 1, N, d, _DT[k.dtype])
    _check(_lib.kta_gla_chunk_state(_ptr(k, h0 * d), _ptr(v, h0 * d), _ptr(alpha), _ptr(S0),
                                    _ptr(S_out), s, H, Htot, chunk, _stream(stream)),
           "kta_gla_chunk_state")
    return S_out


def gla_delta_fwd(q, k, v, alpha, beta, *, chunk: int = 64, scale: float = 1.0, S0=None,
                  return_state: bool = False, heads=None, out=None, stream=None,
                  erase_decayed: bool = False):
    """Gated delta rule; alpha, beta [B, N, H] fp32. Returns o (and the final state).
    erase_decayed: the GatedDeltaNet form M = alpha M (I - beta k k^T) + beta v k^T."""
    return _linear(True, q, k, v, alpha, beta, chunk, scale, S0, return_state, heads, out, stream,
                   erase_decayed)


def proj_fwd(x, w, segs, stream=None):
    """Y = x w^T on the tensor cores, routed by column ranges. x [..., K] bf16 (M rows), w [N, K]
    bf16; segs: list of (col_begin, col_end, dst tensor, mode[, bias]) with mode PROJ_BF16 (dst
    bf16), PROJ_SIGMOID_F32 or PROJ_F32 (dst fp32) and an optional fp32 bias of the range's width;
    dst row r holds columns [col_begin, col_end) of row r (dst viewed as [M, -1])."""
    _need(x, "x", torch.bfloat16)
    _need(w, "w", torch.bfloat16)
    K = x.shape[-1]
    M = x.numel() // K
    N = w.shape[0]
    if w.shape[1] != K:
        raise ValueError("w must be [N, K] with K = x.shape[-1]")
    arr = (ProjSeg * len(segs))()
    for i, sg in enumerate(segs):
        c0, c1, dst, mode = sg[:4]
        bias = sg[4] if len(sg) > 4 else None
        _need(dst, f"segment {i} dst", torch.bfloat16 if mode == PROJ_BF16 else torch.float32)
        if dst.numel() % M:
            raise ValueError(f"segment {i}: dst does not have M = {M} rows")
        if bias is not None:
            _need(bias, f"segment {i} bias", torch.float32)
            if bias.numel() != c1 - c0:
                raise ValueError(f"segment {i}: bias must have {c1 - c0} entries")
        arr[i] = ProjSeg(c0, c1, dst.data_ptr(), dst.numel() // M, mode,
                         None if bias is None else bias.data_ptr())
    _check(_lib.kta_proj_fwd(_ptr(x), _ptr(w), M, N, K, arr, len(segs), _stream(stream)),
           "kta_proj_fwd")


def linear(x, w, *, out=None, stream=None):
    """x [..., K] bf16 times w [N, K]^T -> [..., N] bf16 (e.g. the output projection)."""
    y = torch.empty(x.shape[:-1] + (w.shape[0],), device=x.device, dtype=torch.bfloat16) \
        if out is None else out
    proj_fwd(x, w, [(0, w.shape[0], y, PROJ_BF16)], stream)
    return y


def qkv_gate_proj(x, w, *, H: int, d: int, n_gla: int, gla_delta: bool = False, gate_bias=None,
                  stream=None):
    """One launch for every input of hybrid_fwd: x [B, N, C] bf16 and the stacked weight
    w = [W_Q; W_K; W_V; W_alpha (; W_beta)] ([3 H d + n_gla d, C] for vector GLA,
    [3 H d + 2 n_gla, C] for the delta rule). Returns q, k, v [B, N, H, d] bf16 and
    alpha = sigmoid(W_alpha x) ([B, N, n_gla, d] or [B, N, n_gla] fp32), beta = sigmoid(W_beta x)
    ([B, N, n_gla] fp32, delta rule only, else None). gate_bias: optional fp32 offsets of the
    alpha logits (one per alpha column)."""
    B, N, _ = x.shape
    hd = H * d
    q, k, v = (torch.empty((B, N, H, d), device=x.device, dtype=torch.bfloat16)
               for _ in range(3))
    segs = [(0, hd, q, PROJ_BF16), (hd, 2 * hd, k, PROJ_BF16), (2 * hd, 3 * hd, v, PROJ_BF16)]
    alpha = beta = None
    if n_gla:
        ga = n_gla if gla_delta else n_gla * d
        alpha = torch.empty((B, N, n_gla) if gla_delta else (B, N, n_gla, d), device=x.device,
                            dtype=torch.float32)
        segs.append((3 * hd, 3 * hd + ga, alpha, PROJ_SIGMOID_F32, gate_bias))
        if gla_delta:
            beta = torch.empty((B, N, n_gla), device=x.device, dtype=torch.float32)
            segs.append((3 * hd + ga, 3 * hd + 2 * ga, beta, PROJ_SIGMOID_F32))
    want = segs[-1][1]
    if w.shape[0] != want:
        raise ValueError(f"stacked weight must have {want} rows, got {w.shape[0]}")
    proj_fwd(x, w, segs, stream)
    return q, k, v, alpha, beta


def softmax_fwd_lse(q, k, v, *, P: int, W: int, dil: int = 1, scale: float | None = None,
                    heads=None, out=None, stream=None):
    """SWA (dil = 1) / DSWA forward, bf16, that also returns each row's base-2 log-sum-exp:
    (o, lse) with lse [B, H, N] fp32 for the heads in range (the bf16 backward's input)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, torch.bfloat16)
    B, N, Htot, d = q.shape
    h0, h1 = heads if heads is not None else (0, Htot)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, h1 - h0, N), device=q.device, dtype=torch.float32)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    _check(_lib.kta_softmax_fwd_lse(_ptr(q, h0 * d), _ptr(k, h0 * d), _ptr(v, h0 * d),
                                    _ptr(o, h0 * d), _ptr(lse), _shape(q, P), h1 - h0, Htot, W, dil,
                                    scale, _stream(stream)), "kta_softmax_fwd_lse")
    return o, lse


def softmax_bwd_bf16(q, k, v, o, lse, dout, *, P: int, W: int, dil: int = 1,
                     scale: float | None = None, heads=None, out=None, stream=None):
    """Tensor-core gradients (dq, dk, dv) of sum(dout * o) for SWA / DSWA heads, bf16, from the
    forward's o and lse (softmax_fwd_lse). Heads outside the range are left zero."""
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _need(t, n, torch.bfloat16)
    _need(lse, "lse", torch.float32)
    B, N, Htot, d = q.shape
    h0, h1 = heads if heads is not None else (0, Htot)
    if out is None:
        dq, dk, dv = (torch.zeros_like(q) for _ in range(3))
    else:
        dq, dk, dv = out
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    args = [_ptr(t, h0 * d) for t in (q, k, v, o)] + [_ptr(lse), _ptr(dout, h0 * d)]
    args += [_ptr(t, h0 * d) for t in (dq, dk, dv)]
    _check(_lib.kta_softmax_bwd_bf16(*args, _shape(q, P), h1 - h0, Htot, W, dil, scale,
                                     _stream(stream)), "kta_softmax_bwd_bf16")
    return dq, dk, dv


def _grads(q, out):
    """Gradient buffers: `out` (three tensors shaped like q) or fresh zeros."""
    if out is None:
        return tuple(torch.zeros_like(q) for _ in range(3))
    for n, t in zip(("dq", "dk", "dv"), out):
        _need(t, n, torch.float32)
        if t.shape != q.shape:
            raise ValueError(f"{n} must have q's shape")
    return tuple(out)


def _softmax_bwd(fn, q, k, v, dout, P, W, dil, scale, heads, out, stream):
    for n, t in (("q", q), ("k", k), ("v", v), ("dout", dout)):
        _need(t, n, torch.float32)
    Htot, d = q.shape[2], q.shape[3]
    h0, h1 = heads if heads is not None else (0, Htot)
    dq, dk, dv = _grads(q, out)
    s = _shape(q, P)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    args = [_ptr(t, h0 * d) for t in (q, k, v, dout, dq, dk, dv)] + [s, h1 - h0, Htot, W]
    if dil is not None:
        args.append(dil)
    _check(fn(*args, scale, _stream(stream)), fn.__name__)
    return dq, dk, dv


def swa_bwd(q, k, v, dout, *, P: int, W: int, scale: float | None = None, heads=None, out=None,
            stream=None):
    """Gradients (dq, dk, dv) of sum(dout * swa_fwd(q, k, v)); fp32. Only the heads in range are
    written (fresh buffers are zero elsewhere); out = (dq, dk, dv) reuses buffers."""
    return _softmax_bwd(_lib.kta_swa_bwd, q, k, v, dout, P, W, None, scale, heads, out, stream)


def dswa_bwd(q, k, v, dout, *, P: int, W: int, dil: int, scale: float | None = None, heads=None,
             out=None, stream=None):
    """Gradients (dq, dk, dv) of sum(dout * dswa_fwd(q, k, v)); fp32."""
    return _softmax_bwd(_lib.kta_dswa_bwd, q, k, v, dout, P, W, dil, scale, heads, out, stream)


def _linear_bwd(delta, q, k, v, alpha, beta, dout, scale, S0, heads, out, stream, erase_decayed):
    for n, t in (("q", q), ("k", k), ("v", v), ("dout", dout), ("alpha", alpha)):
        _need(t, n, torch.float32)
    if delta:
        _need(beta, "beta", torch.float32)
    if S0 is not None:
        _need(S0, "S0", torch.float32)
    B, N, Htot, d = q.shape
    h0, h1 = heads if heads is not None else (0, Htot)
    H = h1 - h0
    dq, dk, dv = _grads(q, out)
    dalpha = torch.empty_like(alpha)
    dbeta = torch.empty_like(beta) if delta else None
    dS0 = torch.empty((B, H, d, d), device=q.device, dtype=torch.float32)
    s = Shape(B, 1, N, d, _DT[q.dtype])
    ptrs = [_ptr(t, h0 * d) for t in (q, k, v)]
    grads = [_ptr(t, h0 * d) for t in (dq, dk, dv)]
    if delta:
        st = _lib.kta_gla_delta_bwd(*ptrs, _ptr(alpha), _ptr(beta), _ptr(S0), _ptr(dout, h0 * d),
                                    *grads, _ptr(dalpha), _ptr(dbeta), _ptr(dS0), s, H, Htot,
                                    scale, int(erase_decayed), _stream(stream))
        _check(st, "kta_gla_delta_bwd")
        return dq, dk, dv, dalpha, dbeta, dS0
    st = _lib.kta_gla_bwd(*ptrs, _ptr(alpha), _ptr(S0), _ptr(dout, h0 * d), *grads, _ptr(dalpha),
                          _ptr(dS0), s, H, Htot, scale, _stream(stream))
    _check(st, "kta_gla_bwd")
    return dq, dk, dv, dalpha, dS0


def gla_bwd(q, k, v, alpha, dout, *, scale: float = 1.0, S0=None, heads=None, out=None,
            stream=None):
    """Gradients (dq, dk, dv, dalpha, dS0) of sum(dout * gla_chunk_fwd(...)); fp32."""
    return _linear_bwd(False, q, k, v, alpha, None, dout, scale, S0, heads, out, stream, False)


def gla_delta_bwd(q, k, v, alpha, beta, dout, *, scale: float = 1.0, S0=None, heads=None,
                  out=None, stream=None, erase_decayed: bool = False):
    """Gradients (dq, dk, dv, dalpha, dbeta, dS0) of sum(dout * gla_delta_fwd(...)); fp32."""
    return _linear_bwd(True, q, k, v, alpha, beta, dout, scale, S0, heads, out, stream,
                       erase_decayed)


def hybrid_cfg(*, B: int, F: int, P: int, d: int, dtype=torch.bfloat16, n_swa: int, n_dswa: int,
               n_gla: int, W_swa: int = 3, W_dswa: int = 4, dil: int = 3, chunk: int = 64,
               gla_delta: int = 0, scale_softmax: float | None = None,
               scale_gla: float = 1.0) -> HybridCfg:
    return HybridCfg(Shape(B, F, P, d, _DT[dtype]), n_swa, n_dswa, n_gla, W_swa, W_dswa, dil, chunk,
                     int(gla_delta), 1.0 / math.sqrt(d) if scale_softmax is None else scale_softmax,
                     scale_gla)


def cfg_from_workload(w, B: int | None = None, F: int | None = None) -> HybridCfg:
    """HybridCfg of a synth.Workload."""
    return hybrid_cfg(B=w.B if B is None else B, F=w.F if F is None else F, P=w.P, d=w.d,
                      dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32,
                      n_swa=w.n_swa, n_dswa=w.n_dswa, n_gla=w.n_gla, W_swa=w.W_swa,
                      W_dswa=w.W_dswa, dil=w.dil, chunk=w.chunk, gla_delta=w.gla_delta,
                      scale_softmax=w.scale_softmax)


def hybrid_fwd(cfg: HybridCfg, q, k, v, alpha=None, beta=None, *, out=None, stream=None):
    """Hybrid layer: SWA heads, DSWA heads, GLA heads (outputs concatenated by head)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, q.dtype)
    o = torch.empty_like(q) if out is None else out
    _check(_lib.kta_hybrid_fwd(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                               _ptr(beta), _ptr(o), _stream(stream)), "kta_hybrid_fwd")
    return o


def hybrid_fwd_window(cfg: HybridCfg, f0: int, q, k, v, alpha=None, beta=None, *, S0=None,
                      return_state: bool = False, out=None, stream=None):
    """Hybrid layer for the query frames f0 .. F-1 of a key / value span of cfg.s.F frames (one
    sequence): q, alpha, beta cover the query frames, k and v the whole span; the GLA heads start
    from S0 ([1, n_gla, d, d] fp32 or None) and, with return_state, also return their end state."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, q.dtype)
    if S0 is not None:
        _need(S0, "S0", torch.float32)
    o = torch.empty_like(q) if out is None else out
    S_out = None
    if return_state:
        S_out = torch.empty((q.shape[0], cfg.n_gla, cfg.s.d, cfg.s.d), device=q.device,
                            dtype=torch.float32)
    _check(_lib.kta_hybrid_fwd_window(ctypes.byref(cfg), f0, _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(alpha), _ptr(beta), _ptr(S0), _ptr(S_out), _ptr(o),
                                      _stream(stream)), "kta_hybrid_fwd_window")
    return (o, S_out) if return_state else o


def gla_transition(alpha, *, out=None, stream=None):
    """T = diag(prod_t alpha_t) [B, H, d, d] of a vector-gated GLA run; alpha [B, N, H, d] fp32."""
    _need(alpha, "alpha", torch.float32)
    B, N, H, d = alpha.shape
    T = torch.empty((B, H, d, d), device=alpha.device, dtype=torch.float32) if out is None else out
    _need(T, "out", torch.float32)
    _check(_lib.kta_gla_transition(_ptr(alpha), _ptr(T), B, N, H, d, _stream(stream)),
           "kta_gla_transition")
    return T


def state_affine(A, X, E=None, *, out=None, stream=None):
    """Y = A X + E for stacks of square fp32 matrices [..., d, d] (E optional)."""
    for n, t in (("A", A), ("X", X)):
        _need(t, n, torch.float32)
    if E is not None:
        _need(E, "E", torch.float32)
    d = A.shape[-1]
    Y = torch.empty_like(X) if out is None else out
    _check(_lib.kta_state_affine(_ptr(A), _ptr(X), _ptr(E), _ptr(Y), A.numel() // (d * d), d,
                                 _stream(stream)), "kta_state_affine")
    return Y


class Stream:
    """One-frame-at-a-time rollout with carried GLA state and rolling K/V rings."""

    def __init__(self, cfg: HybridCfg):
        self.cfg = cfg
        h = ctypes.c_void_p()
        _check(_lib.kta_stream_create(ctypes.byref(cfg), ctypes.byref(h)), "kta_stream_create")
        self._h = h

    def step(self, q_f, k_f, v_f, alpha_f=None, beta_f=None, *, out=None, stream=None):
        o = torch.empty_like(q_f) if out is None else out
        _check(_lib.kta_stream_step(self._h, _ptr(q_f), _ptr(k_f), _ptr(v_f), _ptr(alpha_f),
                                    _ptr(beta_f), _ptr(o), _stream(stream)), "kta_stream_step")
        return o

    def reset(self, stream=None):
        _check(_lib.kta_stream_reset(self._h, _stream(stream)), "kta_stream_reset")

    @property
    def frame(self) -> int:
        return int(_lib.kta_stream_frame(self._h))

    @property
    def state_bytes(self) -> int:
        return int(_lib.kta_stream_state_bytes(self._h))

    def save(self, stream=None) -> torch.Tensor:
        blob = torch.empty(self.state_bytes, dtype=torch.uint8, device="cuda")
        _check(_lib.kta_stream_save(self._h, _ptr(blob), _stream(stream)), "kta_stream_save")
        return blob

    def load(self, blob: torch.Tensor, stream=None):
        _check(_lib.kta_stream_load(self._h, _ptr(blob), _stream(stream)), "kta_stream_load")

    def close(self):
        if self._h is not None:
            _check(_lib.kta_stream_destroy(self._h), "kta_stream_destroy")
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def device_status(stream=None):
    """Raise KtaError if a bounded device wait expired since the last check."""
    _check(_lib.kta_device_status(_stream(stream)), "kta_device_status")


def selftest_wait_timeout(budget_cycles: int, stream=None):
    _check(_lib.kta_selftest_wait_timeout(int(budget_cycles), _stream(stream)),
           "kta_selftest_wait_timeout")


class trace:
    """Context manager: per-kernel launch counts and device milliseconds of every library kernel
    launched inside the block (CUDA events on each launch's own stream)."""

    def __enter__(self):
        _check(_lib.kta_trace_begin(), "kta_trace_begin")
        self.kernels = {}
        return self

    def __exit__(self, *exc):
        cap = 32
        n = _i()
        names = (ctypes.c_char_p * cap)()
        launches = (_i * cap)()
        ms = (ctypes.c_double * cap)()
        _check(_lib.kta_trace_end(ctypes.byref(n), names, launches, ms, cap), "kta_trace_end")
        self.kernels = {names[i].decode(): {"launches": launches[i], "ms": ms[i]}
                        for i in range(min(n.value, cap))}
        return False


def raw_call(name: str, *args) -> int:
    """Call an exported entry point with raw ctypes arguments; returns the kta_status code."""
    return int(getattr(_lib, name)(*args))


def last_error() -> str:
    return _lib.kta_last_error().decode()
