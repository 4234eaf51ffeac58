"""Plain fp64 CPU oracle for the Hybrid Linear Temporal Attention operator.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package; the CUDA product path never does, and this package imports nothing from
it. The arithmetic lives in ``kta_oracle.c`` (plain loops in double precision, one function per
branch, each citing the page passage it follows). This module only compiles that file with gcc
and marshals numpy arrays into it.

Sources, by page title and section:
  - paper-read "Kairos: A Native World Model Stack for Physical AI" (yingwang.github.io),
    section 2 "Method", second pillar: SWA, DSWA and GLA paragraphs and the gated delta-rule
    equations;
  - ai-papers.net "Kairos ... hybrid attention" summary, section "3-layer hybrid temporal
    architecture".

Parity status: every function here is pinned by tests/test_oracle_pins.py against closed forms,
special cases that reduce to textbook attention, a page identity (the DSWA reshape), exact
brute-force mask counts and the geometric-decay claim. None is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kta_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_int = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile kta_oracle.c into oracle/_build/liboracle.so (gcc, -O2, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_swa.argtypes = [_f32p, _f32p, _f32p, _f64p] + [_int] * 8 + [
                ctypes.c_double, _i64p, ctypes.c_int64]
            lib.oracle_dswa.argtypes = [_f32p, _f32p, _f32p, _f64p] + [_int] * 9 + [
                ctypes.c_double, _i64p, ctypes.c_int64]
            lib.oracle_gla.argtypes = [_f32p, _f32p, _f32p, _f32p, _f64p, _f64p, _f64p] + [
                _int] * 6 + [ctypes.c_double]
            lib.oracle_delta.argtypes = [_f32p, _f32p, _f32p, _f32p, _f32p, _f64p, _f64p,
                                         _f64p] + [_int] * 6 + [ctypes.c_double, _int]
            lib.oracle_visible.argtypes = [_i64p, _i64p, ctypes.c_int64, _int, _int, _int, _int,
                                           _u8p]
            lib.oracle_softmax_bwd.argtypes = [_f32p, _f32p, _f32p, _f64p, _f64p, _f64p, _f64p] + [
                _int] * 10 + [ctypes.c_double]
            lib.oracle_gla_bwd.argtypes = [_f32p, _f32p, _f32p, _f32p, _f64p, _f64p, _f64p, _f64p,
                                           _f64p, _f64p, _f64p] + [_int] * 6 + [ctypes.c_double]
            lib.oracle_delta_bwd.argtypes = [_f32p, _f32p, _f32p, _f32p, _f32p, _f64p, _f64p,
                                             _f64p, _f64p, _f64p, _f64p, _f64p, _f64p] + [
                _int] * 6 + [ctypes.c_double, _int]
            lib.oracle_proj.argtypes = [_f32p, _f32p, _f32p, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_int64, _i64p, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_int64, _f64p]
            lib.oracle_set_threads.argtypes = [_int]
            lib.oracle_get_threads.restype = _int
            for name in ("oracle_swa", "oracle_dswa", "oracle_gla", "oracle_delta",
                         "oracle_softmax_bwd", "oracle_gla_bwd", "oracle_delta_bwd",
                         "oracle_proj"):
                getattr(lib, name).restype = _int
            _lib = lib
    return _lib


def set_threads(n: int) -> None:
    """Number of OpenMP threads the oracle uses (0 = all host cores)."""
    _load().oracle_set_threads(int(n))


def threads() -> int:
    return int(_load().oracle_get_threads())


def _f32(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a CPU torch tensor of any float dtype
        x = x.detach().float().contiguous().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().double().contiguous().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _rows(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(rows, dtype=np.int64)
    return r, int(r.size)


def _check(rc: int, name: str):
    if rc != 0:
        raise ValueError(f"{name}: invalid arguments")


def swa(q, k, v, P: int, W: int, scale: float, heads=None, rows=None, out=None) -> np.ndarray:
    """Sliding-window softmax attention over frames of P tokens, window W frames.

    q, k, v: [B, N, H, d]. heads = (h0, h1) computes those heads only (others of ``out`` are
    left as they were; NaN in a fresh output). rows = query token indices to evaluate (None =
    all). Returns o [B, N, H, d] float64.
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, N, H, d = q.shape
    h0, h1 = heads if heads is not None else (0, H)
    o = np.full((B, N, H, d), np.nan) if out is None else out
    r, nr = _rows(rows)
    rc = _load().oracle_swa(_p(q, _f32p), _p(k, _f32p), _p(v, _f32p), _p(o, _f64p),
                            B, N, H, d, h0, h1, P, W, float(scale),
                            None if r is None else _p(r, _i64p), nr)
    _check(rc, "swa")
    return o


def dswa(q, k, v, P: int, W: int, dil: int, scale: float, heads=None, rows=None,
         out=None) -> np.ndarray:
    """Dilated sliding-window attention: frames f, f-dil, ..., f-(W-1)*dil of query frame f."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, N, H, d = q.shape
    h0, h1 = heads if heads is not None else (0, H)
    o = np.full((B, N, H, d), np.nan) if out is None else out
    r, nr = _rows(rows)
    rc = _load().oracle_dswa(_p(q, _f32p), _p(k, _f32p), _p(v, _f32p), _p(o, _f64p),
                             B, N, H, d, h0, h1, P, W, dil, float(scale),
                             None if r is None else _p(r, _i64p), nr)
    _check(rc, "dswa")
    return o


def gla(q, k, v, alpha, scale: float = 1.0, S0=None, heads=None, out=None):
    """Vector-gated linear attention recurrence. alpha: [B, N, h1-h0, d].

    Returns (o [B, N, H, d] float64, S_out [B, h1-h0, d, d] float64, key-major).
    """
    q, k, v, a = _f32(q), _f32(k), _f32(v), _f32(alpha)
    B, N, H, d = q.shape
    h0, h1 = heads if heads is not None else (0, H)
    o = np.full((B, N, H, d), np.nan) if out is None else out
    S_out = np.zeros((B, h1 - h0, d, d))
    s0 = None if S0 is None else _f64(S0)
    rc = _load().oracle_gla(_p(q, _f32p), _p(k, _f32p), _p(v, _f32p), _p(a, _f32p),
                            None if s0 is None else _p(s0, _f64p), _p(o, _f64p),
                            _p(S_out, _f64p), B, N, H, d, h0, h1, float(scale))
    _check(rc, "gla")
    return o, S_out


def delta(q, k, v, alpha, beta, scale: float = 1.0, S0=None, heads=None, out=None,
          erase_decayed: bool = False):
    """Gated delta rule in the page's form; alpha, beta: [B, N, h1-h0] scalars. With
    erase_decayed the erase term is decayed too (the GatedDeltaNet form
    M_t = alpha_t M_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T).

    Returns (o [B, N, H, d] float64, S_out [B, h1-h0, d, d] float64, key-major, i.e. the
    transpose of the page's d_v x d_k state).
    """
    q, k, v, a, be = _f32(q), _f32(k), _f32(v), _f32(alpha), _f32(beta)
    B, N, H, d = q.shape
    h0, h1 = heads if heads is not None else (0, H)
    o = np.full((B, N, H, d), np.nan) if out is None else out
    S_out = np.zeros((B, h1 - h0, d, d))
    s0 = None if S0 is None else _f64(S0)
    rc = _load().oracle_delta(_p(q, _f32p), _p(k, _f32p), _p(v, _f32p), _p(a, _f32p),
                              _p(be, _f32p), None if s0 is None else _p(s0, _f64p),
                              _p(o, _f64p), _p(S_out, _f64p), B, N, H, d, h0, h1, float(scale),
                              int(bool(erase_decayed)))
    _check(rc, "delta")
    return o, S_out


def hybrid(q, k, v, alpha, beta, *, P: int, n_swa: int, n_dswa: int, n_gla: int,
           W_swa: int, W_dswa: int, dil: int, gla_delta: int = 0,
           scale_softmax: float, scale_gla: float = 1.0, rows=None):
    """Per-head split (SWA heads, then DSWA heads, then GLA heads), outputs concatenated by
    head. The pages only say that the three branches are mixed; the head split is the
    declared reading. GLA rows are always computed in full (the recurrence needs every
    token); ``rows`` restricts the softmax heads only."""
    q32, k32, v32 = _f32(q), _f32(k), _f32(v)
    B, N, H, d = q32.shape
    assert n_swa + n_dswa + n_gla == H
    o = np.full((B, N, H, d), np.nan)
    if n_swa:
        swa(q32, k32, v32, P, W_swa, scale_softmax, heads=(0, n_swa), rows=rows, out=o)
    if n_dswa:
        dswa(q32, k32, v32, P, W_dswa, dil, scale_softmax, heads=(n_swa, n_swa + n_dswa),
             rows=rows, out=o)
    S = None
    if n_gla:
        hg = (n_swa + n_dswa, H)
        if gla_delta:  # 1: the page's delta rule; 2: its decayed-erase form
            _, S = delta(q32, k32, v32, alpha, beta, scale_gla, heads=hg, out=o,
                         erase_decayed=int(gla_delta) == 2)
        else:
            _, S = gla(q32, k32, v32, alpha, scale_gla, heads=hg, out=o)
    return o, S


def softmax_bwd(q, k, v, dout, P: int, W: int, scale: float, dil: int = 1,
                dilated: bool = False, heads=None):
    """Reverse mode of swa (dilated=False) / dswa: the gradients (dq, dk, dv) of
    L = sum(dout * o) for the heads (h0, h1); other heads are zero. float64 [B, N, H, d]."""
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f64(dout)
    B, N, H, d = q.shape
    h0, h1 = heads if heads is not None else (0, H)
    dq, dk, dv = (np.zeros((B, N, H, d)) for _ in range(3))
    rc = _load().oracle_softmax_bwd(_p(q, _f32p), _p(k, _f32p), _p(v, _f32p), _p(do, _f64p),
                                    _p(dq, _f64p), _p(dk, _f64p), _p(dv, _f64p), B, N, H, d, h0,
                                    h1, P, W, dil, int(bool(dilated)), float(scale))
    _check(rc, "softmax_bwd")
    return dq, dk, dv


def gla_bwd(q, k, v, alpha, dout, scale: float = 1.0, S0=None, heads=None):
    """Reverse mode of gla: (dq, dk, dv, dalpha, dS0) of L = sum(dout * o)."""
    q, k, v, a, do = _f32(q), _f32(k), _f32(v), _f32(alpha), _f64(dout)
    B, N, H, d = q.shape
    h0, h1 = heads if heads is not None else (0, H)
    dq, dk, dv = (np.zeros((B, N, H, d)) for _ in range(3))
    da = np.zeros((B, N, h1 - h0, d))
    dS0 = np.zeros((B, h1 - h0, d, d))
    s0 = None if S0 is None else _f64(S0)
    rc = _load().oracle_gla_bwd(_p(q, _f32p), _p(k, _f32p), _p(v, _f32p), _p(a, _f32p),
                                None if s0 is None else _p(s0, _f64p), _p(do, _f64p),
                                _p(dq, _f64p), _p(dk, _f64p), _p(dv, _f64p), _p(da, _f64p),
                                _p(dS0, _f64p), B, N, H, d, h0, h1, float(scale))
    _check(rc, "gla_bwd")
    return dq, dk, dv, da, dS0


def delta_bwd(q, k, v, alpha, beta, dout, scale: float = 1.0, S0=None, heads=None,
              erase_decayed: bool = False):
    """Reverse mode of delta: (dq, dk, dv, dalpha, dbeta, dS0) of L = sum(dout * o)."""
    q, k, v, a, be, do = _f32(q), _f32(k), _f32(v), _f32(alpha), _f32(beta), _f64(dout)
    B, N, H, d = q.shape
    h0, h1 = heads if heads is not None else (0, H)
    dq, dk, dv = (np.zeros((B, N, H, d)) for _ in range(3))
    da, db = np.zeros((B, N, h1 - h0)), np.zeros((B, N, h1 - h0))
    dS0 = np.zeros((B, h1 - h0, d, d))
    s0 = None if S0 is None else _f64(S0)
    rc = _load().oracle_delta_bwd(_p(q, _f32p), _p(k, _f32p), _p(v, _f32p), _p(a, _f32p),
                                  _p(be, _f32p), None if s0 is None else _p(s0, _f64p),
                                  _p(do, _f64p), _p(dq, _f64p), _p(dk, _f64p), _p(dv, _f64p),
                                  _p(da, _f64p), _p(db, _f64p), _p(dS0, _f64p), B, N, H, d, h0,
                                  h1, float(scale), int(bool(erase_decayed)))
    _check(rc, "delta_bwd")
    return dq, dk, dv, da, db, dS0


def proj(x, w, rows=None, sigmoid_cols=None, bias=None) -> np.ndarray:
    """The projections (q = W_Q x, ..., beta = sigmoid(W_beta x)) as one product: x [..., K]
    (M rows), w [N, K] -> y [rows, N] float64, y = x w^T with columns in sigmoid_cols = (c0, c1)
    passed through the logistic sigmoid. rows: indices of the rows of x to compute (all if
    None). bias: optional [N] offsets added to every row before the sigmoid."""
    x = _f32(x)
    K = x.shape[-1]
    x2 = x.reshape(-1, K)
    w = _f32(w)
    N = w.shape[0]
    if w.shape[1] != K:
        raise ValueError("w must be [N, K]")
    r, nr = _rows(rows)
    R = nr if r is not None else x2.shape[0]
    y = np.empty((R, N))
    c0, c1 = sigmoid_cols if sigmoid_cols is not None else (0, 0)
    b = None if bias is None else _f32(bias)
    if b is not None and b.shape != (N,):
        raise ValueError("bias must be [N]")
    rc = _load().oracle_proj(_p(x2, _f32p), _p(w, _f32p), None if b is None else _p(b, _f32p),
                             x2.shape[0], N, K, None if r is None else _p(r, _i64p), nr, c0, c1,
                             _p(y, _f64p))
    _check(rc, "proj")
    return y


def visible(t, s, P: int, W: int, dil: int = 1, dilated: bool = False) -> np.ndarray:
    """The oracle's visibility predicate, elementwise over index arrays t (query) and s (key)."""
    t = np.ascontiguousarray(t, dtype=np.int64).ravel()
    s = np.ascontiguousarray(s, dtype=np.int64).ravel()
    out = np.zeros(t.size, dtype=np.uint8)
    _load().oracle_visible(_p(t, _i64p), _p(s, _i64p), t.size, P, W, dil, int(dilated),
                           _p(out, _u8p))
    return out.astype(bool)
