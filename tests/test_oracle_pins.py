"""Pins for the fp64 CPU oracle (CPU only).

Each test compares the oracle with something other than itself: a closed form written out
independently here, a special case that reduces to textbook attention, the DSWA reshape
identity stated on the Kairos paper-read (section 2, second pillar, DSWA paragraph), exact
brute-force mask counts from the window described in words, and the geometric-decay claim of
the error bound (paper-read section 2, Theorem 2; ai-papers.net summary, "error accumulation"
section). Sizes are tiny so fp64 agreement is near machine precision.
"""
import itertools
import math

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(12345)


def rnd(*shape, scale=1.0):
    return (RNG.standard_normal(shape) * scale).astype(np.float32)


def gates(*shape, lo=0.3, hi=0.999):
    return RNG.uniform(lo, hi, size=shape).astype(np.float32)


def relerr(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ----------------------------------------------------------------------------- GLA


def gla_closed_form(q, k, v, a, scale, S0=None):
    """o_t = scale * [ sum_{s<=t} sum_i q_ti k_si prod_{r=s+1..t} a_ri v_s
                      + sum_i q_ti prod_{r<=t} a_ri S0_i ]   (quadratic, masked form)."""
    q, k, v, a = (x.astype(np.float64) for x in (q, k, v, a))
    N, d = q.shape
    o = np.zeros((N, d))
    for t in range(N):
        for s in range(t + 1):
            decay = np.prod(a[s + 1:t + 1], axis=0) if s < t else np.ones(d)
            o[t] += np.sum(q[t] * k[s] * decay) * v[s]
        if S0 is not None:
            o[t] += (q[t] * np.prod(a[:t + 1], axis=0)) @ S0
    return scale * o


GLA_LIM = 64.0  # the bf16 kernel's bound on |b_t - b_m| (bits) for one span's decayed operands


def gla_chunked_middle_reference(q, k, v, a, scale, C, S0, dtype=np.float64, fallback=True,
                                 levels=None):
    """The chunked GLA algebra of the bf16 kernel, written out. Spans of C tokens; per span
    b_t = cumulative log2 gate (log2 clamped at -200), m = n // 2 the middle token,
    Qi_t = q_t 2^(b_t - b_m), Ki_s = k_s 2^(b_m - b_s),
    o_t = scale [Qi_t (2^(b_m) S_0) + sum_{s<=t} (Qi_t . Ki_s) v_s],
    S_end = 2^(b_n - b_m) (2^(b_m) S_0 + Ki^T V). With `fallback`, a span whose decayed operands
    would need |b_t - b_m| > GLA_LIM bits in some key dim is redone as 16-token sub-spans, and a
    sub-span that still fails token by token. Evaluated in `dtype`; `levels` (a list) collects
    the granularity used for each span."""
    q, k, v, a = (x.astype(dtype) for x in (q, k, v, a))
    N, d = q.shape
    S = S0.astype(dtype).copy()
    o = np.zeros((N, d), dtype=dtype)

    def span(c0, n, lvl):
        nonlocal S
        with np.errstate(over="ignore", invalid="ignore", divide="ignore"):
            b = np.cumsum(np.maximum(np.log2(a[c0:c0 + n]), dtype(-200)), axis=0).astype(dtype)
            bm = b[n // 2]
            if fallback and n > 1 and np.max(np.abs(b - bm)) > GLA_LIM:
                sub = 16 if (lvl == 0 and C > 16) else 1
                for u in range(0, n, sub):
                    span(c0 + u, min(sub, n - u), 1 if sub == 16 else 2)
                return
            if levels is not None:
                levels.append(lvl)
            Qi = q[c0:c0 + n] * np.exp2(b - bm)
            Ki = k[c0:c0 + n] * np.exp2(bm - b)
            Sm = np.exp2(bm)[:, None] * S
            A = np.tril(Qi @ Ki.T)
            o[c0:c0 + n] = scale * (Qi @ Sm + A @ v[c0:c0 + n])
            S = np.exp2(b[-1] - bm)[:, None] * (Sm + Ki.T @ v[c0:c0 + n])

    for c0 in range(0, N, C):
        span(c0, min(C, N - c0), 0)
    return o, S


@pytest.mark.parametrize("C", [16, 32, 64])
def test_gla_equals_middle_reference_chunked_form(C):
    """The bf16 kernel's chunked algebra equals the oracle's token recurrence (fp64)."""
    N, d = 150, 8
    q, k, v = rnd(N, d), rnd(N, d), rnd(N, d)
    a = gates(N, d, lo=0.5)
    S0 = RNG.standard_normal((d, d))
    o, S = oracle.gla(q[None, :, None], k[None, :, None], v[None, :, None], a[None, :, None],
                      scale=0.8, S0=S0[None, None])
    lv = []
    ref, Sref = gla_chunked_middle_reference(q, k, v, a, 0.8, C, S0, levels=lv)
    assert set(lv) == {0}  # these gates never need the finer spans
    assert relerr(o[0, :, 0], ref) < 1e-11
    assert relerr(S[0, 0], Sref) < 1e-11


def test_single_middle_reference_overflows_without_the_fallback():
    """In fp32 one middle reference per 64-token chunk overflows once the product of 32
    consecutive gates falls below 2^-126: the reason the kernel checks each span's range."""
    N, d, C = 64, 4, 64
    q, k, v = rnd(N, d), rnd(N, d), rnd(N, d)
    S0 = np.zeros((d, d))
    outside = np.full((N, d), 0.05, dtype=np.float32)    # 32 * log2(0.05) = -138.3
    o_out, _ = gla_chunked_middle_reference(q, k, v, outside, 1.0, C, S0, dtype=np.float32,
                                            fallback=False)
    assert not np.all(np.isfinite(o_out))


def _small_gates(kind, N, d):
    if kind == "const0.05":
        return np.full((N, d), 0.05, dtype=np.float32)
    if kind == "uniform":
        return RNG.uniform(1e-4, 0.1, size=(N, d)).astype(np.float32)
    if kind == "sigmoid-3":
        z = RNG.standard_normal((N, d)) - 3.0
        return (1.0 / (1.0 + np.exp(-z))).astype(np.float32)
    # mixed: mostly ordinary gates with exact zeros, 1e-30 and 1e-12 sprinkled in
    a = RNG.uniform(0.3, 0.999, size=(N, d)).astype(np.float32)
    idx = RNG.choice(N * d, size=N * d // 10, replace=False)
    a.flat[idx[0::3]] = 0.0
    a.flat[idx[1::3]] = 1e-30
    a.flat[idx[2::3]] = 1e-12
    return a


@pytest.mark.parametrize("C", [16, 32, 64])
@pytest.mark.parametrize("kind", ["const0.05", "uniform", "sigmoid-3", "mixed"])
def test_ranged_chunked_form_is_finite_and_exact_for_small_gates(C, kind):
    """With the per-span range check and the 16-token / single-token fallback, the chunked
    algebra evaluated in fp32 stays finite and equals the oracle's fp64 recurrence (to fp32
    rounding) for gates down to 0, which are valid forget gates (GLA paragraph: alpha_t in
    (0, 1))."""
    N, d = 4 * C + 9, 8
    q, k, v = rnd(N, d), rnd(N, d), rnd(N, d)
    a = _small_gates(kind, N, d)
    S0 = RNG.standard_normal((d, d))
    o, S = oracle.gla(q[None, :, None], k[None, :, None], v[None, :, None], a[None, :, None],
                      scale=0.8, S0=S0[None, None])
    lv = []
    got, Sg = gla_chunked_middle_reference(q, k, v, a, 0.8, C, S0, dtype=np.float32, levels=lv)
    assert np.all(np.isfinite(got)) and np.all(np.isfinite(Sg))
    assert relerr(got, o[0, :, 0]) < 1e-5
    assert relerr(Sg, S[0, 0]) < 1e-5
    if kind == "const0.05" and C > 16:
        # full chunk-level spans fail, their 16-token sub-spans pass (the 9-token tail span is
        # short enough for level 0)
        assert lv.count(0) == 1 and lv.count(1) == 4 * (C // 16) and 2 not in lv
    if kind == "mixed":
        assert 2 in lv  # zeros need single-token spans


@pytest.mark.parametrize("N,d,with_s0", [(1, 4, False), (37, 8, False), (24, 6, True)])
def test_gla_recurrence_equals_quadratic_closed_form(N, d, with_s0):
    B, H = 2, 3
    q, k, v = rnd(B, N, H, d), rnd(B, N, H, d), rnd(B, N, H, d)
    a = gates(B, N, 2, d)
    S0 = RNG.standard_normal((B, 2, d, d)) if with_s0 else None
    o, S = oracle.gla(q, k, v, a, scale=0.7, S0=S0, heads=(1, 3))
    assert np.all(np.isnan(o[:, :, 0]))          # heads outside the range untouched
    for b, hg in itertools.product(range(B), range(2)):
        h = 1 + hg
        ref = gla_closed_form(q[b, :, h], k[b, :, h], v[b, :, h], a[b, :, hg], 0.7,
                              None if S0 is None else S0[b, hg])
        assert relerr(o[b, :, h], ref) < 1e-12


def test_gla_unit_gate_is_causal_linear_attention():
    B, N, H, d = 1, 30, 2, 5
    q, k, v = rnd(B, N, H, d), rnd(B, N, H, d), rnd(B, N, H, d)
    o, S = oracle.gla(q, k, v, np.ones((B, N, H, d), np.float32), scale=1.0)
    for h in range(H):
        kv = np.cumsum(np.einsum("ni,nj->nij", k[0, :, h].astype(np.float64),
                                 v[0, :, h].astype(np.float64)), axis=0)
        ref = np.einsum("ni,nij->nj", q[0, :, h].astype(np.float64), kv)
        assert relerr(o[0, :, h], ref) < 1e-12
        assert relerr(S[0, h], kv[-1]) < 1e-12


def test_gla_state_carry_splits_sequence():
    """Running the recurrence on [0, N) equals running [0, m) then [m, N) from its end state."""
    B, N, H, d, m = 1, 40, 1, 6, 17
    q, k, v, a = rnd(B, N, H, d), rnd(B, N, H, d), rnd(B, N, H, d), gates(B, N, H, d)
    o, S = oracle.gla(q, k, v, a)
    o1, S1 = oracle.gla(q[:, :m], k[:, :m], v[:, :m], a[:, :m])
    o2, S2 = oracle.gla(q[:, m:], k[:, m:], v[:, m:], a[:, m:], S0=S1)
    assert relerr(np.concatenate([o1, o2], axis=1), o) < 1e-13
    assert relerr(S2, S) < 1e-13


# ----------------------------------------------------------------------------- delta rule


def delta_standard_form(q, k, v, a, be, scale, M0=None):
    """GatedDeltaNet-style recurrence M_t = a~ M (I - b~ k k^T) + b~ v~ k^T with b~ = be/a and
    v~ = a v, o_t = scale M_t q_t. Algebraically equal to the page's four lines."""
    q, k, v, a, be = (x.astype(np.float64) for x in (q, k, v, a, be))
    N, d = q.shape
    M = np.zeros((d, d)) if M0 is None else M0.copy()
    o = np.zeros((N, d))
    for t in range(N):
        bt = be[t] / a[t]
        vt = a[t] * v[t]
        M = a[t] * M @ (np.eye(d) - bt * np.outer(k[t], k[t])) + bt * np.outer(vt, k[t])
        o[t] = scale * M @ q[t]
    return o, M


def delta_chunked(q, k, v, a, be, scale, C, M0=None, decayed=False):
    """Chunked (UT / triangular-solve) form of the page's delta rule, derived by unrolling the
    recurrence inside a chunk:  gamma_t = prod_{r<=t} a_r,
       (I + T) U = diag(be) V - diag(be * gamma_{t-1}) K M0^T,  T_ts = be_t g_{t-1}/g_s (k_t.k_s)
       o_t = gamma_t M0 q_t + sum_{s<=t} gamma_t/gamma_s (q_t.k_s) u_s
       M_C = gamma_C M0 + sum_s gamma_C/gamma_s u_s k_s^T.
    With the decayed erase (u_t = be_t (v_t - a_t M_{t-1} k_t)) every gamma_{t-1} above becomes
    gamma_t."""
    q, k, v, a, be = (x.astype(np.float64) for x in (q, k, v, a, be))
    N, d = q.shape
    M = np.zeros((d, d)) if M0 is None else M0.copy()
    o = np.zeros((N, d))
    for c0 in range(0, N, C):
        sl = slice(c0, min(c0 + C, N))
        Q, K, V, A, Bt = q[sl], k[sl], v[sl], a[sl], be[sl]
        n = Q.shape[0]
        g = np.cumprod(A)
        gprev = g.copy() if decayed else np.concatenate([[1.0], g[:-1]])
        T = np.zeros((n, n))
        for t in range(n):
            for s in range(t):
                T[t, s] = Bt[t] * gprev[t] / g[s] * (K[t] @ K[s])
        rhs = Bt[:, None] * V - (Bt * gprev)[:, None] * (K @ M.T)
        U = np.linalg.solve(np.eye(n) + T, rhs)
        G = np.tril(g[:, None] / g[None, :])
        o[sl] = scale * (g[:, None] * (Q @ M.T) + (G * (Q @ K.T)) @ U)
        M = g[-1] * M + (U * (g[-1] / g)[:, None]).T @ K
    return o, M


def test_delta_equals_gated_deltanet_form():
    B, N, H, d = 1, 33, 2, 6
    q, v = rnd(B, N, H, d), rnd(B, N, H, d)
    k = rnd(B, N, H, d)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    a, be = gates(B, N, H, lo=0.5), gates(B, N, H, lo=0.05, hi=0.95)
    M0 = RNG.standard_normal((B, H, d, d))
    o, S = oracle.delta(q, k, v, a, be, scale=0.9, S0=M0)
    for h in range(H):
        ref, Mref = delta_standard_form(q[0, :, h], k[0, :, h], v[0, :, h], a[0, :, h],
                                        be[0, :, h], 0.9, M0[0, h].T)
        assert relerr(o[0, :, h], ref) < 1e-11
        assert relerr(S[0, h].T, Mref) < 1e-11


@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_delta_equals_chunked_ut_form(C):
    B, N, H, d = 1, 50, 1, 8
    q, v = rnd(B, N, H, d), rnd(B, N, H, d)
    k = rnd(B, N, H, d)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    a, be = gates(B, N, H, lo=0.6), gates(B, N, H, lo=0.05, hi=0.95)
    M0 = RNG.standard_normal((B, H, d, d))
    o, S = oracle.delta(q, k, v, a, be, scale=1.0, S0=M0)
    ref, Mref = delta_chunked(q[0, :, 0], k[0, :, 0], v[0, :, 0], a[0, :, 0], be[0, :, 0],
                              1.0, C, M0[0, 0].T)
    assert relerr(o[0, :, 0], ref) < 1e-10
    assert relerr(S[0, 0].T, Mref) < 1e-10


def test_delta_beta_zero_keeps_state():
    B, N, H, d = 1, 20, 1, 5
    q, k, v = rnd(B, N, H, d), rnd(B, N, H, d), rnd(B, N, H, d)
    M0 = RNG.standard_normal((B, H, d, d))
    # alpha == 1: the state is unchanged (the literal form subtracts and re-adds v_old k^T,
    # so equality holds to fp64 rounding, not bit for bit).
    o, S = oracle.delta(q, k, v, np.ones((B, N, H), np.float32), np.zeros((B, N, H), np.float32),
                        S0=M0)
    assert relerr(S, M0) < 1e-14
    assert relerr(o[0, :, 0], q[0, :, 0].astype(np.float64) @ M0[0, 0]) < 1e-14
    # general alpha: the state only decays, M_t = prod_{r<=t} a_r M0.
    a = gates(B, N, H)
    o, S = oracle.delta(q, k, v, a, np.zeros((B, N, H), np.float32), S0=M0)
    g = np.cumprod(a[0, :, 0].astype(np.float64))
    assert relerr(o[0, :, 0], g[:, None] * (q[0, :, 0].astype(np.float64) @ M0[0, 0])) < 1e-13
    assert relerr(S[0, 0], g[-1] * M0[0, 0]) < 1e-13


def test_delta_exact_associative_recall():
    """alpha = beta = 1, orthonormal keys: after writing (k_j, v_j), M k_j = v_j."""
    d = 8
    Qm, _ = np.linalg.qr(RNG.standard_normal((d, d)))
    k = Qm.T[None, :, None, :].astype(np.float32)           # token j writes key row j
    kk = k[0, :, 0].astype(np.float64)
    v = rnd(1, d, 1, d)
    o, S = oracle.delta(k, k, v, np.ones((1, d, 1), np.float32), np.ones((1, d, 1), np.float32))
    M = S[0, 0].T
    # keys stored in fp32 are orthonormal to ~1e-7, so recall is exact to that level
    assert relerr(M @ kk.T, v[0, :, 0].astype(np.float64).T) < 1e-5
    # o_t = M_t q_t with q_t = k_t reads back the value just written
    assert relerr(o[0, :, 0], v[0, :, 0].astype(np.float64)) < 1e-5


# ----------------------------------------------------------------------------- delta, decayed erase


def pow2_gates(*shape):
    """Forget gates that are powers of two, so that v / alpha and alpha * beta are exact."""
    return RNG.choice(np.array([1.0, 0.5, 0.25], np.float32), size=shape)


def test_decayed_erase_equals_page_form_with_rescaled_inputs():
    # alpha M (I - b k k^T) + b v k^T = alpha M + (alpha b) ((v / alpha) - M k) k^T
    B, N, H, d = 2, 29, 2, 5
    q, v = rnd(B, N, H, d), rnd(B, N, H, d)
    k = rnd(B, N, H, d)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    a, be = pow2_gates(B, N, H), gates(B, N, H, lo=0.05, hi=0.95)
    M0 = RNG.standard_normal((B, H, d, d))
    o, S = oracle.delta(q, k, v, a, be, scale=0.7, S0=M0, erase_decayed=True)
    o2, S2 = oracle.delta(q, k, v / a[..., None], a, a * be, scale=0.7, S0=M0)
    assert relerr(o, o2) < 1e-12
    assert relerr(S, S2) < 1e-12


def test_decayed_erase_equals_gated_deltanet_standard_form():
    B, N, H, d = 1, 31, 1, 6
    q, v = rnd(B, N, H, d), rnd(B, N, H, d)
    k = rnd(B, N, H, d)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    a, be = pow2_gates(B, N, H), gates(B, N, H, lo=0.05, hi=0.95)
    M0 = RNG.standard_normal((B, H, d, d))
    o, S = oracle.delta(q, k, v, a, be, scale=1.0, S0=M0, erase_decayed=True)
    # delta_standard_form(a, b', v') runs M = a M (I - (b'/a) k k^T) + (b'/a)(a v') k^T
    ref, Mref = delta_standard_form(q[0, :, 0], k[0, :, 0], v[0, :, 0] / a[0, :, 0, None],
                                    a[0, :, 0], a[0, :, 0] * be[0, :, 0], 1.0, M0[0, 0].T)
    assert relerr(o[0, :, 0], ref) < 1e-11
    assert relerr(S[0, 0].T, Mref) < 1e-11


def test_decayed_erase_with_unit_gate_is_the_page_form():
    B, N, H, d = 1, 25, 1, 6
    q, k, v = rnd(B, N, H, d), rnd(B, N, H, d), rnd(B, N, H, d)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    ones, be = np.ones((B, N, H), np.float32), gates(B, N, H, lo=0.05, hi=0.95)
    o1, S1 = oracle.delta(q, k, v, ones, be, erase_decayed=True)
    o2, S2 = oracle.delta(q, k, v, ones, be)
    assert relerr(o1, o2) < 1e-13 and relerr(S1, S2) < 1e-13


@pytest.mark.parametrize("C", [1, 8, 64])
def test_decayed_erase_equals_its_chunked_ut_form(C):
    B, N, H, d = 1, 70, 1, 8
    q, v = rnd(B, N, H, d), rnd(B, N, H, d)
    k = rnd(B, N, H, d)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    a, be = gates(B, N, H, lo=0.6), gates(B, N, H, lo=0.05, hi=0.95)
    M0 = RNG.standard_normal((B, H, d, d))
    o, S = oracle.delta(q, k, v, a, be, scale=1.0, S0=M0, erase_decayed=True)
    ref, Mref = delta_chunked(q[0, :, 0], k[0, :, 0], v[0, :, 0], a[0, :, 0], be[0, :, 0], 1.0,
                              C, M0[0, 0].T, decayed=True)
    assert relerr(o[0, :, 0], ref) < 1e-10
    assert relerr(S[0, 0].T, Mref) < 1e-10
    # and the two forms really differ when alpha < 1
    o_page, _ = oracle.delta(q, k, v, a, be, scale=1.0, S0=M0)
    assert relerr(o_page, o) > 1e-3


# ----------------------------------------------------------------------------- softmax branches


def dense_masked_softmax(q, k, v, mask, scale):
    s = scale * q.astype(np.float64) @ k.astype(np.float64).T
    s = np.where(mask, s, -np.inf)
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v.astype(np.float64)


def test_swa_full_window_is_frame_causal_attention():
    B, F, P, H, d = 2, 5, 7, 2, 8
    N = F * P
    q, k, v = rnd(B, N, H, d), rnd(B, N, H, d), rnd(B, N, H, d)
    o = oracle.swa(q, k, v, P=P, W=F, scale=0.3)
    fr = np.arange(N) // P
    mask = fr[None, :] <= fr[:, None]
    for b, h in itertools.product(range(B), range(H)):
        ref = dense_masked_softmax(q[b, :, h], k[b, :, h], v[b, :, h], mask, 0.3)
        assert relerr(o[b, :, h], ref) < 1e-13


def test_swa_single_token_frames_is_causal_attention():
    N, d = 23, 6
    q, k, v = rnd(1, N, 1, d), rnd(1, N, 1, d), rnd(1, N, 1, d)
    o = oracle.swa(q, k, v, P=1, W=N + 5, scale=1 / math.sqrt(d))
    ref = dense_masked_softmax(q[0, :, 0], k[0, :, 0], v[0, :, 0],
                               np.tril(np.ones((N, N), bool)), 1 / math.sqrt(d))
    assert relerr(o[0, :, 0], ref) < 1e-13


def test_swa_window_equals_dense_banded_mask():
    F, P, d, W = 9, 4, 8, 3
    N = F * P
    q, k, v = rnd(1, N, 1, d), rnd(1, N, 1, d), rnd(1, N, 1, d)
    o = oracle.swa(q, k, v, P=P, W=W, scale=0.5)
    fr = np.arange(N) // P
    lag = fr[:, None] - fr[None, :]
    ref = dense_masked_softmax(q[0, :, 0], k[0, :, 0], v[0, :, 0], (lag >= 0) & (lag < W), 0.5)
    assert relerr(o[0, :, 0], ref) < 1e-13


def test_dswa_dilation_one_is_swa():
    F, P, H, d = 10, 6, 2, 8
    N = F * P
    q, k, v = rnd(1, N, H, d), rnd(1, N, H, d), rnd(1, N, H, d)
    for W in (1, 2, 4, 11):
        assert np.array_equal(oracle.dswa(q, k, v, P, W, 1, 0.4), oracle.swa(q, k, v, P, W, 0.4))


@pytest.mark.parametrize("dil,W", [(2, 2), (3, 2), (3, 4)])
def test_dswa_equals_swa_on_page_reshape(dil, W):
    """Page identity: DSWA = SWA after reshaping (B, F*L, D) -> (B*dil, F/dil*L, D) with frame
    f going to group f mod dil (interleaved groups), then undoing the reshape."""
    B, F, P, H, d = 2, 12, 5, 2, 8
    N = F * P
    q, k, v = rnd(B, N, H, d), rnd(B, N, H, d), rnd(B, N, H, d)
    o = oracle.dswa(q, k, v, P, W, dil, 0.35)

    def fwd(x):   # [B, F*P, H, d] -> [B*dil, F/dil*P, H, d]
        x = x.reshape(B, F // dil, dil, P, H, d).transpose(0, 2, 1, 3, 4, 5)
        return np.ascontiguousarray(x.reshape(B * dil, (F // dil) * P, H, d))

    og = oracle.swa(fwd(q), fwd(k), fwd(v), P, W, 0.35)
    back = og.reshape(B, dil, F // dil, P, H, d).transpose(0, 2, 1, 3, 4, 5).reshape(B, N, H, d)
    assert relerr(o, back) < 1e-13


def _visible_frames(f, W, dil, F):
    """The window in words: frames f, f-dil, ..., f-(W-1)*dil that exist."""
    return {f - j * dil for j in range(W) if f - j * dil >= 0}


@pytest.mark.parametrize("W,dil", [(1, 1), (2, 1), (3, 1), (2, 2), (4, 3), (20, 1)])
def test_mask_probe_counts_are_exact(W, dil):
    """q = k = 0 makes every visible key weigh the same; v = one-hot(frame of key) turns
    o_t into the fraction of visible keys per frame, which must equal |frame|/|window|."""
    F, P, d = 9, 5, 16
    N = F * P
    q = np.zeros((1, N, 1, d), np.float32)
    v = np.zeros((1, N, 1, d), np.float32)
    v[0, np.arange(N), 0, np.arange(N) // P] = 1.0
    o = oracle.dswa(q, q, v, P, W, dil, 1.0)[0, :, 0]
    for t in range(N):
        fr = _visible_frames(t // P, W, dil, F)
        expect = np.zeros(d)
        for g in fr:
            expect[g] = 1.0 / len(fr)
        assert np.array_equal(o[t] != 0, expect != 0), (t, fr)
        assert np.max(np.abs(o[t] - expect)) < 1e-15


def test_visible_predicate_matches_window_in_words():
    F, P = 13, 3
    N = F * P
    t, s = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    for W, dil in [(1, 1), (3, 1), (4, 3), (2, 5)]:
        vis = oracle.visible(t, s, P, W, dil, dilated=True).reshape(N, N)
        ref = np.array([[(ss // P) in _visible_frames(tt // P, W, dil, F) for ss in range(N)]
                        for tt in range(N)])
        assert np.array_equal(vis, ref)
        if dil == 1:
            assert np.array_equal(oracle.visible(t, s, P, W).reshape(N, N), ref)


def test_softmax_shift_invariance_and_constant_values():
    F, P, d = 6, 4, 8
    N = F * P
    q, k, v = rnd(1, N, 1, d), rnd(1, N, 1, d), rnd(1, N, 1, d)
    o = oracle.dswa(q, k, v, P, 3, 2, 0.5)
    # append a coordinate with q = c/0.5 and k = 1: every score of a row shifts by c
    c = 3.25
    q2 = np.concatenate([q, np.full((1, N, 1, 1), c / 0.5, np.float32)], axis=-1)
    k2 = np.concatenate([k, np.ones((1, N, 1, 1), np.float32)], axis=-1)
    v2 = np.concatenate([v, np.zeros((1, N, 1, 1), np.float32)], axis=-1)
    o2 = oracle.dswa(q2, k2, v2, P, 3, 2, 0.5)
    assert relerr(o2[..., :d], o) < 1e-13
    oc = oracle.swa(q, k, np.full_like(v, 1.75), P, 2, 0.5)
    assert np.max(np.abs(oc - 1.75)) < 1e-14


# ----------------------------------------------------------------------------- decay claims


def test_gla_perturbation_decays_geometrically():
    """Gates <= rho: a change of v at token t0 changes o_t by at most
    scale * |q_t| * |dS_t0|_F * rho^(t - t0)."""
    B, N, H, d, t0, rho = 1, 60, 1, 6, 10, 0.8
    q, k, v = rnd(B, N, H, d), rnd(B, N, H, d), rnd(B, N, H, d)
    a = gates(B, N, H, d, lo=0.2, hi=rho)
    o, _ = oracle.gla(q, k, v, a)
    v2 = v.copy()
    v2[0, t0, 0] += rnd(d)
    o2, _ = oracle.gla(q, k, v2, a)
    dv = v2[0, t0, 0].astype(np.float64) - v[0, t0, 0].astype(np.float64)
    dS0 = np.linalg.norm(np.outer(k[0, t0, 0].astype(np.float64), dv))
    assert np.all(o2[0, :t0] == o[0, :t0])
    for t in range(t0, N):
        bound = np.linalg.norm(q[0, t, 0]) * dS0 * rho ** (t - t0)
        assert np.linalg.norm(o2[0, t, 0] - o[0, t, 0]) <= bound * (1 + 1e-9) + 1e-300


def test_delta_error_stays_below_contraction_bound():
    """Unit keys: the delta transition is alpha I - beta k k^T with norm
    rho_t = max(alpha_t, |alpha_t - beta_t|) < 1. With a perturbation of at most xi on every
    step, the state error stays below xi / (1 - rho) (the bound's recurrence e_t <= rho e_{t-1}
    + xi)."""
    B, N, H, d = 1, 80, 1, 6
    q, v = rnd(B, N, H, d), rnd(B, N, H, d)
    k = rnd(B, N, H, d)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    a, be = gates(B, N, H, lo=0.3, hi=0.85), gates(B, N, H, lo=0.05, hi=0.9)
    dv = rnd(B, N, H, d, scale=1e-2)
    rho = float(np.max(np.maximum(a, np.abs(a - be))))
    xi = float(np.max(be[..., None] * np.abs(dv)) * math.sqrt(d))
    err_prev = 0.0
    for n in range(1, N + 1, 7):
        _, S1 = oracle.delta(q[:, :n], k[:, :n], v[:, :n], a[:, :n], be[:, :n])
        _, S2 = oracle.delta(q[:, :n], k[:, :n], v[:, :n] + dv[:, :n], a[:, :n], be[:, :n])
        err = np.linalg.norm(S2[0, 0] - S1[0, 0], 2)
        assert err <= xi / (1 - rho) * (1 + 1e-9)
        err_prev = err
    assert err_prev > 0


# ----------------------------------------------------------------------------- hybrid head split


@pytest.mark.parametrize("gla_delta", [0, 1, 2])
def test_hybrid_head_slices_equal_branches_on_those_heads_alone(gla_delta):
    """The hybrid (per-head split, outputs concatenated by head) places each branch on its own
    head range: every head slice equals the branch run on a tensor holding only those heads, so
    a wrong head offset, a swapped branch or a branch reading another head's data fails here."""
    B, F, P, d = 2, 5, 6, 8
    n_swa, n_dswa, n_gla = 2, 1, 2
    H, N = n_swa + n_dswa + n_gla, F * P
    q, k, v = rnd(B, N, H, d), rnd(B, N, H, d), rnd(B, N, H, d)
    if gla_delta:
        kn = k[:, :, n_swa + n_dswa:]
        k[:, :, n_swa + n_dswa:] = kn / np.linalg.norm(kn, axis=-1, keepdims=True)
        alpha, beta = gates(B, N, n_gla), gates(B, N, n_gla, lo=0.1, hi=0.9)
    else:
        alpha, beta = gates(B, N, n_gla, d), None
    W_swa, W_dswa, dil, sc = 2, 2, 2, d ** -0.5
    o, S = oracle.hybrid(q, k, v, alpha, beta, P=P, n_swa=n_swa, n_dswa=n_dswa, n_gla=n_gla,
                         W_swa=W_swa, W_dswa=W_dswa, dil=dil, gla_delta=gla_delta,
                         scale_softmax=sc, scale_gla=0.5)
    assert np.all(np.isfinite(o))

    def only(x, h0, h1):
        return np.ascontiguousarray(x[:, :, h0:h1])

    hs = (0, n_swa)
    r = oracle.swa(only(q, *hs), only(k, *hs), only(v, *hs), P, W_swa, sc)
    np.testing.assert_array_equal(o[:, :, 0:n_swa], r)
    hd = (n_swa, n_swa + n_dswa)
    r = oracle.dswa(only(q, *hd), only(k, *hd), only(v, *hd), P, W_dswa, dil, sc)
    np.testing.assert_array_equal(o[:, :, hd[0]:hd[1]], r)
    hg = (n_swa + n_dswa, H)
    if gla_delta:
        r, Sr = oracle.delta(only(q, *hg), only(k, *hg), only(v, *hg), alpha, beta, 0.5,
                             erase_decayed=gla_delta == 2)
    else:
        r, Sr = oracle.gla(only(q, *hg), only(k, *hg), only(v, *hg), alpha, 0.5)
    np.testing.assert_array_equal(o[:, :, hg[0]:], r)
    np.testing.assert_array_equal(S, Sr)
    # the three branches really differ on these inputs (the check above is not vacuous)
    r_swa_on_gla = oracle.swa(only(q, *hg), only(k, *hg), only(v, *hg), P, W_swa, sc)
    assert relerr(r_swa_on_gla, o[:, :, hg[0]:]) > 0.1
