"""Pins of the oracle's reverse mode: its gradients against central finite differences of its
own forward (a different computation from the backward formulas).

Inputs lie on a 2^-6 grid and the step is h = 2^-10, so x +/- h is exact in the fp32 the oracle
reads; the finite-difference error is O(h^2) ~ 1e-6.
"""
import numpy as np
import pytest

import oracle

H_STEP = 2.0 ** -10
RNG = np.random.default_rng(777)


def grid(shape, lo=None, hi=None):
    if lo is None:
        x = RNG.standard_normal(shape)
    else:
        x = RNG.uniform(lo, hi, size=shape)
    return (np.round(x * 64) / 64).astype(np.float32)


def fd_grad(loss, arr, idx):
    """Central difference of loss() with respect to arr[idx] (arr is modified in place)."""
    x0 = arr[idx]
    arr[idx] = x0 + H_STEP
    lp = loss()
    arr[idx] = x0 - H_STEP
    lm = loss()
    arr[idx] = x0
    return (lp - lm) / (2 * H_STEP)


def check(loss, arr, grad, n_samples=None):
    idxs = list(np.ndindex(arr.shape))
    if n_samples is not None and len(idxs) > n_samples:
        pick = RNG.choice(len(idxs), size=n_samples, replace=False)
        idxs = [idxs[i] for i in pick]
    fd = np.array([fd_grad(loss, arr, i) for i in idxs])
    an = np.array([grad[i] for i in idxs])
    err = np.linalg.norm(an - fd) / max(np.linalg.norm(fd), 1e-12)
    assert err < 1e-4, f"relative error {err:.2e}"


@pytest.mark.parametrize("dilated,F,P,W,dil", [(False, 4, 3, 2, 1), (True, 6, 2, 2, 2),
                                               (False, 3, 4, 5, 1)])
def test_softmax_backward_matches_finite_differences(dilated, F, P, W, dil):
    B, N, H, d = 1, F * P, 2, 3
    q, k, v = grid((B, N, H, d)), grid((B, N, H, d)), grid((B, N, H, d))
    do = RNG.standard_normal((B, N, H, d))
    scale = 0.75

    def loss():
        if dilated:
            o = oracle.dswa(q, k, v, P, W, dil, scale)
        else:
            o = oracle.swa(q, k, v, P, W, scale)
        return float(np.sum(do * o))

    dq, dk, dv = oracle.softmax_bwd(q, k, v, do, P, W, scale, dil=dil, dilated=dilated)
    for arr, g in ((q, dq), (k, dk), (v, dv)):
        check(loss, arr, g)


def test_softmax_backward_head_range_leaves_other_heads_zero():
    B, N, H, d, P = 1, 8, 3, 2, 2
    q, k, v = grid((B, N, H, d)), grid((B, N, H, d)), grid((B, N, H, d))
    do = RNG.standard_normal((B, N, H, d))
    dq, dk, dv = oracle.softmax_bwd(q, k, v, do, P, 2, 1.0, heads=(1, 2))
    for g in (dq, dk, dv):
        assert np.all(g[:, :, 0] == 0) and np.all(g[:, :, 2] == 0) and np.any(g[:, :, 1] != 0)


@pytest.mark.parametrize("with_s0", [False, True])
def test_gla_backward_matches_finite_differences(with_s0):
    B, N, H, d = 1, 7, 2, 3
    q, k, v = grid((B, N, H, d)), grid((B, N, H, d)), grid((B, N, H, d))
    a = grid((B, N, H, d), 0.5, 0.95)
    S0 = RNG.standard_normal((B, H, d, d)) if with_s0 else None
    do = RNG.standard_normal((B, N, H, d))
    scale = 0.9

    def loss():
        o, _ = oracle.gla(q, k, v, a, scale=scale, S0=S0)
        return float(np.sum(do * o))

    dq, dk, dv, da, dS0 = oracle.gla_bwd(q, k, v, a, do, scale=scale, S0=S0)
    for arr, g in ((q, dq), (k, dk), (v, dv), (a, da)):
        check(loss, arr, g)
    if with_s0:
        check(loss, S0, dS0)


@pytest.mark.parametrize("erase_decayed", [False, True])
def test_delta_backward_matches_finite_differences(erase_decayed):
    B, N, H, d = 1, 6, 2, 3
    q, k, v = grid((B, N, H, d)), grid((B, N, H, d)), grid((B, N, H, d))
    a = grid((B, N, H), 0.5, 0.95)
    be = grid((B, N, H), 0.1, 0.9)
    S0 = RNG.standard_normal((B, H, d, d))
    do = RNG.standard_normal((B, N, H, d))
    scale = 1.1

    def loss():
        o, _ = oracle.delta(q, k, v, a, be, scale=scale, S0=S0, erase_decayed=erase_decayed)
        return float(np.sum(do * o))

    dq, dk, dv, da, db, dS0 = oracle.delta_bwd(q, k, v, a, be, do, scale=scale, S0=S0,
                                               erase_decayed=erase_decayed)
    for arr, g in ((q, dq), (k, dk), (v, dv), (a, da), (be, db), (S0, dS0)):
        check(loss, arr, g)


def test_gla_gate_gradient_equals_log_gate_form():
    """The GLA gate gradient the oracle forms directly, sum_j G_t[i][j] S_{t-1}[i][j], equals the
    log-gate form (1 / alpha_t) sum_{u >= t} (q_u dq_u - k_u dk_u) built from the oracle's own dq
    and dk (q enters as q e^{b_t}, k as k e^{-b_t}, b_t the cumulative log gate): the identity
    the GPU's stateless GLA backward evaluates."""
    B, N, H, d = 2, 23, 2, 5
    q, k, v = grid((B, N, H, d)), grid((B, N, H, d)), grid((B, N, H, d))
    a = grid((B, N, H, d), 0.3, 0.97)
    S0 = RNG.standard_normal((B, H, d, d))
    do = RNG.standard_normal((B, N, H, d))
    dq, dk, dv, da, dS0 = oracle.gla_bwd(q, k, v, a, do, scale=0.7, S0=S0)
    y = q.astype(np.float64) * dq - k.astype(np.float64) * dk
    suffix = np.flip(np.cumsum(np.flip(y, axis=1), axis=1), axis=1)
    np.testing.assert_allclose(suffix / a.astype(np.float64), da, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("form", ["gla", "delta", "gdn"])
def test_state_after_a_run_is_affine_in_the_entering_state(form):
    """S_end(S0) = T S0 + E with E = S_end(0) and T = S_end(I) for v = 0: the map the
    sequence-sharded forward folds across ranks (checked on random entering states)."""
    B, N, H, d = 1, 17, 2, 4
    q, k, v = grid((B, N, H, d)), grid((B, N, H, d)), grid((B, N, H, d))
    if form == "gla":
        a = grid((B, N, H, d), 0.5, 0.99)

        def run(vv, S):
            return oracle.gla(q, k, vv, a, S0=S)[1]
    else:
        k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
        a = grid((B, N, H), 0.5, 0.99)
        be = grid((B, N, H), 0.1, 0.9)

        def run(vv, S):
            return oracle.delta(q, k, vv, a, be, S0=S, erase_decayed=form == "gdn")[1]
    E = run(v, np.zeros((B, H, d, d)))
    T = run(np.zeros_like(v), np.broadcast_to(np.eye(d), (B, H, d, d)).copy())
    for _ in range(3):
        S0 = RNG.standard_normal((B, H, d, d))
        np.testing.assert_allclose(run(v, S0), T @ S0 + E, rtol=1e-10, atol=1e-12)
