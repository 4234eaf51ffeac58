"""The sequence-sharded hybrid forward's host logic on CPU ranks over gloo (world sizes 2 and 3):
frame runs, the K/V halo all-gather (including a halo that spans two predecessor ranks) and the
GLA / delta state prefix, with the per-rank compute done by the fp64 oracle. Every rank's rows
must equal the oracle's forward over the whole sequence."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from hybrid_linear_temporal_kta_b200 import seqshard  # noqa: E402


def test_frame_split_and_halo_plan():
    for F in (1, 5, 7, 21, 64):
        for R in range(1, 9):
            split = seqshard.frame_split(F, R)
            assert sum(c for _, c in split) == F
            assert all(split[i][0] + split[i][1] == split[i + 1][0] for i in range(R - 1))
            for halo in (0, 1, 4, 9):
                for r in range(R):
                    plan = seqshard.halo_plan(r, split, halo)
                    assert len(plan) == min(halo, split[r][0])
                    # the planned frames are exactly the global frames just before this run
                    glob = []
                    for j, f in plan:
                        first_j, cnt_j = split[j]
                        have = min(halo, cnt_j)
                        glob.append(first_j + cnt_j - have + (f - (halo - have)))
                    assert glob == list(range(split[r][0] - len(plan), split[r][0]))


def test_halo_sends_match_receives():
    """Every frame a rank receives is sent by exactly that source, with the same offset and
    count, so the point-to-point exchange is matched on both sides."""
    for F in (1, 5, 7, 21, 64):
        for R in range(1, 9):
            split = seqshard.frame_split(F, R)
            for halo in (0, 1, 4, 9):
                sends = {(r, dst, f0, n) for r in range(R)
                         for dst, f0, n in seqshard.halo_sends(r, split, halo)}
                recvs = {(src, r, f0, n) for r in range(R)
                         for src, f0, n in seqshard.halo_recvs(r, split, halo)}
                assert sends == recvs
                for r in range(R):
                    got = sum(n for _, _, n in seqshard.halo_recvs(r, split, halo))
                    assert got == min(halo, split[r][0])


class OracleOps:
    """CPU stand-in for the kernels: the fp64 oracle (test infrastructure)."""

    def __init__(self):
        import oracle
        self.o = oracle

    def lin_state(self, c, q, k, v, alpha, beta, S0):
        hs = slice(c.n_swa + c.n_dswa, c.H)
        S0n = None if S0 is None else S0.double().numpy()
        if c.gla_delta:
            _, S = self.o.delta(q[:, :, hs], k[:, :, hs], v[:, :, hs], alpha, beta,
                                scale=c.scale_gla, S0=S0n, erase_decayed=c.gla_delta == 2)
        else:
            _, S = self.o.gla(q[:, :, hs], k[:, :, hs], v[:, :, hs], alpha, scale=c.scale_gla,
                              S0=S0n)
        return torch.from_numpy(np.ascontiguousarray(S))

    def lin_transition(self, c, q, k, v, alpha, beta):
        """The run's transition: the end state from the identity with v = 0."""
        eye = torch.eye(c.d, dtype=torch.float64).expand(1, c.n_gla, c.d, c.d)
        return self.lin_state(c, q, k, torch.zeros_like(v), alpha, beta, eye)

    def state_affine(self, A, X, E):
        return torch.from_numpy(A.double().numpy() @ X.double().numpy() + E.double().numpy())

    def hybrid_window(self, c, f0, q, k_ext, v_ext, alpha, beta, S0):
        P, H, d = c.P, c.H, c.d
        n = q.shape[1]
        q_ext = torch.cat([torch.zeros((1, f0 * P, H, d), dtype=q.dtype), q], 1)
        rows = np.arange(f0 * P, f0 * P + n)
        out = np.zeros((1, n, H, d))
        sc = c.scale_softmax if c.scale_softmax is not None else d ** -0.5
        if c.n_swa:
            h = (0, c.n_swa)
            o = self.o.swa(q_ext, k_ext, v_ext, P, c.W_swa, sc, heads=h, rows=rows)
            out[:, :, :c.n_swa] = o[:, rows, :c.n_swa]
        if c.n_dswa:
            h = (c.n_swa, c.n_swa + c.n_dswa)
            o = self.o.dswa(q_ext, k_ext, v_ext, P, c.W_dswa, c.dil, sc, heads=h, rows=rows)
            out[:, :, h[0]:h[1]] = o[:, rows, h[0]:h[1]]
        if c.n_gla:
            hs = slice(c.n_swa + c.n_dswa, H)
            kl, vl = k_ext[:, f0 * P:, hs], v_ext[:, f0 * P:, hs]
            S0n = None if S0 is None else S0.double().numpy()
            if c.gla_delta:
                o, _ = self.o.delta(q[:, :, hs], kl, vl, alpha, beta, scale=c.scale_gla, S0=S0n,
                                    erase_decayed=c.gla_delta == 2)
            else:
                o, _ = self.o.gla(q[:, :, hs], kl, vl, alpha, scale=c.scale_gla, S0=S0n)
            out[:, :, hs] = o
        return torch.from_numpy(out)


def _inputs(c, seed):
    rng = np.random.default_rng(seed)
    N = c.F * c.P
    q, k, v = (torch.from_numpy(rng.standard_normal((1, N, c.H, c.d)).astype(np.float32))
               for _ in range(3))
    if c.gla_delta:
        k[:, :, c.n_swa + c.n_dswa:] /= k[:, :, c.n_swa + c.n_dswa:].norm(dim=-1, keepdim=True)
        a = torch.from_numpy(rng.uniform(0.7, 0.99, (1, N, c.n_gla)).astype(np.float32))
        b = torch.from_numpy(rng.uniform(0.1, 0.9, (1, N, c.n_gla)).astype(np.float32))
    else:
        a = torch.from_numpy(rng.uniform(0.6, 0.99, (1, N, c.n_gla, c.d)).astype(np.float32))
        b = None
    S0 = torch.from_numpy(rng.standard_normal((1, c.n_gla, c.d, c.d)) * 0.3)
    return q, k, v, a, b, S0


def _full_reference(c, q, k, v, a, b, S0):
    """The oracle over the whole sequence, GLA heads from S0."""
    import oracle
    sc = c.d ** -0.5
    o = np.zeros((1, c.F * c.P, c.H, c.d))
    oracle.swa(q, k, v, c.P, c.W_swa, sc, heads=(0, c.n_swa), out=o)
    oracle.dswa(q, k, v, c.P, c.W_dswa, c.dil, sc, heads=(c.n_swa, c.n_swa + c.n_dswa), out=o)
    hg = (c.n_swa + c.n_dswa, c.H)
    if c.gla_delta:
        oracle.delta(q, k, v, a, b, c.scale_gla, S0=S0.numpy(), heads=hg, out=o,
                     erase_decayed=c.gla_delta == 2)
    else:
        oracle.gla(q, k, v, a, c.scale_gla, S0=S0.numpy(), heads=hg, out=o)
    return o


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, cfg_kw, qout):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        c = seqshard.ShardCfg(**cfg_kw)
        q, k, v, a, b, S0 = _inputs(c, 123)
        first, count = seqshard.frame_split(c.F, world)[rank]
        rs = slice(first * c.P, (first + count) * c.P)
        loc = lambda t: None if t is None else t[:, rs].contiguous()  # noqa: E731
        o = seqshard.sharded_hybrid_fwd(c, loc(q), loc(k), loc(v), loc(a), loc(b),
                                        ops=OracleOps(), S0=S0)
        qout.put((rank, first, o.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,gla_delta", [(2, 0), (3, 0), (3, 1), (2, 2), (4, 0)])
def test_sharded_forward_equals_whole_sequence(world, gla_delta):
    cfg_kw = dict(F=7, P=6, d=8, n_swa=1, n_dswa=1, n_gla=1, W_swa=2, W_dswa=3, dil=2,
                  gla_delta=gla_delta, chunk=16)
    c = seqshard.ShardCfg(**cfg_kw)
    assert c.halo == 4
    port = _free_port()
    ctx = mp.get_context("spawn")
    qout = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cfg_kw, qout)) for r in range(world)]
    for p in procs:
        p.start()
    res = [qout.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v, a, b, S0 = _inputs(c, 123)
    ref = _full_reference(c, q, k, v, a, b, S0)
    for rank, first, o in res:
        r0 = first * c.P
        exp = ref[:, r0:r0 + o.shape[1]]
        err = np.abs(o - exp).max() / np.abs(exp).max()
        assert err < 1e-10, f"rank {rank}: max relative error {err:.2e}"


@pytest.mark.parametrize("R,gla_delta", [(1, 0), (4, 0), (5, 1), (7, 2)])
def test_emulated_ranks_equal_whole_sequence(R, gla_delta):
    c = seqshard.ShardCfg(F=7, P=6, d=8, n_swa=1, n_dswa=1, n_gla=1, W_swa=2, W_dswa=3, dil=2,
                          gla_delta=gla_delta, chunk=16)
    q, k, v, a, b, S0 = _inputs(c, 321)
    o = seqshard.emulate_ranks(c, R, q, k, v, a, b, ops=OracleOps(), S0=S0).numpy()
    ref = _full_reference(c, q, k, v, a, b, S0)
    assert np.abs(o - ref).max() / np.abs(ref).max() < 1e-10
