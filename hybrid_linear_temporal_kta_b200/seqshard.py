"""Sequence-sharded hybrid forward: one long sequence split into runs of frames across ranks.

Each rank holds a contiguous run of frames (q, k, v and gates of those frames) and computes
their outputs. Two things cross rank boundaries:
- the softmax heads' K/V halo: the windows of a rank's first frames reach back
  max(W_swa - 1, (W_dswa - 1) * dil) frames (paper-read, section 2, second pillar, SWA and DSWA
  paragraphs). Each rank sends point to point exactly the frames each successor needs (a rank
  holding fewer frames than the halo passes on what it has, and the successor takes the rest
  from earlier ranks);
- the GLA / delta-rule state at the rank's first token. The state after a run is an affine map
  of the state entering it, S_end = T S_start + E (GLA paragraph: the update is linear in S).
  Every rank computes its run's E (the end state from zero) and T (its transition: for the
  vector-gated GLA the diagonal of gate products over the run, for the delta rule the end state
  from the identity with v = 0), the pairs are all-gathered, and each rank folds its
  predecessors' maps into its entering state.
The rank then runs the hybrid layer on its frames with the halo in front of its K/V and the
entering state (kta_hybrid_fwd_window).

The compute steps go through an `ops` object, so that the same orchestration runs on the GPU
(KtaOps: the library's kernels, NCCL) and, in tests, on CPU ranks over gloo with a CPU stand-in.
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist


def frame_split(F: int, R: int) -> list[tuple[int, int]]:
    """Contiguous, balanced runs of frames: rank r holds frames [first_r, first_r + count_r)."""
    return [(r * F // R, (r + 1) * F // R - r * F // R) for r in range(R)]


def halo_frames(n_swa: int, n_dswa: int, W_swa: int, W_dswa: int, dil: int) -> int:
    """Frames before a query frame that its softmax windows can reach."""
    return max((W_swa - 1) if n_swa else 0, (W_dswa - 1) * dil if n_dswa else 0)


def halo_plan(r: int, split: list[tuple[int, int]], halo: int) -> list[tuple[int, int]]:
    """Which frames rank r receives, oldest first, as (source rank, frame offset within that
    rank's halo block); each rank's block holds its last min(halo, count) frames at the END of a
    block of `halo` frames. Rank r needs min(halo, first_r) frames."""
    need = min(halo, split[r][0])
    out = []
    j = r - 1
    while need > 0 and j >= 0:
        have = min(halo, split[j][1])
        take = min(need, have)
        out = [(j, halo - take + i) for i in range(take)] + out
        need -= take
        j -= 1
    return out


@dataclasses.dataclass
class ShardCfg:
    F: int            # frames of the whole sequence
    P: int
    d: int
    n_swa: int
    n_dswa: int
    n_gla: int
    W_swa: int
    W_dswa: int
    dil: int
    gla_delta: int = 0
    chunk: int = 64
    scale_softmax: float | None = None
    scale_gla: float = 1.0

    @property
    def H(self) -> int:
        return self.n_swa + self.n_dswa + self.n_gla

    @property
    def halo(self) -> int:
        return halo_frames(self.n_swa, self.n_dswa, self.W_swa, self.W_dswa, self.dil)


def halo_sends(r: int, split: list[tuple[int, int]], halo: int) -> list[tuple[int, int, int]]:
    """What rank r sends: (destination rank, first frame offset, frame count) within r's halo
    block, the frames of r that each later rank's halo_plan takes from r."""
    out = []
    for r2 in range(r + 1, len(split)):
        fs = [f for j, f in halo_plan(r2, split, halo) if j == r]
        if fs:
            out.append((r2, fs[0], len(fs)))
    return out


def halo_recvs(r: int, split: list[tuple[int, int]], halo: int) -> list[tuple[int, int, int]]:
    """What rank r receives: (source rank, first frame offset in the source's halo block, frame
    count), oldest source first."""
    out: list[tuple[int, int, int]] = []
    for j, f in halo_plan(r, split, halo):
        if out and out[-1][0] == j:
            out[-1] = (j, out[-1][1], out[-1][2] + 1)
        else:
            out.append((j, f, 1))
    return out


def _exchange_halo(c: "ShardCfg", r: int, R: int, blk: torch.Tensor, group) -> dict:
    """Point-to-point halo exchange: {source rank: (first frame offset, [2, n*P, ns, d] K/V)}."""
    split = frame_split(c.F, R)
    P = c.P
    ops, got = [], {}
    for dst, f0, n in halo_sends(r, split, c.halo):
        ops.append(dist.P2POp(dist.isend, blk[:, f0 * P:(f0 + n) * P].contiguous(),
                              dist.get_global_rank(group, dst) if group is not None else dst,
                              group))
    for src, f0, n in halo_recvs(r, split, c.halo):
        buf = torch.empty((2, n * P) + tuple(blk.shape[2:]), dtype=blk.dtype, device=blk.device)
        got[src] = (f0, buf)
        ops.append(dist.P2POp(dist.irecv, buf,
                              dist.get_global_rank(group, src) if group is not None else src,
                              group))
    if ops:
        for w in dist.batch_isend_irecv(ops):
            w.wait()
    return got


def _all_gather(t: torch.Tensor, group) -> list[torch.Tensor]:
    R = dist.get_world_size(group)
    bufs = [torch.empty_like(t) for _ in range(R)]
    dist.all_gather(bufs, t.contiguous(), group=group)
    return bufs


def local_contribution(c: ShardCfg, r: int, R: int, q, k, v, alpha=None, beta=None, *, ops):
    """What rank r sends to the others: its halo block (the softmax heads' K and V of its last
    min(halo, count) frames, at the end of a block of `halo` frames) and, with GLA heads and
    R > 1, its run's state map (E: end state from zero; T: its transition, ops.lin_transition)."""
    first, count = frame_split(c.F, R)[r]
    P, d = c.P, c.d
    ns = c.n_swa + c.n_dswa
    if q.shape[1] != count * P:
        raise ValueError(f"rank {r} holds {count} frames of {P} tokens, got {q.shape[1]} rows")
    blk = None
    if ns and c.halo:
        halo = c.halo
        blk = torch.zeros((2, halo * P, ns, d), dtype=k.dtype, device=k.device)
        have = min(halo, count)
        if have:
            blk[0, (halo - have) * P:] = k[0, (count - have) * P:, :ns]
            blk[1, (halo - have) * P:] = v[0, (count - have) * P:, :ns]
    E = T = None
    if c.n_gla and R > 1:
        E = ops.lin_state(c, q, k, v, alpha, beta, None)
        T = ops.lin_transition(c, q, k, v, alpha, beta)
    return blk, E, T


def finish(c: ShardCfg, r: int, R: int, q, k, v, alpha, beta, halo_in, Es, Ts, *, ops, S0=None):
    """Rank r's outputs from what it received: the halo in front of its K/V (halo_in: {source
    rank: (first frame offset within the source's halo block, its K/V [2, n*P, ns, d])}), the
    entering GLA state folded from its predecessors' maps, then the windowed hybrid layer."""
    split = frame_split(c.F, R)
    first, count = split[r]
    P, d, H = c.P, c.d, c.H
    ns = c.n_swa + c.n_dswa
    plan = halo_plan(r, split, c.halo) if (ns and c.halo) else []
    hk = len(plan)
    k_ext, v_ext = k, v
    if hk:
        k_ext = torch.zeros((1, (hk + count) * P, H, d), dtype=k.dtype, device=k.device)
        v_ext = torch.zeros_like(k_ext)
        for i, (j, f) in enumerate(plan):
            f0, blk = halo_in[j]
            k_ext[0, i * P:(i + 1) * P, :ns] = blk[0, (f - f0) * P:(f - f0 + 1) * P]
            v_ext[0, i * P:(i + 1) * P, :ns] = blk[1, (f - f0) * P:(f - f0 + 1) * P]
        k_ext[0, hk * P:] = k[0]
        v_ext[0, hk * P:] = v[0]
    S_in = S0
    if c.n_gla and R > 1 and r > 0:
        S = S0 if S0 is not None else torch.zeros((1, c.n_gla, d, d), dtype=torch.float32,
                                                  device=q.device)
        for j in range(r):
            S = ops.state_affine(Ts[j], S, Es[j])
        S_in = S
    return ops.hybrid_window(c, hk, q, k_ext, v_ext, alpha, beta, S_in)


def sharded_hybrid_fwd(c: ShardCfg, q, k, v, alpha=None, beta=None, *, ops, group=None, S0=None):
    """This rank's outputs [1, count*P, H, d] for its frames, one rank per process of `group`.
    q, k, v: [1, count*P, H, d]; alpha / beta: this rank's gates (vector GLA
    [1, count*P, n_gla, d], delta [1, count*P, n_gla]); S0: the sequence's initial GLA state
    [1, n_gla, d, d] (None = zero). Every rank calls this with the same ShardCfg; ranks take
    frames by frame_split(F, world size). The exchange is point-to-point sends of halo frames to
    the ranks that need them and two all-gathers of the (small) state maps."""
    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    blk, E, T = local_contribution(c, r, R, q, k, v, alpha, beta, ops=ops)
    halo_in = _exchange_halo(c, r, R, blk, group) if blk is not None else {}
    Es = _all_gather(E, group) if E is not None else None
    Ts = _all_gather(T, group) if T is not None else None
    return finish(c, r, R, q, k, v, alpha, beta, halo_in, Es, Ts, ops=ops, S0=S0)


def emulate_ranks(c: ShardCfg, R: int, q, k, v, alpha=None, beta=None, *, ops, S0=None):
    """The R ranks' computation in one process (each rank's steps run one after another, with
    the exchange done by collecting the contributions): the whole sequence's outputs."""
    split = frame_split(c.F, R)
    P = c.P
    sl = [slice(f * P, (f + n) * P) for f, n in split]
    loc = [tuple(None if t is None else t[:, s_].contiguous() for t in (q, k, v, alpha, beta))
           for s_ in sl]
    contrib = [local_contribution(c, r, R, *loc[r], ops=ops) for r in range(R)]
    Es = [x[1] for x in contrib]
    Ts = [x[2] for x in contrib]
    outs = []
    for r in range(R):
        halo_in = {}
        if contrib[r][0] is not None:
            for src, f0, n in halo_recvs(r, split, c.halo):
                halo_in[src] = (f0, contrib[src][0][:, f0 * P:(f0 + n) * P])
        outs.append(finish(c, r, R, *loc[r], halo_in, Es, Ts, ops=ops, S0=S0))
    return torch.cat(outs, 1)


class KtaOps:
    """The library's kernels (one GPU per rank)."""

    def __init__(self):
        from . import kta
        self.kta = kta

    def _cfg(self, c: ShardCfg, F: int, dtype):
        return self.kta.hybrid_cfg(B=1, F=F, P=c.P, d=c.d, dtype=dtype, n_swa=c.n_swa,
                                   n_dswa=c.n_dswa,
                                   n_gla=c.n_gla, W_swa=c.W_swa, W_dswa=c.W_dswa, dil=c.dil,
                                   chunk=c.chunk, gla_delta=c.gla_delta,
                                   scale_softmax=c.scale_softmax, scale_gla=c.scale_gla)

    def lin_state(self, c: ShardCfg, q, k, v, alpha, beta, S0):
        heads = (c.n_swa + c.n_dswa, c.H)
        if not c.gla_delta and q.dtype == torch.bfloat16:
            # the end state alone: state pass and segment fold, no output pass
            return self.kta.gla_chunk_state(k, v, alpha, chunk=c.chunk, S0=S0, heads=heads)
        scratch = torch.empty_like(q)
        if c.gla_delta:
            _, S = self.kta.gla_delta_fwd(q, k, v, alpha, beta, chunk=c.chunk, scale=c.scale_gla,
                                          S0=S0, return_state=True, heads=heads, out=scratch,
                                          erase_decayed=c.gla_delta == 2)
        else:
            _, S = self.kta.gla_chunk_fwd(q, k, v, alpha, chunk=c.chunk, scale=c.scale_gla, S0=S0,
                                          return_state=True, heads=heads, out=scratch)
        return S

    def lin_transition(self, c: ShardCfg, q, k, v, alpha, beta):
        """T of the run: the diagonal of gate products for vector GLA (one pass over the gates);
        for the delta rule, whose transition is dense, the end state from the identity with
        v = 0."""
        if not c.gla_delta:
            return self.kta.gla_transition(alpha)
        d = c.d
        eye = torch.eye(d, dtype=torch.float32, device=q.device).expand(1, c.n_gla, d, d)
        return self.lin_state(c, q, k, torch.zeros_like(v), alpha, beta, eye.contiguous())

    def state_affine(self, A, X, E):
        return self.kta.state_affine(A, X, E)

    def hybrid_window(self, c: ShardCfg, f0: int, q, k_ext, v_ext, alpha, beta, S0):
        F_ext = k_ext.shape[1] // c.P
        return self.kta.hybrid_fwd_window(self._cfg(c, F_ext, q.dtype), f0, q, k_ext, v_ext, alpha,
                                          beta, S0=S0)
