#!/usr/bin/env python
"""Throughput benchmark of the hybrid temporal attention forward on B200.

Workload (one step = one hybrid layer forward over one batch): B = 1 sequence of F = 21 latent
frames x P = 1560 tokens (32,760 tokens), 24 heads of d = 128 (8 SWA with W = 3, 8 DSWA with
W = 4 and dil = 3, 8 GLA with 64-token chunks), bf16, inputs N(0,1) and alpha = sigmoid(N(3,1)),
synthetic and seeded. Metric: tokens per second (positions through all 24 heads), whole job.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kta|reference]
For N > 1 launch one process per GPU with torch.distributed.run; every rank runs its own
sequences (no collective on the data path: weak scaling) and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "hybrid temporal attn fwd tokens/s (bf16, 1xB200); % of HBM/tensor roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("kta", "reference"), default="kta")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle timing leg (faster profiling runs)")
    ap.add_argument("--frames", type=int, default=None,
                    help="profiling only: override the hybrid workload's frame count (the "
                         "headline line is the default, 21 frames)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="profiling only: override the delta workload's tokens per sequence")
    ap.add_argument("--workload", choices=("hybrid", "delta", "stream", "sweep", "backward",
                                           "layer", "seqshard", "backward_bf16"),
                    default="hybrid",
                    help="hybrid: the 21-frame hybrid layer (the headline line); delta: gated "
                         "delta rule, 2 x 65,536 tokens x 16 heads; stream: 240-frame rollout one "
                         "frame per call; sweep: hybrid layer vs full frame-causal attention for "
                         "F = 8..256 frames of 1,024 tokens (one line per F); backward: the "
                         "hybrid layer's reverse mode in fp32; layer: input projections + hybrid "
                         "operator + output projection; seqshard: the hybrid layer split by frames "
                         "over 4 ranks, emulated one after another on one GPU; backward_bf16: the "
                         "hybrid layer's reverse mode with the softmax heads on tensor cores")
    return ap.parse_args()


# --------------------------------------------------------------------------- workload algebra


def visible_pairs(w) -> int:
    """(query, key) pairs the softmax heads attend to: P^2 per visible (query frame, key frame)."""
    swa = sum(min(f + 1, w.W_swa) for f in range(w.F))
    dswa = sum(min(w.W_dswa, f // w.dil + 1) for f in range(w.F))
    return w.B * w.P * w.P * (w.n_swa * swa + w.n_dswa * dswa)


def softmax_flops(w) -> float:
    """Algorithmic FLOPs of the softmax branches: 2d for q.k and 2d for p*v per visible pair."""
    return 4.0 * w.d * visible_pairs(w)


def gla_bytes(w) -> float:
    """Algorithmic HBM bytes of the vector-GLA heads: q, k, v, o bf16 + alpha fp32 per token-head."""
    return 12.0 * w.d * w.B * w.N * w.n_gla


def delta_bytes(w) -> float:
    """Algorithmic HBM bytes of the delta-rule heads: q, k, v, o bf16 + alpha, beta fp32."""
    return (8.0 * w.d + 8.0) * w.B * w.N * w.n_gla


def delta_flops(w) -> float:
    """MMA FLOPs of the chunked delta rule: 10 C d + 6 d^2 per token-head."""
    return (10.0 * w.chunk * w.d + 6.0 * w.d * w.d) * w.B * w.N * w.n_gla


def softmax_bwd_flops(w) -> dict:
    """Algorithmic FLOPs of the softmax branches' reverse mode, 2d per product per visible pair:
    the dq kernel forms S, dP and dQ (6d), the key-major kernel S, dP, dV and dK (8d)."""
    n = visible_pairs(w)
    return {"softmax_bwd_q_f32": 6.0 * w.d * n, "softmax_bwd_kv_f32": 8.0 * w.d * n}


def layer_proj_flops(w) -> float:
    """Projection FLOPs of one layer step with model width C = H d: the stacked q/k/v/alpha
    product (3 H d + n_gla d outputs) and the output projection (C outputs), 2 per MAC."""
    C = w.H * w.d
    return 2.0 * w.B * w.N * C * (3 * w.H * w.d + w.n_gla * w.d) + 2.0 * w.B * w.N * C * C


def fp32_alu_tflops(sm_mhz: float) -> float:
    """fp32 FMA peak: 148 SMs x 128 lanes x 2 FLOP per clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def full_causal_flops(w) -> float:
    """Frame-causal attention over every earlier frame on all heads: 4 d per visible pair."""
    return 4.0 * w.d * w.B * w.P * w.P * w.F * (w.F + 1) // 2 * w.H


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


KERNEL_SOURCES = {
    "win_attn_tc": ("win_attn_tc.cuh", "kta_ptx.cuh"),
    "gla_tc_state": ("gla_tc.cuh", "mma_sync.cuh", "kta_ptx.cuh"),
    "gla_tc_out": ("gla_tc.cuh", "mma_sync.cuh", "kta_ptx.cuh"),
    "delta_prep": ("delta_chunk.cuh", "mma_sync.cuh"),
    "delta_scan": ("delta_chunk.cuh", "mma_sync.cuh", "kta_ptx.cuh"),
}


def kernel_source_hash(kernel: str) -> str:
    """Hash of the source files a kernel is built from (its ncu counters go stale when it moves)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hybrid_linear_temporal_kta_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it was taken on the
    current kernel sources and for this workload (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    if e.get("config_workload") != workload:
        return None
    return e.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.dev = device_id
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        loaded = [x for x in sm if x > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------------------- distributed


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(val: float, ws: int, device) -> float:
    """Max of a per-rank scalar over all ranks (the job's time is its slowest rank's)."""
    if ws == 1:
        return val
    import torch
    import torch.distributed as dist
    t = torch.tensor([val], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(ws: int, tokens_per_rank_step: int, steps: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank processes its own sequences (weak scaling)."""
    return ws * tokens_per_rank_step * steps / (ms_max / 1e3)


def rank_seed_base(base: int, rank: int) -> int:
    """Each rank draws its own sequences."""
    return base + 100 * rank


def hybrid_config(w, ws: int) -> dict:
    """The workload description both arms print (same keys, so their lines compare)."""
    h2d = w.B * w.N * w.H * w.d * 2 * 3 + w.B * w.N * w.n_gla * w.d * 4
    return {"workload": w.name, "B": w.B, "F": w.F, "P": w.P, "N": w.N, "H": w.H, "d": w.d,
            "heads": f"{w.n_swa} SWA W={w.W_swa} | {w.n_dswa} DSWA W={w.W_dswa} dil={w.dil} | "
                     f"{w.n_gla} GLA chunk={w.chunk}",
            "parallelism": f"dp{ws} (independent sequences per GPU, no collective)",
            "l2": f"inputs {h2d / 1e6:.0f} MB per step"
                  f"{' > 126 MB L2; no flush' if h2d > 126e6 else ' (fits L2)'}"}


# --------------------------------------------------------------------------- CPU oracle timing


def oracle_sample(w, x, target_s: float = 20.0):
    """Time the fp64 CPU oracle on a bounded sample of the workload: M query rows (seeded) of the
    16 softmax heads plus the first M tokens of the 8 GLA heads. Returns tokens/s and details."""
    import numpy as np

    import oracle

    oracle.set_threads(0)
    q = x["q"].float().numpy()
    k = x["k"].float().numpy()
    v = x["v"].float().numpy()
    a = x["alpha"].numpy()
    rng = np.random.default_rng(17)
    hs, hd = (0, w.n_swa), (w.n_swa, w.n_swa + w.n_dswa)
    hg = (w.n_swa + w.n_dswa, w.H)

    out = np.full(q.shape, np.nan)  # written only at the sampled rows; allocated once

    def run(M):
        rows = np.sort(rng.choice(w.N, size=M, replace=False))
        t0 = time.perf_counter()
        oracle.swa(q, k, v, w.P, w.W_swa, w.scale_softmax, heads=hs, rows=rows, out=out)
        oracle.dswa(q, k, v, w.P, w.W_dswa, w.dil, w.scale_softmax, heads=hd, rows=rows, out=out)
        oracle.gla(q[:, :M], k[:, :M], v[:, :M], a[:, :M], heads=hg)
        return time.perf_counter() - t0

    M = 256
    t = run(M)
    M = int(min(w.N, max(64, M * target_s / max(t, 1e-3))))
    t = run(M)
    return {"value": M * w.B / t, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
            "sample_s": t, "sample_tokens": M * w.B,
            "sample": f"{M} seeded query rows of the 16 softmax heads + the first {M} tokens of the "
                      f"8 GLA heads (fp64 CPU oracle), {t:.1f} s"}


# --------------------------------------------------------------------------- arms


def run_reference(args):
    """Reference arm: the fp64 CPU oracle on the host cores. Each step is one bounded sample of
    the workload (seeded query rows of the softmax heads plus leading tokens of the GLA heads),
    sized so that warm-up and timed steps together take about two minutes; ms_per_step is the
    measured wall time of a sample, and the time the oracle would need for the whole layer is
    reported separately as an extrapolation."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    from hybrid_linear_temporal_kta_b200 import synth

    w = synth.HYBRID_BF16
    x = synth.make_inputs(w)
    per_step = min(5.0, max(0.5, 120.0 / max(args.steps + args.warmup, 1)))
    for _ in range(args.warmup):
        oracle_sample(w, x, target_s=min(per_step, 1.0))
    vals = [oracle_sample(w, x, target_s=per_step) for _ in range(args.steps)]
    v = statistics.median(r["value"] for r in vals)
    ms = statistics.median(r["sample_s"] for r in vals) * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "ms_per_step_kind": "measured wall time of one bounded oracle sample per step",
            "full_layer_ms_extrapolated": w.B * w.N / v * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": hybrid_config(w, ws),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": vals[-1]["cores"],
                             "kind": "oracle", "sample": vals[-1]["sample"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_kta(args):
    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    if args.gpus != ws and ws > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {ws}", file=sys.stderr)
    torch.cuda.set_device(local)
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    from hybrid_linear_temporal_kta_b200 import kta, synth

    w = synth.HYBRID_BF16 if args.frames is None else synth.HYBRID_BF16.replace(
        name=f"hybrid_bf16_F{args.frames}_P1560", F=args.frames)
    x = synth.make_inputs(w, seed_base=rank_seed_base(w.seed_base, rank))
    cfg = kta.cfg_from_workload(w)
    host = {n: x[n].pin_memory() for n in ("q", "k", "v", "alpha")}
    devx = {n: host[n].cuda() for n in host}
    o = torch.empty_like(devx["q"])
    o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    stream = torch.cuda.current_stream()

    def step():
        kta.hybrid_fwd(cfg, devx["q"], devx["k"], devx["v"], devx["alpha"], out=o)

    def barrier():
        if ws > 1:
            dist.barrier()

    def max_over_ranks(val: float) -> float:
        return reduce_max(val, ws, torch.device("cuda", local))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    kta.device_status()

    # ---- device-resident timed region: exactly K steps
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    uuid = str(getattr(props, "uuid", "") or "")
    clocks = ClockSampler(("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else
                          (uuid or str(torch.cuda.current_device())))
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    kta.device_status()
    ms = max_over_ranks(e0.elapsed_time(e1))
    value = whole_job_rate(ws, w.B * w.N, args.steps, ms)

    # ---- the same steps with per-kernel tracing (device time of every launch, on its stream)
    with kta.trace() as tr:
        for _ in range(args.steps):
            step()
    torch.cuda.synchronize()
    kern = tr.kernels

    # ---- the GLA heads alone (same call the hybrid makes on its side stream), so that their
    # kernel times are not stretched by waiting for SMs held by the softmax kernel
    hg = (w.n_swa + w.n_dswa, w.H)
    for _ in range(2):
        kta.gla_chunk_fwd(devx["q"], devx["k"], devx["v"], devx["alpha"], chunk=w.chunk,
                          heads=hg, out=o)
    torch.cuda.synchronize()
    with kta.trace() as trg:
        for _ in range(args.steps):
            kta.gla_chunk_fwd(devx["q"], devx["k"], devx["v"], devx["alpha"], chunk=w.chunk,
                              heads=hg, out=o)
    torch.cuda.synchronize()
    kern_gla = trg.kernels

    # ---- end to end through the public call with host buffers: every step copies its inputs
    # from pinned host memory (H2D), runs the forward and copies the output back (D2H). Two
    # device buffer sets and three streams let step s+1's upload and step s-1's download overlap
    # step s's forward; the timed region runs from the first upload to the last download.
    h2d = sum(host[n].numel() * host[n].element_size() for n in host)
    d2h = o.numel() * o.element_size()
    dev2 = [devx, {n: torch.empty_like(devx[n]) for n in devx}]
    out2 = [o, torch.empty_like(o)]
    ohost2 = [o_host, torch.empty(o.shape, dtype=o.dtype, pin_memory=True)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event(), torch.cuda.Event()]
    ev_done = [torch.cuda.Event(), torch.cuda.Event()]
    ev_out = [torch.cuda.Event(), torch.cuda.Event()]

    def e2e_run(nsteps):
        for i in range(nsteps):
            bsel = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[bsel])  # the forward of step i-2 has read these inputs
                for n in host:
                    dev2[bsel][n].copy_(host[n], non_blocking=True)
                ev_in[bsel].record(s_in)
            stream.wait_event(ev_in[bsel])
            if i >= 2:
                stream.wait_event(ev_out[bsel])  # step i-2's output has been copied out
            kta.hybrid_fwd(cfg, dev2[bsel]["q"], dev2[bsel]["k"], dev2[bsel]["v"],
                           dev2[bsel]["alpha"], out=out2[bsel], stream=stream)
            ev_done[bsel].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[bsel])
                ohost2[bsel].copy_(out2[bsel], non_blocking=True)
                ev_out[bsel].record(s_out)

    e2e_run(3)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    e2e_run(args.steps)
    s_out.wait_event(ev_done[(args.steps - 1) & 1])
    t1.record(s_out)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = max_over_ranks(t0.elapsed_time(t1))
    kta.device_status()

    peaks, peaks_kind = load_peaks()
    sm = kern.get("win_attn_tc", {"launches": 0, "ms": float("nan")})
    t_launch = sm["ms"] / max(sm["launches"], 1) / 1e3
    flops = softmax_flops(w)
    achieved = flops / t_launch / 1e12
    peak = float(peaks["bf16_tflops"])
    traffic = recorded_traffic("win_attn_tc", w.name)
    # DRAM bytes of one GLA call (state pass + output pass) from the committed ncu summary
    gla_parts = [recorded_traffic(k, w.name) for k in ("gla_tc_state", "gla_tc_out")]
    gla_traffic = sum(gla_parts) if all(x is not None for x in gla_parts) else None
    t_gla = sum(v["ms"] for v in kern_gla.values()) / args.steps / 1e3
    launches = sum(v["launches"] for v in kern.values()) // args.steps * args.steps

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": hybrid_config(w, ws),
        "roofline": {"kernel": "win_attn_tc (SWA+DSWA heads, tcgen05)", "bound": "tensor",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"bf16_tflops burst ({peaks_kind})",
                     "algorithmic_flops_per_launch": flops,
                     "launch_ms": t_launch * 1e3},
        "kernels": {k: {"launches": v["launches"] // args.steps,
                        "ms_per_step": v["ms"] / args.steps} for k, v in kern.items()},
        "kernels_note": "in-step event spans; launches on the forked GLA stream include time spent "
                        "waiting for SMs held by the softmax kernel (see gla_roofline for the GLA "
                        "kernels timed alone)",
        "gla_roofline": {"kernels": {k: {"launches": v["launches"] // args.steps,
                                         "ms_per_call": v["ms"] / args.steps}
                                     for k, v in kern_gla.items()},
                         "timed": "the GLA heads alone, one call per step, nothing else running",
                         "ms_per_call": t_gla * 1e3,
                         "bound": "hbm", "achieved": gla_bytes(w) / t_gla / 1e9 if t_gla > 0 else None,
                         "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                         "frac": gla_bytes(w) / t_gla / 1e9 / float(peaks["hbm_gbs"]) if t_gla > 0 else None,
                         "algorithmic_bytes": gla_bytes(w), "traffic": gla_traffic},
        "e2e": {"value": whole_job_rate(ws, w.B * w.N, args.steps, ms_e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample(w, x)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- other workloads


def _device_ms(fn, steps: int, warmup: int) -> float:
    """Mean device milliseconds of fn() over `steps` calls after `warmup` calls (CUDA events on
    the current stream, synchronised on both sides)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def _traced(fn, steps: int) -> dict:
    import torch

    from hybrid_linear_temporal_kta_b200 import kta
    with kta.trace() as tr:
        for _ in range(steps):
            fn()
    torch.cuda.synchronize()
    return {k: {"launches": v["launches"] // steps, "ms_per_step": v["ms"] / steps}
            for k, v in tr.kernels.items()}


def run_other(args):
    """Timing of the workloads other than the headline hybrid layer (one GPU; one JSON line per
    workload, or per F for the sweep). Inputs are drawn on the device with the same recipe; the
    inputs of every workload are larger than the 126 MB L2, so no flush is needed."""
    import torch

    from hybrid_linear_temporal_kta_b200 import kta, synth

    torch.cuda.set_device(0)
    peaks, peaks_kind = load_peaks()
    hbm, tc = float(peaks["hbm_gbs"]), float(peaks["bf16_tflops"])
    lines = []
    if args.workload == "delta":
        w = synth.DELTA_BF16
        if args.tokens is not None:
            w = w.replace(name=f"gated_delta_bf16_B2_L{args.tokens}", F=1, P=args.tokens)
        x = synth.make_inputs_device(w, seed=w.seed_base)
        o = torch.empty_like(x["q"])

        def step():
            kta.gla_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], chunk=w.chunk,
                              out=o)
        ms = _device_ms(step, args.steps, args.warmup)
        kern = _traced(step, args.steps)
        t_star = max(delta_bytes(w) / (hbm * 1e9), delta_flops(w) / (tc * 1e12))
        lines.append({
            "workload": w.name, "metric": "gated delta rule fwd tokens/s", "unit": "tokens/s",
            "value": w.B * w.N / (ms / 1e3), "ms_per_step": ms, "steps": args.steps,
            "config": {"B": w.B, "N": w.N, "H": w.n_gla, "d": w.d, "chunk": w.chunk},
            "roofline": {"bound": "hbm", "algorithmic_bytes": delta_bytes(w),
                         "algorithmic_flops": delta_flops(w),
                         "achieved_gbs": delta_bytes(w) / (ms / 1e3) / 1e9, "peak_gbs": hbm,
                         "t_star_ms": t_star * 1e3, "frac": t_star / (ms / 1e3),
                         "peak_source": peaks_kind},
            "kernels": kern})
    elif args.workload == "stream":
        w = synth.STREAM_BF16
        x = synth.make_inputs_device(w, seed=w.seed_base)
        cfg = kta.cfg_from_workload(w)
        st = kta.Stream(cfg)
        o = torch.empty_like(x["q"])
        P = w.P
        frames = [tuple(x[n][:, f * P:(f + 1) * P] for n in ("q", "k", "v", "alpha")) +
                  (o[:, f * P:(f + 1) * P],) for f in range(w.F)]

        def rollout():
            st.reset()
            for q, k, v, a, of in frames:
                st.step(q, k, v, a, out=of)
        ms = _device_ms(rollout, args.steps, args.warmup)
        kern = _traced(rollout, args.steps)
        # the same rollout captured once as a CUDA graph (240 steps' launches replayed together)
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            rollout()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph):
            rollout()
        ms_graph = _device_ms(graph.replay, args.steps, args.warmup)
        del graph
        flops = softmax_flops(w)
        t_star = max(flops / (tc * 1e12), (8.0 * w.d * w.B * w.N * (w.n_swa + w.n_dswa) +
                                          gla_bytes(w)) / (hbm * 1e9))
        lines.append({
            "workload": w.name, "metric": "streaming rollout tokens/s (one frame per call)",
            "unit": "tokens/s", "value": w.B * w.N / (ms / 1e3), "ms_per_rollout": ms,
            "us_per_frame": ms * 1e3 / w.F, "steps": args.steps,
            "graph": {"value": w.B * w.N / (ms_graph / 1e3), "ms_per_rollout": ms_graph,
                      "us_per_frame": ms_graph * 1e3 / w.F,
                      "note": "the rollout captured once with torch.cuda.graph and replayed"},
            "config": {"B": w.B, "F": w.F, "P": w.P, "H": w.H, "d": w.d,
                       "state_bytes": st.state_bytes},
            "roofline": {"bound": "tensor", "t_star_ms": t_star * 1e3, "frac": t_star / (ms / 1e3),
                         "peak_source": peaks_kind},
            "kernels": kern})
        st.close()
    elif args.workload == "backward":
        w = synth.HYBRID_BWD_F32
        x = synth.make_inputs_device(w, seed=w.seed_base)
        g = torch.Generator(device="cuda")
        g.manual_seed(w.seed_base + 1)
        dout = torch.randn(x["q"].shape, generator=g, device="cuda")
        grads = tuple(torch.zeros_like(x["q"]) for _ in range(3))
        q, k, v, a = x["q"], x["k"], x["v"], x["alpha"]
        ns, nd = w.n_swa, w.n_dswa
        side = torch.cuda.Stream()

        def step():
            # the GLA heads' reverse recurrence (one CTA per head) runs beside the softmax heads
            main = torch.cuda.current_stream()
            side.wait_stream(main)
            kta.gla_bwd(q, k, v, a, dout, heads=(ns + nd, w.H), out=grads, stream=side)
            kta.swa_bwd(q, k, v, dout, P=w.P, W=w.W_swa, heads=(0, ns), out=grads)
            kta.dswa_bwd(q, k, v, dout, P=w.P, W=w.W_dswa, dil=w.dil, heads=(ns, ns + nd),
                         out=grads)
            main.wait_stream(side)
        steps, warm = min(args.steps, 5), max(1, min(args.warmup, 3))
        clk = ClockSampler("0")
        clk.start()
        ms = _device_ms(step, steps, warm)
        clocks = clk.stop() or {}
        kern = _traced(step, steps)
        sm_mhz = clocks.get("sm_mhz") or 1965.0
        peak = fp32_alu_tflops(sm_mhz)
        fl = softmax_bwd_flops(w)
        top = max(fl, key=lambda n: kern.get(n, {}).get("ms_per_step", 0.0))
        k_ms = kern[top]["ms_per_step"]
        lines.append({
            "workload": w.name, "metric": "hybrid layer reverse mode tokens/s (fp32)",
            "unit": "tokens/s", "value": w.B * w.N / (ms / 1e3), "ms_per_step": ms,
            "steps": steps, "warmup": warm, "dtype": "f32",
            "config": {"B": w.B, "F": w.F, "P": w.P, "H": w.H, "d": w.d},
            "roofline": {"kernel": top, "bound": "alu", "unit": "TFLOP/s",
                         "achieved": fl[top] / (k_ms / 1e3) / 1e12, "peak": peak,
                         "frac": fl[top] / (k_ms / 1e3) / 1e12 / peak,
                         "peak_source": f"fp32 FMA lanes x median SM clock {sm_mhz:.0f} MHz"},
            "clocks": clocks, "kernels": kern})
    elif args.workload == "layer":
        w = synth.HYBRID_BF16
        C, hd = w.H * w.d, w.H * w.d
        g = torch.Generator(device="cuda")
        g.manual_seed(w.seed_base + 7)
        x = torch.randn((w.B, w.N, C), generator=g, device="cuda").to(torch.bfloat16)
        n_in = 3 * hd + w.n_gla * w.d
        w_in = (torch.randn((n_in, C), generator=g, device="cuda") * C ** -0.5).to(torch.bfloat16)
        w_out = (torch.randn((C, hd), generator=g, device="cuda") * hd ** -0.5).to(torch.bfloat16)
        # alpha = sigmoid(W_alpha x + mu) with W_alpha x ~ N(0, 1): the input recipe's gates
        gate_bias = torch.full((w.n_gla * w.d,), w.alpha_mu, device="cuda")
        cfg = kta.cfg_from_workload(w)
        o = torch.empty((w.B, w.N, w.H, w.d), device="cuda", dtype=torch.bfloat16)
        y = torch.empty((w.B, w.N, C), device="cuda", dtype=torch.bfloat16)

        def step():
            q, k, v, a, _ = kta.qkv_gate_proj(x, w_in, H=w.H, d=w.d, n_gla=w.n_gla,
                                              gate_bias=gate_bias)
            kta.hybrid_fwd(cfg, q, k, v, a, out=o)
            kta.linear(o.view(w.B, w.N, hd), w_out, out=y)
        clk = ClockSampler("0")
        clk.start()
        ms = _device_ms(step, args.steps, args.warmup)
        clocks = clk.stop() or {}
        kern = _traced(step, args.steps)
        pf = layer_proj_flops(w)
        k_ms = kern["proj_gemm"]["ms_per_step"]
        tc_s = float(peaks.get("bf16_tflops_sustained", tc))
        lines.append({
            "workload": "layer_bf16_F21_P1560_C3072", "unit": "tokens/s",
            "metric": "attention layer fwd tokens/s (q/k/v/gate projection + hybrid operator + "
                      "output projection)",
            "value": w.B * w.N / (ms / 1e3), "ms_per_step": ms, "steps": args.steps,
            "dtype": "bf16",
            "config": {"B": w.B, "F": w.F, "P": w.P, "H": w.H, "d": w.d, "C": C,
                       "proj_outputs": n_in},
            "roofline": {"kernel": "proj_gemm", "bound": "tensor", "unit": "TFLOP/s",
                         "algorithmic_tflop": pf / 1e12,
                         "achieved": pf / (k_ms / 1e3) / 1e12, "peak": tc,
                         "frac": pf / (k_ms / 1e3) / 1e12 / tc,
                         "frac_of_sustained": pf / (k_ms / 1e3) / 1e12 / tc_s,
                         "peak_source": peaks_kind},
            "clocks": clocks, "kernels": kern})
    elif args.workload == "seqshard":
        from hybrid_linear_temporal_kta_b200 import seqshard
        w = synth.HYBRID_BF16
        R = 4
        c = seqshard.ShardCfg(F=w.F, P=w.P, d=w.d, n_swa=w.n_swa, n_dswa=w.n_dswa,
                              n_gla=w.n_gla, W_swa=w.W_swa, W_dswa=w.W_dswa, dil=w.dil,
                              chunk=w.chunk)
        x = synth.make_inputs_device(w, seed=w.seed_base)
        ops = seqshard.KtaOps()
        cfg = kta.cfg_from_workload(w)
        o = torch.empty_like(x["q"])

        def whole():
            kta.hybrid_fwd(cfg, x["q"], x["k"], x["v"], x["alpha"], out=o)

        def split():
            seqshard.emulate_ranks(c, R, x["q"], x["k"], x["v"], x["alpha"], ops=ops)
        ms_w = _device_ms(whole, args.steps, args.warmup)
        ms_s = _device_ms(split, args.steps, args.warmup)
        kern = _traced(split, args.steps)
        lines.append({
            "workload": f"seqshard_bf16_F21_P1560_R{R}_emulated", "unit": "tokens/s",
            "metric": "hybrid layer split by frames over 4 ranks, all ranks run one after another "
                      "on one GPU (work and exchange overhead of the split, not a multi-GPU time)",
            "value": w.B * w.N / (ms_s / 1e3), "ms_per_step": ms_s, "steps": args.steps,
            "unsharded_ms": ms_w, "overhead": ms_s / ms_w,
            "frames_per_rank": [n for _, n in seqshard.frame_split(w.F, R)],
            "halo_frames": c.halo, "kernels": kern})
    elif args.workload == "backward_bf16":
        w = synth.HYBRID_BF16
        x = synth.make_inputs_device(w, seed=w.seed_base + 9)
        g = torch.Generator(device="cuda")
        g.manual_seed(w.seed_base + 10)
        dout = torch.randn(x["q"].shape, generator=g, device="cuda").to(torch.bfloat16)
        q, k, v, a = x["q"], x["k"], x["v"], x["alpha"]
        ns, nd = w.n_swa, w.n_dswa
        o = torch.empty_like(q)
        lse = [kta.softmax_fwd_lse(q, k, v, P=w.P, W=w.W_swa, heads=(0, ns), out=o)[1],
               kta.softmax_fwd_lse(q, k, v, P=w.P, W=w.W_dswa, dil=w.dil, heads=(ns, ns + nd),
                                   out=o)[1]]
        hg = (ns + nd, w.H)
        # the GLA heads' reverse mode is fp32: their inputs converted once, outside the timed steps
        qf, kf, vf, dof = (t.float() for t in (q, k, v, dout))
        grads = tuple(torch.zeros_like(q) for _ in range(3))
        grads_f = tuple(torch.zeros_like(qf) for _ in range(3))

        def step():
            # one after another: the fp32 GLA backward holds most SMs for its whole run (one
            # ~200 KB CTA per SM), so beside it the softmax kernels would only get leftover SMs
            kta.softmax_bwd_bf16(q, k, v, o, lse[0], dout, P=w.P, W=w.W_swa, heads=(0, ns),
                                 out=grads)
            kta.softmax_bwd_bf16(q, k, v, o, lse[1], dout, P=w.P, W=w.W_dswa, dil=w.dil,
                                 heads=(ns, ns + nd), out=grads)
            kta.gla_bwd(qf, kf, vf, a, dof, heads=hg, out=grads_f)
        clk = ClockSampler("0")
        clk.start()
        ms = _device_ms(step, args.steps, args.warmup)
        clocks = clk.stop() or {}
        kern = _traced(step, args.steps)
        n = visible_pairs(w)
        fl = {"win_bwd_dq": 6.0 * w.d * n, "win_bwd_dkv": 8.0 * w.d * n}
        roof = {}
        for kname, f_alg in fl.items():
            k_ms = kern[kname]["ms_per_step"]
            roof[kname] = {"bound": "tensor", "unit": "TFLOP/s",
                           "achieved": f_alg / (k_ms / 1e3) / 1e12, "peak": tc,
                           "frac": f_alg / (k_ms / 1e3) / 1e12 / tc, "peak_source": peaks_kind,
                           "algorithmic_tflop": f_alg / 1e12}
        top = max(fl, key=lambda kn: kern[kn]["ms_per_step"])
        lines.append({
            "workload": "hybrid_bwd_bf16_F21_P1560", "unit": "tokens/s",
            "metric": "hybrid layer reverse mode tokens/s (softmax heads bf16 on tensor cores, "
                      "GLA heads fp32)",
            "value": w.B * w.N / (ms / 1e3), "ms_per_step": ms, "steps": args.steps,
            "dtype": "bf16", "config": {"B": w.B, "F": w.F, "P": w.P, "H": w.H, "d": w.d},
            "roofline": dict(roof[top], kernel=top), "kernel_rooflines": roof,
            "clocks": clocks, "kernels": kern})
    else:  # sweep
        for F in (8, 16, 32, 64, 128, 256):
            w = synth.sweep_workload(F)
            x = synth.make_inputs_device(w, seed=w.seed_base + F)
            cfg = kta.cfg_from_workload(w)
            o = torch.empty_like(x["q"])

            def hyb():
                kta.hybrid_fwd(cfg, x["q"], x["k"], x["v"], x["alpha"], out=o)

            def full():
                kta.swa_fwd(x["q"], x["k"], x["v"], P=w.P, W=w.F, out=o)
            ms_h = _device_ms(hyb, args.steps, args.warmup)
            steps_f = max(1, min(args.steps, 3 if F >= 128 else args.steps))
            ms_f = _device_ms(full, steps_f, min(args.warmup, 1))
            fl_h = softmax_flops(w)
            t_star_h = max(fl_h / (tc * 1e12), (8.0 * w.d * w.B * w.N * (w.n_swa + w.n_dswa) +
                                                gla_bytes(w)) / (hbm * 1e9))
            fl_f = full_causal_flops(w)
            lines.append({
                "workload": w.name, "metric": "tokens/s, hybrid vs full frame-causal attention",
                "unit": "tokens/s", "F": F, "N": w.N,
                "hybrid": {"value": w.B * w.N / (ms_h / 1e3), "ms": ms_h,
                           "softmax_tflops": fl_h / 1e12, "t_star_ms": t_star_h * 1e3,
                           "frac": t_star_h / (ms_h / 1e3)},
                "full_causal": {"value": w.B * w.N / (ms_f / 1e3), "ms": ms_f,
                                "tflops": fl_f / 1e12,
                                "achieved_tflops": fl_f / (ms_f / 1e3) / 1e12,
                                "frac": fl_f / (ms_f / 1e3) / 1e12 / tc},
                "speedup": ms_f / ms_h})
            del x, o
            torch.cuda.empty_cache()
    kta.device_status()
    for ln in lines:
        print(json.dumps(ln), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload != "hybrid":
        return run_other(args)
    return run_kta(args)


if __name__ == "__main__":
    sys.exit(main())
