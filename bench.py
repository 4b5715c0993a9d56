#!/usr/bin/env python
"""Benchmark of the CPR Gated DeltaNet layer (one JSON line on rank 0).

Metric: CPR-GDN tokens/s per layer on the rollout-prefill shape (5 x 2048
tokens packed, H=16, d_k=d_v=128, chunk 64, bf16 q/k/v, fp32 beta/g/state),
with the decode shape (256 sequences x 1 token, prefixes uniform in
[1, 2047], 512 consecutive steps) reported in the same line under "decode".
One step = one gdn_cpr_forward over the whole batch (chunk table, boundary
prep, boundary walk, intra-chunk fill).  Inputs are resident in HBM; L2 is
flushed (a 256 MiB write) before every timed step, outside the step's
events.  Per-kernel times come from CUDA events the library records on the
launching stream between its kernels.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); every rank runs its own batch
(weak scaling, no collective on the data path); the reported time is the
max over ranks.  --impl reference times the fp64 CPU oracle on the host.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CPR-GDN tokens/s per layer (prefill 5x2048, decode 256x1); % HBM roofline"
H, D, C = 16, 128, 64
PREFILL_LENS = [2048] * 5
FLUSH_BYTES = 256 << 20
PAGES_H100 = {"prefill_ms": 1.412, "decode_ms": 0.0846, "trainer_fwd_bwd_ms": 7.386}
# The per-layer table's three layouts on H100 (ms; trainer row is forward +
# backward): native mixed, recurrent everywhere, CPR.
PAGES_H100_LAYOUTS = {"prefill": (0.844, 3.639, 1.412), "trainer_fwd_bwd": (5.177, 22.863, 7.386),
                      "decode": (0.0612, 0.0612, 0.0846)}


# Source files whose kernels a traffic figure belongs to: a recorded figure is
# reported only while these files hash to what they were when it was captured.
TRAFFIC_SOURCES = {
    "forward": ("gdn_kernels.cu", "gdn_boundary.cuh", "gdn_common.cuh", "gdn_fill.cuh",
                "gdn_mma.cuh", "gdn_umma.cuh", "gdn_layout.h"),
    "backward": ("gdn_backward.cu", "gdn_adjoint.cuh", "gdn_boundary.cuh", "gdn_common.cuh",
                 "gdn_fill.cuh",
                 "gdn_mma.cuh", "gdn_umma.cuh", "gdn_layout.h"),
    "pik": ("gdn_pik.cu", "gdn_mma.cuh", "gdn_umma.cuh"),
    "native": ("gdn_native.cuh", "gdn_boundary.cuh", "gdn_common.cuh", "gdn_fill.cuh",
               "gdn_mma.cuh", "gdn_umma.cuh"),
    "recurrent": ("gdn_recurrent.cu", "gdn_fill.cuh", "gdn_common.cuh", "gdn_mma.cuh"),
}


def sources_sha256(group: str) -> str:
    """SHA-256 over the kernel source files of one group (in the order listed)."""
    import hashlib
    csrc = os.path.join(ROOT, "rl_train_numerics_b200", "csrc")
    h = hashlib.sha256()
    for name in TRAFFIC_SOURCES[group]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def ncu_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` (dram__bytes_read.sum + dram__bytes_write.sum
    from a single-kernel ncu capture, profiles/ncu_traffic.json), or None when its
    kernel sources have changed since that capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
            rec = json.load(f)["entries"].get(kernel)
        if rec is None or sources_sha256(rec["group"]) != rec["sources_sha256"]:
            return None
        return rec["bytes"]
    except (OSError, ValueError, KeyError):
        return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", 0.0)),
                "sm_max_mhz": float(p.get("sm_max_mhz", 1965.0)), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0, "source": "fallback"}


# ----------------------------------------------------------------------------
# Algorithmic work, per unit of each measured kernel
# ----------------------------------------------------------------------------

def fill_flops(T, H_, d):
    """Intra-chunk fill: per token and head 3 d^2 fused multiply-adds = 6 d^2 flops
    (the dot with k, the rank-one update of the scaled state, the dot with q)."""
    return 6.0 * d * d * T * H_


def walk_flops(n_full_chunk_heads, d, c=C):
    """Boundary walk per full chunk and head: U = U~ - W S^T (c x d x d MACs) and
    S' = g S + Ud^T K (d x c x d MACs): 4 c d^2 flops."""
    return 4.0 * c * d * d * n_full_chunk_heads


def prep_flops(n_full_chunk_heads, d, c=C):
    """Boundary prep per full chunk and head: K K^T, W, U~ (3 c^2 d MACs)."""
    return 6.0 * c * c * d * n_full_chunk_heads


def prefill_bytes(lens, H_, d, in_bytes=2, out_bytes=2):
    """Minimal HBM bytes of a forward: read q,k,v,beta,g, write o and the two final
    states.  Two-pass bytes add the boundary states written by pass 1 and read by
    pass 2 and pass 1's re-read of k,v,beta,g."""
    T = sum(lens)
    n = len(lens)
    io = T * H_ * (3 * d * in_bytes + 8 + d * out_bytes)
    finals = 2 * n * H_ * d * d * 4
    chunks = sum((L + C - 1) // C for L in lens)
    full = sum(L // C for L in lens)
    two_pass = io + finals + 2 * chunks * H_ * d * d * 4 + full * C * H_ * (2 * d * in_bytes + 8)
    return io + finals, two_pass


def decode_step_bytes(n_rows, n_resync_units, H_, d, in_bytes=2, out_bytes=2):
    """Per token and head: read the running state and write it back (2 x 4 d^2),
    read q,k,v,beta,g, write o, append the token to the chunk buffer, read and
    write pos.  A unit that resyncs also reads the boundary state (4 d^2) and the
    C-token buffer; its running-state write is replaced by the boundary write."""
    per = 2 * 4 * d * d + 3 * d * in_bytes + 8 + d * out_bytes + 2 * d * in_bytes + 8 + 8
    extra = 4 * d * d + C * (2 * d * in_bytes + 8)
    return n_rows * H_ * per + n_resync_units * extra


# ----------------------------------------------------------------------------
# Clock sampling during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"gdn_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)),
                "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------
# Distributed plumbing
# ----------------------------------------------------------------------------

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank number over all ranks (device tensor for NCCL, host for gloo)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, max_ms: float, world: int) -> float:
    """Whole-job throughput: units all ranks processed / the slowest rank's time."""
    return world * units_per_rank / (max_ms / 1e3)


# ----------------------------------------------------------------------------
# Our arm
# ----------------------------------------------------------------------------

def bench_prefill(gdn, W, dev, rank, steps, warmup, flush):
    b = W.prefill(device=dev, seed=rank)
    T = b.total_tokens
    o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    srun = torch.empty((len(b.lengths), H, D, D), dtype=torch.float32, device=dev)
    sbnd = torch.empty_like(srun)
    ws = torch.zeros(gdn.forward_workspace_bytes(len(b.lengths), T, H, D, D), dtype=torch.uint8,
                     device=dev)

    def make_events():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        for e in evs:
            e.record()
        return evs

    # A timed step is the plain forward between two events (as a caller runs
    # it: its kernels are programmatic dependents of one another); the
    # per-kernel breakdown comes from separate steps with an event between
    # kernels, which serialises them and costs a few microseconds.
    def step(evs):
        if len(evs) == 2:
            evs[0].record()
            gdn.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, o=o, s_run_final=srun,
                        s_bnd_final=sbnd, workspace=ws)
            evs[1].record()
        else:
            gdn.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, o=o, s_run_final=srun,
                        s_bnd_final=sbnd, workspace=ws, kernel_events=evs)

    warm_evs = make_events()
    for _ in range(warmup):
        flush.zero_()
        step(warm_evs)
    torch.cuda.synchronize()
    if gdn.check_error(ws) != 0:
        raise RuntimeError("device error word set during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    torch.cuda.synchronize()
    return b, (o, srun, sbnd, ws), step, evs, make_events


def bench_e2e(gdn, b, dev, steps, warmup):
    """Host buffers in, host output back, through the public forward: every step
    copies its inputs from pinned host memory (H2D), runs the forward and copies
    o back (D2H), all inside the timed region.  Measured two ways:
      serial     one stream: H2D, forward, D2H back to back;
      pipelined  a streaming caller: H2D on one copy stream, forwards on a
                 compute stream, D2H on another copy stream, double-buffered
                 device inputs and outputs, so step i+1's H2D and step i-1's D2H
                 overlap step i's forward (events order every reuse of a buffer).
    Returns (serial ms, pipelined ms, h2d bytes, d2h bytes) per step."""
    host = [t.cpu().pin_memory() for t in (b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens)]
    devb = [[torch.empty_like(t, device=dev) for t in host] for _ in range(2)]
    T = b.total_tokens
    o = [torch.empty((T, H, D), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    o_host = [torch.empty((T, H, D), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    ws = torch.zeros(gdn.forward_workspace_bytes(len(b.lengths), T, H, D, D), dtype=torch.uint8,
                     device=dev)
    h2d = sum(t.numel() * t.element_size() for t in host)
    d2h = o_host[0].numel() * o_host[0].element_size()

    def serial_step():
        for dst, src in zip(devb[0], host):
            dst.copy_(src, non_blocking=True)
        gdn.forward(*devb[0], o=o[0], workspace=ws, want_states=False)
        o_host[0].copy_(o[0], non_blocking=True)

    for _ in range(warmup):
        serial_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        serial_step()
    e1.record()
    torch.cuda.synchronize()
    serial_ms = e0.elapsed_time(e1) / steps

    s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def pipelined(n):
        done_run, done_out = {}, {}
        for i in range(n):
            slot = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(done_run[i - 2])  # the forward of step i-2 read this slot
                for dst, src in zip(devb[slot], host):
                    dst.copy_(src, non_blocking=True)
                got = torch.cuda.Event()
                got.record(s_in)
            with torch.cuda.stream(s_run):
                s_run.wait_event(got)
                if i >= 2:
                    s_run.wait_event(done_out[i - 2])  # o of step i-2 has left the device
                gdn.forward(*devb[slot], o=o[slot], workspace=ws, want_states=False)
                done_run[i] = torch.cuda.Event()
                done_run[i].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done_run[i])
                o_host[slot].copy_(o[slot], non_blocking=True)
                done_out[i] = torch.cuda.Event()
                done_out[i].record(s_out)
        return done_out[n - 1]

    pipelined(max(warmup, 2))
    torch.cuda.synchronize()
    p0 = torch.cuda.Event(enable_timing=True)
    p0.record(s_in)
    s_run.wait_event(p0)
    s_out.wait_event(p0)
    last = pipelined(steps)
    p1 = torch.cuda.Event(enable_timing=True)
    s_out.wait_event(last)
    p1.record(s_out)
    torch.cuda.synchronize()
    pipe_ms = p0.elapsed_time(p1) / steps
    return serial_ms, pipe_ms, h2d, d2h


def bench_decode(gdn, W, dev, rank, steps, warmup, slots=256):
    prefix = W.decode_prefix_lengths(slots)
    pre = W.make_batch(prefix, H, D, D, seed=100 + rank, device=dev)
    sscale = torch.empty((slots, H), device=dev)
    _, srun, sbnd, ws = gdn.forward(pre.q, pre.k, pre.v, pre.beta, pre.g, pre.cu_seqlens,
                                    s_run_scale=sscale)
    st = gdn.DecodeState(slots, H, D, D, device=dev)
    gdn.decode_state_from_prefill(st, pre.k, pre.v, pre.beta, pre.g, pre.cu_seqlens, srun, sbnd,
                                  s_run_scale=sscale)
    del pre, srun, sbnd, ws
    torch.cuda.empty_cache()  # keep only the decode state resident
    n_tok = warmup + steps
    toks = W.decode_tokens(n_tok, slots, H, D, D, seed=200 + rank, device=dev)
    o = torch.empty((slots, H, D), dtype=torch.bfloat16, device=dev)
    for s in range(warmup):
        gdn.decode_step(st, toks[0][s], toks[1][s], toks[2][s], toks[3][s], toks[4][s], o=o)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        s = warmup + i
        ev[i][0].record()
        gdn.decode_step(st, toks[0][s], toks[1][s], toks[2][s], toks[3][s], toks[4][s], o=o)
        ev[i][1].record()
    torch.cuda.synchronize()
    if gdn.check_error(st.error) != 0:
        raise RuntimeError("device error word set during decode")
    times = [a.elapsed_time(b_) for a, b_ in ev]
    # which units resynced at each timed step: pos before the step == C - 1
    resync = [sum(1 for P in prefix if (P + warmup + i) % C == C - 1) for i in range(steps)]
    nbytes = sum(decode_step_bytes(slots, r * H, H, D) for r in resync)
    return sum(times), nbytes, resync


def run_decode_part(gdn, W, dev, rank, world, args, peaks):
    slots = args.decode_slots
    dec_ms_total, dec_bytes, resync = bench_decode(gdn, W, dev, rank, args.decode_steps,
                                                   min(16, args.decode_steps), slots)
    dec_ms_total = max_over_ranks(dec_ms_total, world)
    dec_ms = dec_ms_total / args.decode_steps
    dec_gbs = dec_bytes / (dec_ms_total / 1e3) / 1e9
    return {"workload": f"{slots} sequences x 1 token per step, prefixes uniform in "
                        f"[1, 2047], H={H}, d={D}, C={C}, bf16 in/out, fp32 state",
            "steps": args.decode_steps, "ms_per_step": round(dec_ms, 5),
            "tokens_per_s": round(world * slots / (dec_ms / 1e3), 1),
            "resync_units_per_step": round(float(np.mean(resync)) * H, 2),
            "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(dec_gbs / peaks["hbm_gbs"], 4),
                         "traffic": ncu_traffic("decode_step")},
            "pages_h100_ms": PAGES_H100["decode_ms"]}


def native_out_bytes(lens, H_, d, c=C, pack=65920):
    """Algorithmic bytes of the chunked layout's output kernel: per (chunk, head)
    the entry state (fp32 d x d), the chunk's pack, its queries (bf16), g and
    its outputs (bf16)."""
    tot = 0
    for L in lens:
        for a in range(0, L, c):
            n = min(c, L - a)
            tot += H_ * (d * d * 4 + pack + n * d * 2 + n * 4 + n * d * 2)
    return tot


def _mean_ms(fn, steps, warmup, flush):
    """Mean device time of fn() over `steps` calls (L2 flushed before each),
    and the per-kernel split when fn takes 5 recorded events."""
    for _ in range(warmup):
        flush.zero_()
        fn(None)
    torch.cuda.synchronize()
    evs = []
    for _ in range(steps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        for x in e:
            x.record()
        evs.append(e)
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        fn(evs[i])
    torch.cuda.synchronize()
    total = sum(e[0].elapsed_time(e[4]) for e in evs) / steps
    split = [sum(e[j].elapsed_time(e[j + 1]) for e in evs) / steps for j in range(4)]
    return total, split


def run_layouts_part(gdn, W, dev, rank, world, args, flush, cpr_decode_ms, peaks):
    """The per-layer table's three layouts on this GPU: CPR (gdn_cpr_forward),
    native mixed (gdn_native_forward: chunked outputs, recurrent decode) and
    recurrent everywhere (gdn_recurrent_forward / gdn_recurrent_decode_step),
    on the rollout prefill and trainer-forward batches and the 256-row decode."""
    out = {}
    for name, b in (("prefill", W.prefill(device=dev, seed=rank)),
                    ("trainer_forward", W.trainer(device=dev, seed=rank))):
        T, N = b.total_tokens, len(b.lengths)
        o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
        s = torch.empty((N, H, D, D), dtype=torch.float32, device=dev)
        sb = torch.empty_like(s)
        ws = torch.zeros(gdn.forward_workspace_bytes(N, T, H, D, D), dtype=torch.uint8, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        args_in = (b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens)

        def cpr(evs):
            gdn.forward(*args_in, o=o, s_run_final=s, s_bnd_final=sb, workspace=ws,
                        kernel_events=evs)

        def nat(evs):
            gdn.native_forward(*args_in, o=o, s_final=s, s_bnd_final=sb, workspace=ws,
                               kernel_events=evs)

        def rec(evs):
            if evs is not None:
                evs[0].record()
            gdn.recurrent_forward(*args_in, o=o, s_final=s, error=err)
            if evs is not None:
                for e in evs[1:]:
                    e.record()

        t_cpr, k_cpr = _mean_ms(cpr, args.steps, args.warmup, flush)
        t_nat, k_nat = _mean_ms(nat, args.steps, args.warmup, flush)
        t_rec, _ = _mean_ms(rec, args.steps, args.warmup, flush)
        if gdn.check_error(ws) != 0 or gdn.check_error(err) != 0:
            raise RuntimeError("device error word set in the layout comparison")
        t_cpr, t_nat, t_rec = (max_over_ranks(x, world) for x in (t_cpr, t_nat, t_rec))
        nb = native_out_bytes(b.lengths, H, D)
        nat_gbs = nb / (max_over_ranks(k_nat[3], world) / 1e3) / 1e9
        rec_tf = fill_flops(T, H, D) / (t_rec / 1e3) / 1e12
        fp32_peak = 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12
        out[name] = {
            "native_outputs_roofline": {
                "kernel": "k_native_tc", "bound": "hbm", "achieved": round(nat_gbs, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(nat_gbs / peaks["hbm_gbs"], 4),
                "traffic": ncu_traffic("native_outputs") if name == "prefill" else None,
                "algorithmic_bytes": nb},
            "recurrent_roofline": {
                "kernel": "k_recur", "bound": "alu", "achieved": round(rec_tf, 2),
                "peak": round(fp32_peak, 2), "unit": "TFLOP/s",
                "frac": round(rec_tf / fp32_peak, 4),
                "traffic": ncu_traffic("recurrent_forward") if name == "prefill" else None},
            "tokens": T, "cpr_ms": round(t_cpr, 5), "native_ms": round(t_nat, 5),
            "recurrent_ms": round(t_rec, 5),
            "native_kernels_ms": dict(zip(["chunk_table", "boundary_prep", "boundary_walk",
                                           "chunked_outputs"], [round(x, 5) for x in k_nat])),
            "cpr_over_native": round(t_cpr / t_nat, 3),
            "recurrent_over_native": round(t_rec / t_nat, 3),
            "cpr_over_recurrent": round(t_cpr / t_rec, 3)}
    nat_p, rec_p, cpr_p = PAGES_H100_LAYOUTS["prefill"]
    out["prefill"]["pages_h100"] = {"native_ms": nat_p, "recurrent_ms": rec_p, "cpr_ms": cpr_p,
                                    "cpr_over_native": round(cpr_p / nat_p, 3),
                                    "recurrent_over_native": round(rec_p / nat_p, 3)}
    nat_t, rec_t, cpr_t = PAGES_H100_LAYOUTS["trainer_fwd_bwd"]
    out["trainer_forward"]["pages_h100_fwd_bwd"] = {
        "native_ms": nat_t, "recurrent_ms": rec_t, "cpr_ms": cpr_t,
        "cpr_over_native": round(cpr_t / nat_t, 3),
        "recurrent_over_native": round(rec_t / nat_t, 3),
        "note": "the pages' trainer row is forward + backward; the layouts here are forwards"}
    # decode: the recurrent step (the native and recurrent layouts' decode)
    slots, steps = args.decode_slots, 128
    st = torch.zeros((slots, H, D, D), dtype=torch.float32, device=dev)
    sc = torch.ones((slots, H), dtype=torch.float32, device=dev)
    toks = W.decode_tokens(16 + steps, slots, H, D, D, seed=300 + rank, device=dev)
    o = torch.empty((slots, H, D), dtype=torch.bfloat16, device=dev)
    for i in range(16):
        gdn.recurrent_decode_step(toks[0][i], toks[1][i], toks[2][i], toks[3][i], toks[4][i],
                                  st, sc, o=o)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        j = 16 + i
        ev[i][0].record()
        gdn.recurrent_decode_step(toks[0][j], toks[1][j], toks[2][j], toks[3][j], toks[4][j],
                                  st, sc, o=o)
        ev[i][1].record()
    torch.cuda.synchronize()
    t_rd = max_over_ranks(sum(a.elapsed_time(b_) for a, b_ in ev) / steps, world)
    nat_d, _, cpr_d = PAGES_H100_LAYOUTS["decode"]
    out["decode"] = {"recurrent_ms_per_step": round(t_rd, 5),
                     "cpr_ms_per_step": None if cpr_decode_ms is None else round(cpr_decode_ms, 5),
                     "cpr_over_recurrent": None if cpr_decode_ms is None
                     else round(cpr_decode_ms / t_rd, 3),
                     "pages_h100": {"recurrent_ms": nat_d, "cpr_ms": cpr_d,
                                    "cpr_over_recurrent": round(cpr_d / nat_d, 3)}}
    return out


def bwd_gemm_flops(lengths, H, D):
    """Algorithmic FLOPs of the backward's chunk products: per chunk of length L,
    Y (lower triangle incl. diagonal) and X and K K^T (strict) over d, the three
    L x d x d products (DO S_a, W S_a, U mu_e), A K and A^T Q (triangles incl.
    diagonal) and (B + B^T) K (off-diagonal), the dbeta / dg dots (w . v,
    k . (W S_a), k . (U mu_e), q . dq per token, <mu_e, S_a>), two FLOPs per
    multiply-add."""
    mac = 0
    for Ln in lengths:
        for c0 in range(0, Ln, C):
            L = min(C, Ln - c0)
            tri, stri = L * (L + 1) // 2, L * (L - 1) // 2
            mac += D * (3 * tri + 2 * stri + 2 * stri) + 3 * L * D * D + 4 * L * D + D * D
    return 2 * mac * H


def run_train_part(gdn, W, dev, rank, world, args, flush, peaks):
    """Trainer step: the forward (o and final states) and the backward (every
    gradient, from a fixed synthetic dL/do) over the 10240-token trainer batch,
    L2 flushed before every step outside its events."""
    b = W.trainer(device=dev, seed=rank)
    T, N = b.total_tokens, len(b.lengths)
    gen = torch.Generator(device=dev).manual_seed(1000 + rank)
    d_o = torch.randn((T, H, D), generator=gen, device=dev).to(torch.bfloat16)
    o = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    srun = torch.empty((N, H, D, D), dtype=torch.float32, device=dev)
    grads, ws = gdn.backward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, d_o)

    def make_events():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
        for e in evs:
            e.record()
        return evs

    # The forward runs on the backward's workspace, and the backward reuses its
    # first pass (boundary states) instead of running it again.  A timed step
    # is the plain forward + backward between two events; the forward /
    # backward split and the per-kernel times come from separate steps with an
    # event between kernels (which serialises them).
    def step(evs):
        if len(evs) == 2:
            evs[0].record()
            gdn.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, o=o, s_run_final=srun,
                        workspace=ws)
            gdn.backward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, d_o, grads=grads,
                         workspace=ws, reuse_forward=True)
            evs[1].record()
            return
        gdn.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, o=o, s_run_final=srun,
                    workspace=ws, kernel_events=evs[:5])
        gdn.backward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, d_o, grads=grads, workspace=ws,
                     reuse_forward=True, kernel_events=evs[5:])

    steps, warmup = args.steps, args.warmup
    warm = make_events()
    for _ in range(warmup):
        flush.zero_()
        step(warm)
    plain = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        step(plain[i])
    torch.cuda.synchronize()
    barrier(world)
    ms_plain = float(np.mean([e[0].elapsed_time(e[1]) for e in plain]))
    evs = [make_events() for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        step(evs[i])
    torch.cuda.synchronize()
    if gdn.check_error(ws) != 0:
        raise RuntimeError("device error word set in the trainer step")
    el = lambda a, z: float(np.mean([e[a].elapsed_time(e[z]) for e in evs]))  # noqa: E731
    fwd, bwd = el(0, 4), el(5, 9)
    kern = {"fwd_chunk_table": el(0, 1), "fwd_boundary_prep": el(1, 2),
            "fwd_boundary_walk": el(2, 3), "fwd_intra_chunk_fill": el(3, 4),
            "bwd_adjoint_prep_walk": el(6, 7), "bwd_w_solve_and_u": el(7, 8),
            "bwd_chunk_products": el(8, 9)}
    ms = max_over_ranks(ms_plain, world)
    fwd_max = max_over_ranks(fwd, world)
    fp32_peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    gflop = bwd_gemm_flops(b.lengths, H, D) / 1e9
    achieved = gflop / kern["bwd_chunk_products"]  # GFLOP per ms = TFLOP/s
    # The trainer forward on its own: the fill's FP32 roofline and the whole
    # forward's HBM fraction on the minimal and two-pass byte counts.
    fill_tf = fill_flops(T, H, D) / 1e9 / kern["fwd_intra_chunk_fill"]
    minimal, two_pass = prefill_bytes(b.lengths, H, D)
    hbm_bps = peaks["hbm_gbs"] * 1e9
    return {"workload": f"trainer: {T} tokens as {N} documents (lengths {b.lengths}), H={H}, "
                        f"d_k=d_v={D}, C={C}, bf16 q/k/v/do, fp32 beta/g/state/gradients",
            "steps": steps, "ms_per_step": round(ms, 5), "fwd_ms": round(fwd, 5),
            "bwd_ms": round(bwd, 5), "tokens_per_s": round(world * T / (ms / 1e3), 1),
            "timing_note": "ms_per_step: plain forward + backward between two events; fwd_ms, "
                           "bwd_ms and kernels_ms: separate steps with an event between kernels "
                           f"({round(fwd + bwd, 5)} ms per step)",
            "fwd_tokens_per_s": round(world * T / (fwd_max / 1e3), 1),
            "fwd_roofline": {"kernel": "fwd_intra_chunk_fill", "bound": "alu",
                             "achieved": round(fill_tf, 2), "peak": round(fp32_peak, 2),
                             "unit": "TFLOP/s", "frac": round(fill_tf / fp32_peak, 4),
                             "traffic": ncu_traffic("trainer_intra_chunk_fill"),
                             "peak_source": "148 SMs x 128 FP32 lanes x 2 flop x sm_max_mhz "
                                            "(nominal)"},
            "fwd_hbm_roofline": {"minimal_bytes": minimal, "two_pass_bytes": two_pass,
                                 "frac_minimal": round(minimal / (fwd_max / 1e3) / hbm_bps, 4),
                                 "frac_two_pass": round(two_pass / (fwd_max / 1e3) / hbm_bps, 4),
                                 "peak_gbs": peaks["hbm_gbs"], "peak_source": peaks["source"]},
            "kernels_ms": {k: round(v, 5) for k, v in kern.items()},
            "bwd_roofline": {"kernel": "bwd_chunk_products", "bound": "alu",
                             "achieved": round(achieved, 2), "peak": round(fp32_peak, 2),
                             "unit": "TFLOP/s", "frac": round(achieved / fp32_peak, 4),
                             "traffic": ncu_traffic("bwd_chunk_products"),
                             "peak_source": "148 SMs x 128 FP32 lanes x 2 flop x sm_max_mhz "
                                            "(nominal)"},
            # forward: chunk table, prep, walk, fill; backward on the forward's
            # first pass: adjoint prep, reverse walk, W solve + u, chunk products
            "gpu_launches_per_step": 4 + 4,
            "l2": "flushed (256 MiB write) before every timed step",
            "pages_h100_ms": PAGES_H100["trainer_fwd_bwd_ms"]}


PIK_SHAPE = (8192, 8192, 8192, 8)  # M, N, K, leaves (M = N = K = --pik-size)


def run_pik_part(gdn, dev, rank, world, args, flush, peaks):
    """Parallelism-invariant K-leaf GEMM: C = A B^T, M = N = K = 8192, 8 leaves,
    bf16 in, fp32 out, one emulated rank; L2 flushed before every timed call.
    cuBLAS bf16 (torch.matmul) on the same operands is timed beside it."""
    M = N = K = args.pik_size
    L = PIK_SHAPE[3]
    gen = torch.Generator(device=dev).manual_seed(2000 + rank)
    A = torch.randn((M, K), generator=gen, device=dev).to(torch.bfloat16)
    B = torch.randn((N, K), generator=gen, device=dev).to(torch.bfloat16)
    C = torch.empty((M, N), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.empty(max(gdn.pik_workspace_bytes(M, N, K, L, 1), 16), dtype=torch.uint8,
                     device=dev)

    def timed(fn, steps):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for _ in range(args.warmup):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        for e0, e1 in evs:
            flush.zero_()
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        return float(np.mean([e0.elapsed_time(e1) for e0, e1 in evs]))

    steps = max(3, min(args.steps, 10))
    ms = timed(lambda: gdn.pik_gemm(A, B, L, 1, C=C, workspace=ws, error=err), steps)
    if gdn.check_error(err) != 0:
        raise RuntimeError("device error word set by the K-leaf GEMM")
    ms_cublas = timed(lambda: torch.matmul(A, B.T), steps)
    ms = max_over_ranks(ms, world)
    tflops = 2.0 * M * N * K / (ms / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    return {"workload": f"C = A B^T, M=N=K={M}, {L} leaves of {K // L}, bf16 in, fp32 out, "
                        "1 emulated rank (the bits are the same for every rank count)",
            "ms": round(ms, 4), "tflops": round(world * tflops, 1),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                         "traffic": ncu_traffic("pik_gemm"),
                         "peak_source": f"measured cuBLAS bf16 burst ({peaks['source']})"},
            "cublas_bf16_ms": round(ms_cublas, 4),
            "cublas_bf16_tflops": round(2.0 * M * N * K / (ms_cublas / 1e3) / 1e12, 1),
            "gpu_launches_per_call": 1,  # k_pik_gemm (one rank: no combine)
            "l2": "flushed (256 MiB write) before every timed call"}


def _oracle_prefill_passes(oracle, b, seconds, threads=None, max_passes=64):
    """Whole-batch oracle passes over `b` (every sequence and head) until about
    `seconds` have gone by; returns (tokens, passes, elapsed s)."""
    done, passes, t0 = 0, 0, time.perf_counter()
    while passes < max_passes and (passes == 0 or time.perf_counter() - t0 < seconds):
        oracle.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens.numpy(), threads=threads)
        done += b.total_tokens
        passes += 1
    return done, passes, time.perf_counter() - t0


def cpu_baseline_sample(W, seconds=8.0):
    """The fp64 oracle as it stands on the host cores.  The headline figure:
    all cores, whole passes over the 5x2048 prefill batch (all 80 sequence-head
    units, the GPU arm's workload).  Beside it: one core on whole sequence-head
    units of the same batch, the 10240-token trainer forward on all cores, and
    the 256-row decode step (one token per row and head, the state carried as
    h0) on all cores."""
    import oracle
    b = W.prefill(device="cpu", seed=0)
    done, passes, el = _oracle_prefill_passes(oracle, b, seconds)
    out = {"value": round(done / el, 1), "unit": "tokens/s", "cores": oracle.max_threads(),
           "kind": "oracle",
           "sample": f"{passes} pass(es) over the whole 5x2048 prefill batch, {H} heads "
                     f"({done} tokens), fp64 token loop, {el:.1f} s"}
    # one core: whole (sequence, head) units, counted as token-heads / H
    cu = b.cu_seqlens.tolist()
    units, th, t0 = 0, 0, time.perf_counter()
    while units < 2 * H and (units == 0 or time.perf_counter() - t0 < 3.0):
        n, h = units % len(b.lengths), (units // len(b.lengths)) % H
        sl, hs = slice(cu[n], cu[n + 1]), slice(h, h + 1)
        oracle.forward(b.q[sl, hs], b.k[sl, hs], b.v[sl, hs], b.beta[sl, hs], b.g[sl, hs],
                       np.array([0, cu[n + 1] - cu[n]], np.int32), threads=1)
        th += cu[n + 1] - cu[n]
        units += 1
    el1 = time.perf_counter() - t0
    out["one_core"] = {"value": round(th / H / el1, 1), "unit": "tokens/s", "cores": 1,
                       "sample": f"{units} (sequence, head) units of the prefill batch "
                                 f"({th} token-heads = {th / H:.0f} tokens), {el1:.1f} s"}
    # trainer forward, all cores
    bt = W.trainer(device="cpu", seed=0)
    done, passes, el = _oracle_prefill_passes(oracle, bt, 3.0, max_passes=8)
    out["trainer_forward"] = {"value": round(done / el, 1), "unit": "tokens/s",
                              "cores": oracle.max_threads(),
                              "sample": f"{passes} pass(es) over the 10240-token trainer batch "
                                        f"(5 documents, {H} heads), {el:.1f} s"}
    # decode: 256 rows x 1 token per step, fp64 state carried between steps
    slots = 256
    toks = W.decode_tokens(32, slots, H, D, D, seed=2, device="cpu")
    S = np.zeros((slots, H, D, D))
    cu1 = np.arange(slots + 1, dtype=np.int32)
    steps, t0 = 0, time.perf_counter()
    while steps < 32 and (steps == 0 or time.perf_counter() - t0 < 3.0):
        _, S = oracle.forward(*(t[steps] for t in toks), cu1, h0=S)
        steps += 1
    eld = time.perf_counter() - t0
    out["decode"] = {"value": round(steps * slots / eld, 1), "unit": "tokens/s",
                     "cores": oracle.max_threads(),
                     "sample": f"{steps} decode step(s) of {slots} rows x {H} heads from a "
                               f"zero state (one fp64 token-loop step per row), {eld:.1f} s"}
    return out


def run_ours(args):
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from rl_train_numerics_b200 import _abi as gdn
    from rl_train_numerics_b200 import workloads as W

    if args.only == "bwd-small":
        # Profiling case for full ncu captures of the backward kernels: two
        # backward calls on 2 x 1024 tokens, H = 8, d = 128, bf16; no JSON line.
        b = W.make_batch([1024, 1024], 8, D, D, dtype=torch.bfloat16, seed=3, device=dev)
        gen = torch.Generator(device=dev).manual_seed(4)
        d_o = torch.randn((b.total_tokens, 8, D), generator=gen, device=dev).to(torch.bfloat16)
        grads, ws = gdn.backward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, d_o)
        gdn.backward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, d_o, grads=grads, workspace=ws)
        if gdn.check_error(ws) != 0:
            raise RuntimeError("device error word set by the backward")
        return
    peaks = load_peaks()
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    b, bufs, step, evs, make_events = bench_prefill(gdn, W, dev, rank, args.steps, args.warmup,
                                                     flush)
    sampler = ClockSampler(local)
    sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for i in range(args.steps):
        flush.zero_()
        step(evs[i])
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - wall0
    # keep the sampler running on the same work for at least ~1.5 s
    t_soak = time.perf_counter()
    while wall + (time.perf_counter() - t_soak) < 1.5:
        flush.zero_()
        step(evs[0])
        torch.cuda.synchronize()
    clocks = sampler.stop()
    if gdn.check_error(bufs[3]) != 0:
        raise RuntimeError("device error word set in the timed region")
    total = sum(e[0].elapsed_time(e[1]) for e in evs)
    ms_step = max_over_ranks(total / args.steps, world)

    # Per-kernel breakdown: the same steps with an event between kernels.
    names = ["chunk_table", "boundary_prep", "boundary_walk", "intra_chunk_fill"]
    kevs = [make_events() for _ in range(args.steps)]
    torch.cuda.synchronize()
    for e in kevs:
        flush.zero_()
        step(e)
    torch.cuda.synchronize()
    per_k = np.zeros(4)
    instrumented = 0.0
    for e in kevs:
        for j in range(4):
            per_k[j] += e[j].elapsed_time(e[j + 1])
        instrumented += e[0].elapsed_time(e[4])
    per_k /= args.steps
    instrumented /= args.steps
    T = b.total_tokens
    value = weak_scaling_value(T, ms_step, world)

    lens = b.lengths
    full = sum(L // C for L in lens) * H
    work = {
        "intra_chunk_fill": ("alu", fill_flops(T, H, D)),
        "boundary_walk": ("alu", walk_flops(full, D)),
        "boundary_prep": ("alu", prep_flops(full, D)),
    }
    dom = max(range(4), key=lambda j: per_k[j])
    dom_name = names[dom]
    bound, flops = work.get(dom_name, ("alu", 0.0))
    fp32_peak = 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12  # TFLOP/s, FMA = 2
    achieved = flops / (per_k[dom] / 1e3) / 1e12
    roofline = {"kernel": dom_name, "bound": bound, "achieved": round(achieved, 2),
                "peak": round(fp32_peak, 2), "unit": "TFLOP/s",
                "frac": round(achieved / fp32_peak, 4), "traffic": ncu_traffic(dom_name),
                "peak_source": "148 SMs x 128 FP32 lanes x 2 flop x sm_max_mhz (nominal)"}
    minimal, two_pass = prefill_bytes(lens, H, D)
    hbm = {"minimal_bytes": minimal, "two_pass_bytes": two_pass,
           "frac_minimal": round(minimal / (ms_step / 1e3) / (peaks["hbm_gbs"] * 1e9), 4),
           "frac_two_pass": round(two_pass / (ms_step / 1e3) / (peaks["hbm_gbs"] * 1e9), 4),
           "peak_gbs": peaks["hbm_gbs"], "peak_source": peaks["source"]}

    e2e = None
    if args.only == "all":
        serial_ms, pipe_ms, h2d, d2h = bench_e2e(gdn, b, dev, args.steps, args.warmup)
        serial_ms = max_over_ranks(serial_ms, world)
        pipe_ms = max_over_ranks(pipe_ms, world)
        e2e = {"value": round(world * T / (pipe_ms / 1e3), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(pipe_ms, 4),
               "mode": "pipelined: H2D, forward and D2H on three streams, double-buffered, "
                       "every step's copies inside the timed region",
               "serial": {"value": round(world * T / (serial_ms / 1e3), 1),
                          "ms_per_step": round(serial_ms, 4),
                          "mode": "one stream: H2D, forward, D2H back to back"}}
    decode = None
    if args.only in ("all", "decode"):
        decode = run_decode_part(gdn, W, dev, rank, world, args, peaks)
    train = None
    if args.only in ("all", "train"):
        train = run_train_part(gdn, W, dev, rank, world, args, flush, peaks)
    pikr = None
    if args.only in ("all", "pik"):
        pikr = run_pik_part(gdn, dev, rank, world, args, flush, peaks)
    layouts = None
    if args.only in ("all", "layouts"):
        layouts = run_layouts_part(gdn, W, dev, rank, world, args, flush,
                                   None if decode is None else decode["ms_per_step"], peaks)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": round(value / (10240 / (PAGES_H100["prefill_ms"] / 1e3)), 3),
        "vs_baseline_note": "pages' H100 CPR prefill, 1.412 ms per 5x2048 tokens "
                            "(layer shape unstated): context, other hardware",
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": "rollout prefill: 5 sequences x 2048 tokens packed, H=16, "
                               "d_k=d_v=128, C=64, bf16 q/k/v/o, fp32 beta/g/state",
                   "global_batch": world * T, "seq_len": 2048, "parallelism": f"dp{world}",
                   "l2": "flushed (256 MiB write) before every timed step"},
        "roofline": roofline,
        "kernels_ms": {n: round(float(t), 5) for n, t in zip(names, per_k)},
        "kernels_ms_note": "from separate steps with an event between kernels (serialised, "
                           f"{round(instrumented, 5)} ms per step); ms_per_step is the plain "
                           "forward between two events",
        "hbm_roofline": hbm,
        "e2e": e2e,
        "decode": decode,
        "train_step": train,
        "pik_gemm": pikr,
        "layouts": layouts,
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
        "wall_s_timed_region": round(wall, 4),
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_sample(W)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------------------
# Reference arm: the fp64 oracle on the host cores
# ----------------------------------------------------------------------------

def run_reference(args):
    """The fp64 oracle as it stands, on the host cores, over the GPU arm's
    workload: each step is one whole pass over the 5x2048 prefill batch (every
    sequence and head)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from rl_train_numerics_b200 import workloads as W
    b = W.prefill(device="cpu", seed=0)
    cu = b.cu_seqlens.numpy()

    def one():
        oracle.forward(b.q, b.k, b.v, b.beta, b.g, cu)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    el = time.perf_counter() - t0
    value = args.steps * b.total_tokens / el
    sample = (f"each step: one whole pass over the 5x2048 prefill batch, all {H} heads "
              f"({b.total_tokens} tokens, fp64 token loop)")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "rollout prefill: 5 sequences x 2048 tokens packed, H=16, "
                                   "d_k=d_v=128, C=64, bf16 q/k/v/o, fp32 beta/g/state",
                       "global_batch": 10240, "seq_len": 2048, "parallelism": "host"},
            "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s",
                             "cores": oracle.max_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--decode-steps", type=int, default=512)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--only", choices=["all", "prefill", "decode", "train", "pik", "layouts",
                                      "bwd-small"],
                   default="all",
                   help="profiling aid: run only part of the benchmark")
    p.add_argument("--decode-slots", type=int, default=256)
    p.add_argument("--pik-size", type=int, default=PIK_SHAPE[0],
                   help="M = N = K of the K-leaf GEMM (profiling aid: a smaller case)")
    args = p.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
