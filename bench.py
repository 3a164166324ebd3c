#!/usr/bin/env python
"""Benchmark of the fused causal GQA attention, forward + backward, on B200.

One step = the whole hot path over one batch of the workload: the forward
kernel, then the three backward stages (preprocess, main, dQ finalize), all
through the C ABI on one stream.  The metric is attention TFLOP/s with causal
FLOPs counted as half of dense (fwd 2*B*Hq*S^2*D, bwd 5*B*Hq*S^2*D).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
        python bench.py --impl reference ...   (the fp64 CPU oracle, host cores)
The headline workload (default llm1b, B=4 S=2048 Hq=32 Hkv=8 D=64) gives the
line's value, roofline, e2e and cpu_baseline; the other four workloads are
timed after it the same way (fewer steps) and reported under "workloads", each
with its own clocks and oracle baseline; "rope" times the headline step with
the rotary embedding fused, "decode" two decode steps against a paged KV cache
(HBM roofline).  "e2e" is the same step from pinned host memory through the
public torch helpers, uploads and downloads inside the timed region, pipelined
over three streams, its results checked against the device step's.  Under
torchrun (N > 1) every rank runs its own batch of each workload (weak scaling;
no collective on the data path), or with --shard one problem's (b, kv) units.
Timing: CUDA events around each step on the launching stream, L2 flushed
before every step, outside the events (a 256 MiB write, then a 256 MiB read:
the read evicts the write's dirty lines, so their write-back does not land in
the timed kernels); the reported time is the max over ranks.  Rank 0 prints
one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

P_NOM_TFLOPS = 2250.0  # B200 dense bf16, NVIDIA's published figure
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "attention fwd / bwd TFLOP/s (bf16, causal) and % of B200 tensor peak"
# The sources each kernel is compiled from (its own header, the shared PTX
# helpers, and the host file with its launch configuration).
KERNEL_SOURCES = {
    "attn_fwd_kernel": ("attn_fwd.cuh", "sm100_ptx.cuh", "axis_attn.cu"),
    "attn_bwd_kernel": ("attn_bwd.cuh", "attn_rope.cuh", "sm100_ptx.cuh", "axis_attn.cu"),
    "attn_bwd_prep_kernel": ("attn_bwd.cuh", "axis_attn.cu"),
    "attn_bwd_dq_convert_kernel": ("attn_bwd.cuh", "attn_rope.cuh", "axis_attn.cu"),
}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK), "fallback"


def kernel_source_hash(kernel: str, read=None) -> str:
    """Hash of the sources `kernel` is built from; `read(name)` returns a
    source's bytes (default: the working tree)."""
    if read is None:
        def read(name):
            return open(os.path.join(ROOT, "causal_attention_fwd_b200", "csrc", name), "rb").read()
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        h.update(read(name))
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kernel, {})
    if e.get("workload") == workload and e.get("source_hash") == kernel_source_hash(kernel):
        return e.get("dram_bytes_per_launch")
    return None


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock, power and clock-event reasons of one GPU via NVML."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            handle = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    handle = h
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nvml, self.h = pynvml, handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that, do not guess
            self.err = repr(e)

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                t = time.time()
                mhz = n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM)
                rs = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                pw = n.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((t, mhz, rs, pw))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.th = threading.Thread(target=self._run, daemon=True)
            self.th.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.th.join()

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        inside = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples[-5:]
        mhz = statistics.median(s[1] for s in inside) if inside else None
        bits = 0
        for s in inside:
            bits |= s[2]
        reasons = [k for k, v in self.REASONS.items() if bits & v and k != "gpu_idle"]
        return {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(inside),
                "power_w_max": max((s[3] for s in inside), default=None)}


# ----------------------------------------------------------- reference arm
def oracle_head_seconds(w) -> float:
    """Rough time of the oracle on one whole query head (fwd + bwd): it was
    measured at 0.4 s for S = 2048, D = 64 and grows as S^2 D."""
    return 0.4 * (w.S / 2048.0) ** 2 * (w.D / 64.0)


def cpu_sample(w, budget_s: float, max_heads: int | None = None):
    """The oracle, as it stands, on a bounded sample of the workload.  Returns
    TFLOP/s counted like the GPU metric, the threads used, a description and
    the seconds spent.

    Whole query heads (each with its kv head, fwd + bwd) while one head fits
    the budget; otherwise (the longest sequences) sampled query rows through
    the oracle's row functions -- the forward rows and the dQ rows, which
    repeat the full backward's per-row work except its dK/dV accumulation --
    extrapolated to all B*Hq*S rows (so the figure overstates the oracle's
    throughput a little)."""
    import numpy as np

    import oracle
    from causal_attention_fwd_b200.synthetic import workload_inputs

    q, k, v, do = workload_inputs(w)
    G = w.Hq // w.Hkv
    flops = w.fwd_flops + w.bwd_flops
    if oracle_head_seconds(w) <= budget_s or max_heads is not None:
        per_head = flops / (w.B * w.Hq)
        done, t_total, n = 0, 0.0, 0
        while n == 0 or (t_total < budget_s and (max_heads is None or n < max_heads)):
            b, h = n % w.B, (n // w.B) % w.Hq
            sl = lambda t, hh: t[b:b + 1, :, hh:hh + 1].contiguous()  # noqa: E731
            qs, ks, vs, dos = sl(q, h), sl(k, h // G), sl(v, h // G), sl(do, h)
            t0 = time.perf_counter()
            oracle.attn_fwd(qs, ks, vs, w.scale, w.causal)
            oracle.attn_bwd(qs, ks, vs, dos, w.scale, w.causal)
            t_total += time.perf_counter() - t0
            done += 1
            n += 1
        tflops = done * per_head / t_total / 1e12
        desc = (f"{done} whole query head(s) of the workload, each fwd+bwd with its kv head "
                f"(B=1 Hq=1 Hkv=1 S={w.S} D={w.D}); {t_total:.1f} s; the forward runs on all threads, "
                f"the backward of one (b, kv) unit on one")
        return tflops, oracle.max_threads(), desc, t_total
    g = np.random.default_rng(99)
    rows_total = w.B * w.Hq * w.S
    done, t_total, R = 0, 0.0, 64
    while t_total < budget_s / 2:
        rows = [(int(g.integers(w.B)), int(g.integers(w.Hq)), int(g.integers(w.S))) for _ in range(R)]
        t0 = time.perf_counter()
        oracle.attn_fwd_rows(q, k, v, w.scale, w.causal, rows)
        oracle.attn_bwd_dq_rows(q, k, v, do, w.scale, w.causal, rows)
        t_total += time.perf_counter() - t0
        done += R
        R *= 2
    est = t_total / done * rows_total
    tflops = flops / est / 1e12
    desc = (f"extrapolated: {done} sampled query rows through the oracle's forward-row and dQ-row functions "
            f"({t_total:.1f} s), scaled to all {rows_total} rows (a full run would take ~{est:.0f} s)")
    return tflops, oracle.max_threads(), desc, t_total


def workload_config(w, world: int) -> dict:
    """The `config` object of the JSON line; the same for both arms."""
    return {"workload": f"{w.name}: {w.describe()}", "B": w.B, "S": w.S, "Hq": w.Hq, "Hkv": w.Hkv,
            "D": w.D, "global_batch": w.B * world, "parallelism": f"replicas x{world} (no collective)",
            "l2": "GPU arm: flushed before every step (256 MiB write + 256 MiB read, outside the timed events)"}


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return 0
    from causal_attention_fwd_b200.synthetic import WORKLOADS

    w = WORKLOADS[args.workload]
    import oracle

    oracle.build()
    times, vals = [], []
    desc, cores = "", oracle.max_threads()
    for s in range(args.warmup + args.steps):
        v, cores, desc, t = cpu_sample(w, 0.0, max_heads=1)  # one head per step
        if s >= args.warmup:
            times.append(t)
            vals.append(v)
    per_head = (w.fwd_flops + w.bwd_flops) / (w.B * w.Hq)
    value = per_head * len(times) / sum(times) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,sigma^2), bf16-rounded)",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": "one whole query head of the workload per step, fwd+bwd, fp64"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ------------------------------------------------------- multi-rank plumbing
def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch (weak scaling: independent problems)."""
    return base_seed + 100 * rank


def reduce_max(values, world: int, device=None):
    """Element-wise max over ranks of a list of floats (the slowest rank sets
    the time).  Uses the default process group when world > 1."""
    import torch

    t = torch.tensor(list(values), dtype=torch.float64)
    if world > 1:
        import torch.distributed as dist

        t = t.to(device) if device is not None else t
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        t = t.cpu()
    return [float(x) for x in t]


def whole_job_tflops(flops_per_step_per_rank: float, steps: int, max_ms: float, world: int) -> float:
    """Units all ranks processed divided by the slowest rank's device time."""
    return world * flops_per_step_per_rank * steps / (max_ms * 1e-3) / 1e12


# ---------------------------------------------------------------- GPU arm
STAGES = ["attn_fwd_kernel", "attn_bwd_prep_kernel", "attn_bwd_kernel", "attn_bwd_dq_convert_kernel"]


class Problem:
    """Device buffers of one workload and its step through the C ABI."""

    def __init__(self, aa, w, seed: int, dev, det: bool, host=None):
        import ctypes

        import torch

        from causal_attention_fwd_b200.synthetic import workload_inputs

        self.aa, self.w, self.det = aa, w, det
        self.host = workload_inputs(w, seed=seed) if host is None else host
        self.q, self.k, self.v, self.do = (t.to(dev) for t in self.host)
        B, Hq, S = w.B, w.Hq, w.S
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((B, Hq, S), device=dev, dtype=torch.float32)
        self.dq, self.dk, self.dv = torch.empty_like(self.q), torch.empty_like(self.k), torch.empty_like(self.v)
        size_fn = aa.axis_attn_bwd_det_workspace_bytes if det else aa.axis_attn_bwd_workspace_bytes
        self.ws_bytes = size_fn(B, Hq, w.Hkv, S, w.D)
        self.ws = torch.empty(self.ws_bytes, device=dev, dtype=torch.uint8)
        self.stream = torch.cuda.current_stream(dev)
        self.sp = ctypes.c_void_p(self.stream.cuda_stream)

    def _check(self, rc, what):
        if rc:
            raise self.aa.AxisAttnError(rc, what)

    def step(self, ev=None):
        """fwd, then the backward (three stages, or the deterministic call);
        ev: 5 events recorded between the stages."""
        aa, w, st = self.aa, self.w, self.stream
        B, Hq, Hkv, S, D, c = w.B, w.Hq, w.Hkv, w.S, w.D, int(w.causal)
        q, k, v, do = self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(), self.do.data_ptr()
        ws, wsb, sp = self.ws.data_ptr(), self.ws_bytes, self.sp
        rec = (lambda i: ev[i].record(st)) if ev else (lambda i: None)
        rec(0)
        self._check(aa.axis_attn_fwd(q, k, v, self.o.data_ptr(), self.lse.data_ptr(), B, Hq, Hkv, S, D, w.scale,
                                     c, sp), "fwd")
        rec(1)
        if self.det:  # one call, three kernels: timed as a whole (the stage events coincide)
            rec(2)
            rec(3)
            self._check(aa.axis_attn_bwd_det(q, k, v, self.o.data_ptr(), do, self.lse.data_ptr(),
                                             self.dq.data_ptr(), self.dk.data_ptr(), self.dv.data_ptr(), B, Hq,
                                             Hkv, S, D, w.scale, c, ws, wsb, sp), "bwd_det")
            rec(4)
            return
        self._check(aa.axis_attn_bwd_prepare(self.o.data_ptr(), do, self.lse.data_ptr(), B, Hq, Hkv, S, D, w.scale,
                                             ws, wsb, sp), "bwd_prepare")
        rec(2)
        self._check(aa.axis_attn_bwd_main(q, k, v, do, self.dk.data_ptr(), self.dv.data_ptr(), B, Hq, Hkv, S, D,
                                          w.scale, c, ws, wsb, sp), "bwd_main")
        rec(3)
        self._check(aa.axis_attn_bwd_finalize(self.dq.data_ptr(), B, Hq, Hkv, S, D, ws, wsb, sp), "bwd_finalize")
        rec(4)


class L2Flush:
    """Evicts the L2 (126 MB on B200) between timed steps: `fill_` writes a
    256 MiB buffer, then reads another 256 MiB one.  A write alone leaves the
    L2 full of dirty lines, whose write-back to HBM then competes with the
    next timed kernel (measured: +8% on an HBM-bound decode step); after the
    read the L2 holds clean lines of the read buffer only."""

    def __init__(self, dev):
        import torch

        self.w = torch.empty(256 << 20, device=dev, dtype=torch.uint8)
        self.r = torch.ones(64 << 20, device=dev, dtype=torch.float32)

    def fill_(self, v):
        self.w.fill_(v)
        self.r.sum()


def time_steps(prob, steps: int, warmup: int, flush, world: int, dev, sampler):
    """W untimed steps, then K timed steps (events on the launching stream, L2
    flushed before each, outside the events), barrier + synchronize on both
    sides.  Returns (total ms max over ranks, per-stage ms totals max over
    ranks, wall-clock window)."""
    import torch
    import torch.distributed as dist

    for n in range(warmup):
        flush.fill_(1)
        prob.step()
        if n == 0:
            prob.aa.check_status(prob.stream)  # fail fast on a device-side timeout
    prob.aa.check_status(prob.stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    for s in range(steps):
        flush.fill_(s & 0xFF)
        prob.step(evs[s])
    torch.cuda.synchronize()
    t1 = time.time()
    if world > 1:
        dist.barrier()
    prob.aa.check_status(prob.stream)
    per = [[e[i].elapsed_time(e[i + 1]) for i in range(4)] for e in evs]
    stage_ms = [sum(p[i] for p in per) for i in range(4)]
    step_ms = sum(e[0].elapsed_time(e[4]) for e in evs)
    red = reduce_max([step_ms] + stage_ms, world, dev)
    return red[0], red[1:], (t0, t1)


def shard_problem(aa, w, seed: int, dev, det: bool, world: int, rank: int):
    """Head-sharded mode: this rank's (b, kv) units of ONE problem (every rank
    draws the same inputs), packed as a batch of units (B' = units, Hq' = G,
    Hkv' = 1).  Returns the Problem and the whole problem's FLOPs."""
    import dataclasses

    from causal_attention_fwd_b200 import shard
    from causal_attention_fwd_b200.synthetic import workload_inputs

    q, k, v, do = workload_inputs(w, seed=seed)
    G = w.Hq // w.Hkv
    units = shard.rank_units(w.B, w.Hkv, world, rank)
    host = (shard.pack(q, units, G), shard.pack(k, units, 1), shard.pack(v, units, 1), shard.pack(do, units, G))
    wl = dataclasses.replace(w, name=f"{w.name}[units {rank}/{world}]", B=len(units), Hq=G, Hkv=1)
    return Problem(aa, wl, seed, dev, det, host=host)


def time_rope(aa, w, seed, dev, steps, flush, p_meas):
    """The headline step with the rotary embedding fused (axis_attn_fwd_rope +
    axis_attn_bwd_rope): fwd / bwd TFLOP/s counting the same attention FLOPs
    (the rotations add no MMA work), device time per call with CUDA events."""
    import torch

    from causal_attention_fwd_b200.synthetic import workload_inputs

    q, k, v, do = (t.to(dev) for t in workload_inputs(w, seed=seed))
    B, Hq, Hkv, S, D = w.B, w.Hq, w.Hkv, w.S, w.D
    cs = aa.rope_table(S, D, 10000.0, device=dev)
    o, lse = torch.empty_like(q), torch.empty((B, Hq, S), device=dev, dtype=torch.float32)
    q_rot, k_rot = torch.empty_like(q), torch.empty_like(k)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsb = aa.axis_attn_bwd_workspace_bytes(B, Hq, Hkv, S, D)
    ws = torch.empty(wsb, device=dev, dtype=torch.uint8)
    st = torch.cuda.current_stream(dev)
    import ctypes

    sp = ctypes.c_void_p(st.cuda_stream)

    def fwd():
        rc = aa.axis_attn_fwd_rope(q.data_ptr(), k.data_ptr(), v.data_ptr(), cs.data_ptr(), o.data_ptr(),
                                   lse.data_ptr(), q_rot.data_ptr(), k_rot.data_ptr(), B, Hq, Hkv, S, D, w.scale,
                                   int(w.causal), sp)
        if rc:
            raise aa.AxisAttnError(rc, "axis_attn_fwd_rope")

    def bwd():
        rc = aa.axis_attn_bwd_rope(q_rot.data_ptr(), k_rot.data_ptr(), v.data_ptr(), cs.data_ptr(), o.data_ptr(),
                                   do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq,
                                   Hkv, S, D, w.scale, int(w.causal), 0, ws.data_ptr(), wsb, sp)
        if rc:
            raise aa.AxisAttnError(rc, "axis_attn_bwd_rope")

    ev = []
    for n in range(3 + steps):
        flush.fill_(n & 0xFF)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(st)
        fwd()
        e[1].record(st)
        bwd()
        e[2].record(st)
        if n >= 3:
            ev.append(e)
    torch.cuda.synchronize()
    aa.check_status(st)
    f_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / len(ev)
    b_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / len(ev)
    fwd_tf, bwd_tf = w.fwd_flops / f_ms / 1e9, w.bwd_flops / b_ms / 1e9
    return {"fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf, "fwd_ms": f_ms, "bwd_ms": b_ms, "steps": steps,
            "fwd_frac_of_measured": fwd_tf / p_meas, "bwd_frac_of_measured": bwd_tf / p_meas,
            "note": "fwd: Q and K rotated once by an HBM-bound prologue pass, then the forward kernel; bwd: the "
                    "transposed rotation fused into the dQ finalize and the dK epilogue; times include the "
                    "rotations"}


# Decode workloads: one new token per sequence against a paged KV cache of
# `ctx` tokens (the axiomlm model's heads and block size; an 8B-class model),
# each batched one on both pool layouts: NHD [num_pages, page_size, Hkv, D] and
# the head-major HND [num_pages, Hkv, page_size, D]; and one sequence of 32K
# tokens (batch 1: the split-K path and the merge kernel, latency-bound).
DECODE = {
    "decode_gpt2s_gqa": dict(B=256, Hq=12, Hkv=4, D=64, ctx=1024, page=16, layout="NHD"),
    "decode_gpt2s_gqa_hnd": dict(B=256, Hq=12, Hkv=4, D=64, ctx=1024, page=16, layout="HND"),
    "decode_llm8b_gqa": dict(B=32, Hq=32, Hkv=8, D=128, ctx=8192, page=64, layout="NHD"),
    "decode_llm8b_gqa_hnd": dict(B=32, Hq=32, Hkv=8, D=128, ctx=8192, page=64, layout="HND"),
    "decode_llm8b_b1_32k": dict(B=1, Hq=32, Hkv=8, D=128, ctx=32768, page=64, layout="NHD"),
    # 4 new tokens per sequence in one step (proposed tokens checked together)
    "decode_llm8b_gqa_q4": dict(B=32, Hq=32, Hkv=8, D=128, ctx=8192, page=64, layout="NHD", q_len=4),
}


def time_decode(aa, name, dev, steps, flush, hbm_gbs):
    """Decode step timing: HBM GB/s of the cache bytes every call must read
    (K and V of every cached token, plus q and o), against the measured copy
    bandwidth."""
    import torch

    c = DECODE[name]
    B, Hq, Hkv, D, ctx, page = c["B"], c["Hq"], c["Hkv"], c["D"], c["ctx"], c["page"]
    T = c.get("q_len", 1)  # new tokens per sequence
    g = torch.Generator().manual_seed(4000)
    max_pages = ctx // page
    num_pages = B * max_pages
    q = torch.randn((B, Hq, D) if T == 1 else (B, T, Hq, D), generator=g).to(torch.bfloat16).to(dev)
    kc = torch.randn((num_pages, page, Hkv, D), generator=g).to(torch.bfloat16).to(dev)
    vc = torch.randn((num_pages, page, Hkv, D), generator=g).to(torch.bfloat16).to(dev)
    hnd = c["layout"] == "HND"
    if hnd:
        kc, vc = kc.transpose(1, 2).contiguous(), vc.transpose(1, 2).contiguous()
    call = aa.axis_attn_decode_hnd if hnd else aa.axis_attn_decode
    if T > 1:
        call = aa.axis_attn_decode_q
    table = torch.randperm(num_pages, generator=g).to(torch.int32).reshape(B, max_pages).to(dev)
    lens = torch.full((B,), ctx, dtype=torch.int32, device=dev)
    o, lse = torch.empty_like(q), torch.empty((B, Hq, T), device=dev, dtype=torch.float32)
    need = (aa.axis_attn_decode_workspace_bytes(B, Hq, Hkv, D, page, max_pages) if T == 1
            else aa.axis_attn_decode_q_workspace_bytes(B, T, Hq, Hkv, D, page, max_pages))
    ws = torch.empty(max(need, 256), device=dev, dtype=torch.uint8)
    st = torch.cuda.current_stream(dev)
    import ctypes

    sp = ctypes.c_void_p(st.cuda_stream)
    # the C ABI straight (as the main step does): the torch helper's checks would run on the host
    # between the events while the GPU waits, and count as device time
    ptrs = (q.data_ptr(), kc.data_ptr(), vc.data_ptr(), table.data_ptr(), lens.data_ptr(), o.data_ptr(),
            lse.data_ptr())
    if T == 1:
        args = ptrs + (B, Hq, Hkv, D, page, max_pages, num_pages, 1.0 / math.sqrt(D), ws.data_ptr(), ws.numel(), sp)
    else:
        args = ptrs + (B, T, Hq, Hkv, D, page, max_pages, num_pages, 1.0 / math.sqrt(D), int(hnd), ws.data_ptr(),
                       ws.numel(), sp)
    ev = []
    for n in range(3 + steps):
        flush.fill_(n & 0xFF)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record(st)
        rc = call(*args)
        e[1].record(st)
        if rc:
            raise aa.AxisAttnError(rc, call.__name__)
        if n >= 3:
            ev.append(e)
    torch.cuda.synchronize()
    aa.check_status(st)
    ms = sum(e[0].elapsed_time(e[1]) for e in ev) / len(ev)
    nbytes = B * ctx * Hkv * D * 2 * 2 + 2 * B * T * Hq * D * 2
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"config": f"B={B} Hq={Hq} Hkv={Hkv} D={D} context={ctx} page_size={page} new_tokens={T} (bf16 paged "
                      f"cache, {c['layout']} pages, random page order)", "ms": ms, "steps": steps, "algorithmic_bytes": nbytes,
            "launches_per_call": 2 if need > 0 else 1,  # the decode kernel, and the split merge when it splits
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": gbs / hbm_gbs}}


def launches_per_step(aa, w) -> int:
    """Kernels of ours one step launches: the forward, the backward's
    preprocess, main kernel and dQ stage (finalize, or the deterministic dQ
    pass), and the partial dK/dV sum when the backward splits the heads."""
    return 4 + (aa.axis_attn_bwd_head_split(w.B, w.Hq, w.Hkv, w.S, w.D) > 1)


def time_e2e(aa, w, prob, steps: int, det: bool, world: int, dev) -> dict:
    """The step end to end through the public torch helpers, from pinned host
    buffers: every step copies its Q, K, V, dO host->device and its O, LSE,
    dQ, dK, dV device->host inside the timed region.  Three streams form a
    pipeline, as a training loop would run it: step i's inputs go up on the
    copy-in stream while step i-1 computes and step i-2's results come down on
    the copy-out stream (PCIe is full duplex).  Two device buffer sets
    alternate; events order each set's reuse.  Time: from an event before the
    first upload to one after the last download."""
    import torch

    pin = lambda t: t.pin_memory()  # noqa: E731
    q_h, k_h, v_h, do_h = prob.host
    hin = [pin(t) for t in (q_h, k_h, v_h, do_h)]
    hout = [torch.empty_like(hin[0]).pin_memory(),
            torch.empty((w.B, w.Hq, w.S), dtype=torch.float32).pin_memory()] + \
        [torch.empty_like(t).pin_memory() for t in hin[:3]]
    sets = []
    for _ in range(2):
        ins = [torch.empty_like(t) for t in (prob.q, prob.k, prob.v, prob.do)]
        outs = [torch.empty_like(prob.q), torch.empty_like(prob.lse), torch.empty_like(prob.q),
                torch.empty_like(prob.k), torch.empty_like(prob.v)]
        sets.append((ins, outs))
    s_in, s_out, s_comp = torch.cuda.Stream(dev), torch.cuda.Stream(dev), prob.stream
    mk = lambda: [torch.cuda.Event() for _ in range(2)]  # noqa: E731
    ev_in, ev_done, ev_out = mk(), mk(), mk()
    used = [False, False]

    def step(i):
        b = i % 2
        ins, outs = sets[b]
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(ev_done[b])  # the last compute on this set has read its inputs
            for dst, src in zip(ins, hin):
                dst.copy_(src, non_blocking=True)
            ev_in[b].record(s_in)
        s_comp.wait_event(ev_in[b])
        if used[b]:
            s_comp.wait_event(ev_out[b])  # its previous results are on the host
        o, lse = aa.attention_forward(ins[0], ins[1], ins[2], causal=w.causal, scale=w.scale, out=outs[0],
                                      lse=outs[1], stream=s_comp)
        aa.attention_backward(ins[0], ins[1], ins[2], o, lse, ins[3], causal=w.causal, scale=w.scale,
                              workspace=prob.ws, grads=tuple(outs[2:]), stream=s_comp, deterministic=det)
        ev_done[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            for dst, src in zip(hout, outs):
                dst.copy_(src, non_blocking=True)
            ev_out[b].record(s_out)
        used[b] = True

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    e0.record(s_in)
    for i in range(steps):
        step(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    ems = reduce_max([e0.elapsed_time(e1)], world, dev)
    aa.check_status(s_comp)
    # the results that came back to the host are the device step's own: O, LSE, dK, dV bit for bit
    # (the same inputs, deterministic kernels), dQ to rounding (its fp32 additions arrive in any order)
    dev_out = [prob.o, prob.lse, prob.dq, prob.dk, prob.dv]
    same = all(torch.equal(h, d.cpu()) for i, (h, d) in enumerate(zip(hout, dev_out)) if i != 2)
    dq_h, dq_d = hout[2].double(), dev_out[2].cpu().double()
    dq_rel = float((dq_h - dq_d).norm() / dq_d.norm().clamp_min(1e-30))
    h2d = sum(t.numel() * t.element_size() for t in hin)
    d2h = sum(t.numel() * t.element_size() for t in hout)
    return {"value": whole_job_tflops(w.fwd_flops + w.bwd_flops, steps, ems[0], world), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "streams": "copy-in / compute / copy-out, two buffer sets",
            "verified": bool(same and dq_rel <= 1e-3), "dq_rel_to_device_step": dq_rel}


def summarize(w, total_ms, stage_totals, steps, world, p_meas, det):
    """Per-workload figures: fwd / bwd TFLOP/s and fractions of the peaks."""
    avg = [float(t) / steps for t in stage_totals]
    fwd_tf = w.fwd_flops / (avg[0] * 1e-3) / 1e12
    bwd_ms = sum(avg[1:])
    bwd_tf = w.bwd_flops / (bwd_ms * 1e-3) / 1e12
    names = STAGES if not det else ["attn_fwd_kernel", "-", "-", "axis_attn_bwd_det (prep + main + dQ pass)"]
    return {
        "value": whole_job_tflops(w.fwd_flops + w.bwd_flops, steps, total_ms, world),
        "ms_per_step": total_ms / steps, "steps": steps,
        "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
        "fwd_frac_of_measured": fwd_tf / p_meas, "bwd_frac_of_measured": bwd_tf / p_meas,
        "fwd_frac_of_nominal_2250": fwd_tf / P_NOM_TFLOPS, "bwd_frac_of_nominal_2250": bwd_tf / P_NOM_TFLOPS,
        "kernel_ms": {n: t for n, t in zip(names, avg) if n != "-"},
    }, avg, names


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # 200 steps keep the timed region (~0.1 s at llm1b) long enough for ~20+ clock samples
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llm1b")
    ap.add_argument("--others", default="tiny,gpt2s_gqa,llm8b_gqa,longseq",
                    help="further workloads timed after the headline one (comma list; '' for none)")
    ap.add_argument("--other-steps", type=int, default=20)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--deterministic", action="store_true",
                    help="time the bitwise-reproducible backward (axis_attn_bwd_det) instead")
    ap.add_argument("--shard", action="store_true",
                    help="N > 1: split ONE problem's (b, kv) units over the ranks (strong scaling) instead of "
                         "one replica per rank")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist

    import causal_attention_fwd_b200 as aa
    from causal_attention_fwd_b200.synthetic import WORKLOAD_SEED, WORKLOADS

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    det = args.deterministic
    pk, pk_src = peaks()
    p_meas = pk["bf16_tflops"]
    flush = L2Flush(dev)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.05)

    # ---- the headline workload
    w = WORKLOADS[args.workload]
    sharded = args.shard and world > 1
    if sharded:  # one problem, its units over the ranks; kernels time this rank's share
        prob = shard_problem(aa, w, WORKLOAD_SEED[w.name], dev, det, world, rank)
    else:
        prob = Problem(aa, w, rank_seed(WORKLOAD_SEED[w.name], rank), dev, det)
    K = args.steps
    total_ms, totals, win = time_steps(prob, K, args.warmup, flush, world, dev, sampler)
    head, avg_ms, names = summarize(prob.w, total_ms, totals, K, world, p_meas, det)
    if sharded:  # whole-job throughput: the one problem's FLOPs over the slowest rank's time
        head["value"] = (w.fwd_flops + w.bwd_flops) * K / (total_ms * 1e-3) / 1e12
    value = head["value"]

    # dominant kernel and its roofline
    dom = max(range(4), key=lambda i: avg_ms[i])
    dom_flops = prob.w.fwd_flops if dom == 0 else prob.w.bwd_flops
    roof = None
    if dom in (0, 2) or (det and dom == 3):
        achieved = dom_flops / (avg_ms[dom] * 1e-3) / 1e12
        roof = {"kernel": names[dom], "bound": "tensor", "achieved": achieved, "peak": p_meas,
                "peak_source": f"{pk_src} bf16_tflops (burst)", "unit": "TFLOP/s",
                "frac": achieved / p_meas, "frac_of_nominal_2250": achieved / P_NOM_TFLOPS,
                "traffic": profiled_traffic(names[dom], w.name),
                "flops_per_launch": dom_flops, "avg_launch_ms": avg_ms[dom]}

    # ---- end to end through the public API, host buffers, copies inside the timed region
    e2e = None
    if args.e2e_steps > 0 and not sharded:
        e2e = time_e2e(aa, w, prob, args.e2e_steps, det, world, dev)
    clocks = sampler.summary(*win)
    del prob
    torch.cuda.empty_cache()

    # ---- the other workloads: the same step, timed the same way, fewer steps
    others = {}
    for name in [n for n in args.others.split(",") if n and n != w.name and not sharded]:
        wo = WORKLOADS[name]
        po = Problem(aa, wo, rank_seed(WORKLOAD_SEED[wo.name], rank), dev, det)
        ko = max(3, args.other_steps // 2) if wo.S >= 16384 else args.other_steps
        t_ms, tot, wwin = time_steps(po, ko, 3, flush, world, dev, sampler)
        summ, _, _ = summarize(wo, t_ms, tot, ko, world, p_meas, det)
        summ["config"] = wo.describe()
        summ["clocks"] = sampler.summary(*wwin)
        others[name] = summ
        summ["gpu_launches"] = launches_per_step(aa, wo) * ko
        hs = aa.axis_attn_bwd_head_split(wo.B, wo.Hq, wo.Hkv, wo.S, wo.D)
        if hs > 1:  # the main-kernel stage then also holds the partial dK/dV sum
            summ["bwd_head_split"] = hs
        del po
        torch.cuda.empty_cache()
    # ---- the headline workload with RoPE fused, and the decode step
    rope = None
    decode = {}
    if not sharded and not det:
        rope = time_rope(aa, w, rank_seed(WORKLOAD_SEED[w.name], rank), dev, args.other_steps, flush, p_meas)
        torch.cuda.empty_cache()
        for name in DECODE:
            decode[name] = time_decode(aa, name, dev, args.other_steps, flush, pk["hbm_gbs"])
            torch.cuda.empty_cache()
    sampler.stop()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        tf, cores, desc, t = cpu_sample(w, args.cpu_budget)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}
        for name, summ in others.items():
            tf, cores, desc, t = cpu_sample(WORKLOADS[name], args.cpu_budget)
            summ["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                    "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
            "scaling": "strong" if sharded else "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,sigma^2), bf16-rounded; " + (
                "one problem, its (b, kv) units dealt round robin over the ranks)" if sharded else
                "each rank its own batch)"),
            "config": dict(workload_config(w, world), **({"parallelism": f"head-sharded units x{world} "
                                                          "(no collective)"} if sharded else {})),
            **{k: head[k] for k in ("fwd_tflops", "bwd_tflops", "fwd_frac_of_nominal_2250",
                                    "bwd_frac_of_nominal_2250", "fwd_frac_of_measured", "bwd_frac_of_measured",
                                    "kernel_ms")},
            "bwd_mode": "deterministic (axis_attn_bwd_det)" if det else "ordinary (axis_attn_bwd stages)",
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches_per_step(aa, w) * K, "clocks": clocks,
            "workloads": others, "rope": rope, "decode": decode,
        }
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
