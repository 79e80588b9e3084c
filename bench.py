"""Benchmark of the ring-attention hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (one "step"): the long causal zigzag workload -- B=1, 16 query heads
/ 8 KV heads, d=128, N=262144 bf16 tokens, P=8 virtual ranks in the zigzag
(load-balanced) layout, forward + backward, plus the Ulysses seq->head repack
of Q and of the fused K|V ([8 x 32768, 16, 128] -> [8 x 262144, 2, 128], one
call each):
  repack Q, repack K|V, fused ring forward -> ring backward (delta
  preprocess, key-stationary dK/dV kernel, query-stationary dQ kernel), on
  operands in their global token order: each virtual rank's tiles are fetched
  through the zigzag layout by the kernels' TMA coordinates and O, LSE, dQ,
  dK, dV are written back in global order, so the step has no separate
  permute pass (the permute kernel itself is timed in the extras).  K and V
  are two head views of one fused [1, N, 16, 128] buffer.
Inputs are seeded synthetic tensors already resident in HBM; L2 (126 MB) is
flushed between timed steps.  ``value`` is algorithmic TFLOP/s summed over all
ranks: forward 4*d and backward 10*d flops per visible (query, key) pair,
causal pairs only (the repack adds time, no flops).  With --gpus N every rank
runs an independent replica of the workload (the path has no data exchange on
one GPU), so scaling is weak.

``roofline`` is the step's dominant kernel against the bf16 tensor peak: the
burst figure, or the sustained one when the timed region ran for seconds in
the power-capped regime its clock record shows.

``e2e`` is the same step through the same public calls with the inputs copied
in from pinned host memory and every result (O, LSE, dQ, dK, dV and the two
repacked tensors) copied back, each step, pipelined over two device buffer
slots and three streams.

Extra measurements on the same line: fwd+bwd of the causal striped 128k and
the Llama-like zigzag 16k workloads; the LSE merge (8 partials per rank of
the striped 128k shapes, and the two-part in-place merge), the Ulysses repack
(the 256k shapes), the striped layout permute (the 128k Q shape) and the
tabular feature-axis attention in GB/s against HBM (device time of their own
kernels); the tabular row-axis attention (d = 24) against the tensor peak and
the exp unit; USP (Ulysses x ring) and Mesh2D fwd+bwd.  ``--case <group>
[--small]`` runs one group of these alone (for a profiler run).

``--impl reference`` times the CPU fp64 oracle instead, on a bounded sample of
the same workload (the last --ref-sample-queries queries of query head 0,
forward and backward against every key they see), and prints the same metric
with "impl": "reference"; under torchrun only rank 0 runs it.  ``cpu_baseline``
times the same sample.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sequence_attention_rm_b200 import synthetic  # noqa: E402

METRIC = "ring-attn fwd+bwd TFLOP/s and % of BF16 peak at 1 B200; merge GB/s % HBM"
HEADLINE = synthetic.LONG_ZIGZAG_256K
HEADLINE_NAME = ("long-causal-zigzag-256k: B=1 Hq=16 Hkv=8 d=128 N=262144 bf16 P=8 zigzag causal "
                 "fwd+bwd + seq->head repack of Q and fused K|V [8 x 32768, 16, 128] -> "
                 "[8 x 262144, 2, 128]")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def causal_pairs(w) -> int:
    per_head = w.N * (w.N + 1) // 2 if w.causal else w.N * w.N
    return per_head * w.Hq * w.B


def flops_fwd(w) -> float:
    return 4.0 * w.d * causal_pairs(w)


def flops_bwd(w) -> float:
    return 10.0 * w.d * causal_pairs(w)


# ---------------------------------------------------------------------------
# distributed plumbing (independent replicas; barrier + max-over-ranks timing)
# ---------------------------------------------------------------------------
def dist_init(backend: str = "nccl"):
    """One process per GPU from the torchrun environment.  The benchmark uses
    NCCL; the CPU tests of this plumbing use gloo (no device is touched)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend == "nccl":
        torch.cuda.set_device(local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest x over all ranks (the slowest rank's time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Units all ranks processed over the slowest rank's time, per second:
    every rank runs the same replica, so the job did world * steps steps in
    max_ms."""
    return units_per_rank_step * steps * world / (max_ms * 1e-3)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz, mx, pw = float(parts[1]), float(parts[2]), float(parts[3])
            except ValueError:
                continue
            smax = mx
            if pw > 300.0:  # under load
                sm.append(mhz)
            for name, flag in zip(names, parts[5:9]):
                if flag.lower() == "active":
                    reasons.add(name)
        if not sm:  # short runs: fall back to every sample
            for line in getattr(self, "lines", []):
                parts = [p.strip() for p in line.split(",")]
                try:
                    sm.append(float(parts[1]))
                except (ValueError, IndexError):
                    pass
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(getattr(self, "lines", []))}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
class Step:
    """Pre-allocated buffers and one hot-path step of a workload, on operands
    in their global token order: the Ulysses seq->head repack of Q and of the
    fused K|V, the fused ring forward and the ring backward.

    K and V live in one fused buffer [B, N, 2 Hkv, d] (the Hkv K heads, then
    the Hkv V heads of every token); the ring reads them as two strided head
    views, and the repack moves the buffer as 2 Hkv heads, so that the K/V
    exchange is one all-to-all (ringmaster "Status": the Ulysses leg fuses
    K/V).  The repack treats the global-order tensors as P contiguous
    sequence shards [P, N / P, H, d] and writes head-sharded [P, N, H / P, d]
    tensors, each rank's heads over the whole sequence in global order."""

    def __init__(self, rm, w, q, kv, do, repack=True):
        self.rm, self.w = rm, w
        self.q, self.kv, self.do = q, kv, do
        self.k, self.v = kv[:, :, :w.Hkv], kv[:, :, w.Hkv:]
        e = lambda t: torch.empty_like(t)
        self.o, self.dq = e(q), e(q)
        self.dk = torch.empty(q.shape[:2] + (w.Hkv, w.d), dtype=q.dtype, device=q.device)
        self.dv = torch.empty_like(self.dk)
        self.lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=q.device)
        dsc = rm.desc(w.dtype, w.B, w.Hq, w.Hkv, w.d, w.N, w.P, w.layout, w.causal,
                      order="global")
        self.ws = torch.empty(max(rm.ring_workspace_size(dsc, True), 256), dtype=torch.uint8,
                              device=q.device)
        self.repack = repack and w.B == 1
        if self.repack:
            P, L = w.P, w.N // w.P
            self.q_shards = q.view(P, L, w.Hq, w.d)
            self.kv_shards = kv.view(P, L, 2 * w.Hkv, w.d)
            self.qh = torch.empty((P, w.N, w.Hq // P, w.d), dtype=q.dtype, device=q.device)
            self.kvh = torch.empty((P, w.N, 2 * w.Hkv // P, w.d), dtype=q.dtype, device=q.device)
        # repack Q, repack K|V; forward; delta, dK/dV, dQ
        self.launches_per_step = (2 if self.repack else 0) + 1 + 3

    def outputs(self):
        out = [self.o, self.lse, self.dq, self.dk, self.dv]
        return out + ([self.qh, self.kvh] if self.repack else [])

    def repack_bytes(self) -> int:
        if not self.repack:
            return 0
        return 2 * (self.q.numel() + self.kv.numel()) * self.q.element_size()

    def run(self, ev=None):
        rm, w = self.rm, self.w
        lay, P = w.layout, w.P
        if ev:
            ev[0].record()
        if self.repack:
            rm.seq_head_repack(self.q_shards, P, out=self.qh)
            rm.seq_head_repack(self.kv_shards, P, out=self.kvh)
        if ev:
            ev[1].record()
        rm.ring_attn_fwd(self.q, self.k, self.v, P=P, layout=lay, causal=w.causal,
                         order="global", out=self.o, lse=self.lse)
        if ev:
            ev[2].record()
        rm.ring_attn_bwd(self.q, self.k, self.v, self.o, self.lse, self.do, P=P, layout=lay,
                         causal=w.causal, order="global", dq=self.dq, dk=self.dk, dv=self.dv,
                         ws=self.ws)
        if ev:
            ev[3].record()


def fused_kv(k, v):
    """[B, N, Hkv, d] K and V -> one [B, N, 2 Hkv, d] buffer (K heads first)."""
    return torch.cat([k, v], dim=2).contiguous()


# Algorithmic flops per launch of each attention kernel, per visible (query,
# key) pair: the contractions the kernel performs for its outputs.
FLOPS_PER_PAIR = {"tc_fwd_kernel": 4, "tc_bwd_dkdv_kernel": 8, "tc_bwd_dq_kernel": 6}
# dram__bytes_read.sum + dram__bytes_write.sum per launch of each kernel on
# the headline workload (one-pass ncu capture of the current kernels at full
# size, profiles/launch_list_long_zigzag_256k.md).
TRAFFIC = {"tc_fwd_kernel": 8_362_033_920, "tc_bwd_dkdv_kernel": 18_578_496_512,
           "tc_bwd_dq_kernel": 15_350_899_456}


def kernel_table(records, steps, step_ms, w):
    agg = {}
    for name, ms in records:
        a = agg.setdefault(name, [0, 0.0])
        a[0] += 1
        a[1] += ms
    out = {}
    for name, (n, tot) in agg.items():
        ms = tot / n
        e = {"launches_per_step": round(n / steps, 2), "ms": round(ms, 4),
             "share": round(tot / steps / step_ms, 4)}
        if name in FLOPS_PER_PAIR:
            flops = FLOPS_PER_PAIR[name] * w.d * causal_pairs(w)
            e["flops"] = flops
            e["TFLOP/s"] = round(flops / (ms * 1e-3) / 1e12, 2)
        out[name] = e
    return out


def flush_l2(buf):
    buf.zero_()


def time_events(pairs):
    return [a.elapsed_time(b) for a, b in pairs]


def tensor_peak(peaks, peak_src, timed_s, clocks):
    """The bf16 peak a tensor-core kernel is measured against: the burst figure
    (a short region at full clocks), unless the timed region lasted seconds
    and its clock record shows the power-capped regime in which the
    sustained figure was measured (SM clock at most 85% of its maximum under
    load, with sw_power_cap active)."""
    burst = peaks["bf16_tflops"]
    sustained = peaks.get("bf16_tflops_sustained", burst)
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = (timed_s >= 2.0 and mhz is not None and mx
              and mhz <= 0.85 * mx and "sw_power_cap" in clocks.get("reasons", []))
    if capped:
        return sustained, (f"{peak_src} bf16_tflops_sustained: the timed region ran {timed_s:.1f} s "
                           f"at a median {mhz:.0f} of {mx:.0f} MHz under sw_power_cap")
    return burst, f"{peak_src} bf16_tflops (burst)"


def bench_ours(args, world, rank, local):
    from sequence_attention_rm_b200 import rm

    peaks, peak_src = load_peaks()
    w = HEADLINE
    dev = torch.device("cuda", local)
    q_h, k_h, v_h, do_h = synthetic.attention_inputs(w)
    kv_h = fused_kv(k_h, v_h)
    del k_h, v_h
    q, kv, do = (t.to(dev) for t in (q_h, kv_h, do_h))
    step = Step(rm, w, q, kv, do)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    rm.profile_enable(True)  # per-launch CUDA events on the launching stream
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush_l2(flush)
            step.run(evs[i])
        torch.cuda.synchronize()
    barrier(world)
    records = rm.profile_records()
    rm.profile_enable(False)
    per = [time_events([(e[0], e[3]), (e[0], e[1]), (e[1], e[2]), (e[2], e[3])]) for e in evs]
    step_ms = sum(p[0] for p in per)
    repack_ms = statistics.mean(p[1] for p in per)
    fwd_ms = statistics.mean(p[2] for p in per)
    bwd_ms = statistics.mean(p[3] for p in per)
    step_ms_max = max_over_ranks(step_ms, world)
    step_flops = flops_fwd(w) + flops_bwd(w)
    value = whole_job_rate(step_flops, args.steps, world, step_ms_max) / 1e12
    kernels = kernel_table(records, args.steps, step_ms / args.steps, w)
    clocks = clk.summary()

    # end-to-end: pinned host inputs in, every result back to pinned host
    # buffers, every step.  Two device slots and three streams: step i+1's
    # inputs are copied in and step i-1's results copied out while step i
    # computes.
    pin = lambda t: t.pin_memory()
    hq, hkv, hdo = pin(q_h), pin(kv_h), pin(do_h)
    del q_h, kv_h, do_h
    slots = [step, Step(rm, w, *(torch.empty_like(t) for t in (q, kv, do)))]
    # one set of host result buffers: the device->host copies of successive
    # steps run in order on one stream, so each step's results overwrite the
    # previous ones (8 GiB of pinned host memory in all, inputs included)
    host_out = [pin(torch.empty(t.shape, dtype=t.dtype)) for t in step.outputs()]
    h2d = sum(t.numel() * t.element_size() for t in (hq, hkv, hdo))
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    done_in, done_run, done_out = ([ev(), ev()] for _ in range(3))

    def e2e_step(i):
        j = i % 2
        sl = slots[j]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(done_run[j])  # slot j's inputs free again
            for src, dst in ((hq, sl.q), (hkv, sl.kv), (hdo, sl.do)):
                dst.copy_(src, non_blocking=True)
            done_in[j].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(done_in[j])
            if i >= 2:
                s_run.wait_event(done_out[j])  # slot j's results copied out
            sl.run()
            done_run[j].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done_run[j])
            for src, dst in zip(sl.outputs(), host_out):
                dst.copy_(src, non_blocking=True)
            done_out[j].record(s_out)

    for i in range(max(1, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(args.steps):
        e2e_step(i)
    # the last results are on the host once s_out is done; it waited on
    # everything before it
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = whole_job_rate(step_flops, args.steps, world, e2e_ms) / 1e12

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms_max / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": HEADLINE_NAME,
                   "global_batch": w.B * world, "seq_len": w.N,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "flushed between steps (256 MiB write); inputs 3 GiB > L2"},
    }
    peak, peak_note = tensor_peak(peaks, peak_src, step_ms / 1e3, clocks)
    # the dominant tensor-core kernel of the step
    top = max((k for k in kernels if "TFLOP/s" in kernels[k]), key=lambda k: kernels[k]["share"])
    tk = kernels[top]
    line["roofline"] = {
        "bound": "tensor", "kernel": top, "achieved": tk["TFLOP/s"], "peak": peak,
        "unit": "TFLOP/s", "frac": round(tk["TFLOP/s"] / peak, 4), "peak_source": peak_note,
        "traffic": TRAFFIC.get(top),
        "frac_of_burst": round(tk["TFLOP/s"] / peaks["bf16_tflops"], 4),
        "frac_of_sustained": round(tk["TFLOP/s"] / peaks.get("bf16_tflops_sustained",
                                                             peaks["bf16_tflops"]), 4),
        "flops_per_launch": tk["flops"], "ms_per_launch": tk["ms"],
    }
    line["kernels"] = kernels
    line["calls_ms"] = {"repack_q_kv": round(repack_ms, 4), "ring_fwd": round(fwd_ms, 4),
                        "ring_bwd": round(bwd_ms, 4)}
    line["ring_fwd_tflops"] = round(flops_fwd(w) / (fwd_ms * 1e-3) / 1e12, 2)
    line["ring_bwd_tflops"] = round(flops_bwd(w) / (bwd_ms * 1e-3) / 1e12, 2)
    rb = step.repack_bytes()
    line["repack_gbs"] = round(rb / repack_ms / 1e6, 1)
    line["e2e"] = {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                   "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms / args.steps, 4),
                   "pipeline": "2 device slots; host->device copy, step and device->host copy "
                               "on 3 streams (step i+1 in, step i-1 out during step i)"}
    line["gpu_launches"] = len(records)
    line["clocks"] = clocks
    del step, slots, q, kv, do, host_out, hq, hkv, hdo
    torch.cuda.empty_cache()

    if not args.no_extras:
        line["extras"] = extras(rm, peaks, peak_src, dev, flush)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.ref_sample_queries)
    return line


_RECORDS = []  # per-launch (name, ms) of the last _time(..., keep=True) call


def _time(fn, reps, flush, rm=None, keep=False):
    """Median device time of fn() in ms.  A short spin kernel runs before the
    start event, so the host has queued fn's launches before the GPU reaches
    them and the interval holds no host time.  With `rm`, the median of the
    summed per-launch event times the library records around its own kernels
    is returned too: (kernels, call) (the kernels alone, no gaps between
    launches); with `keep` the per-launch records are left in _RECORDS."""
    ts, ks = [], []
    if keep:
        _RECORDS.clear()
    for _ in range(reps):
        if flush is not None:
            flush_l2(flush)
        if _spin is not None:  # keep the GPU busy while the host queues fn
            _spin(SPIN_CYCLES)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if rm is not None:
            rm.profile_enable(True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        if rm is not None:
            recs = rm.profile_records()
            ks.append(sum(ms for _, ms in recs))
            if keep:
                _RECORDS.extend(recs)
            rm.profile_enable(False)
        ts.append(a.elapsed_time(b))
    if rm is None:
        return statistics.median(ts)
    return statistics.median(ks), statistics.median(ts)


# about 1 ms of spinning at the B200's clocks: longer than the host needs to
# queue any call timed here.  torch's spin kernel is a private helper; without
# it the call times include host time, the kernels' own event times do not.
SPIN_CYCLES = 2_000_000
_spin = getattr(torch.cuda, "_sleep", None)


def hbm_row(rm, fn, reps, flush, nbytes, hbm, peak_src, shape):
    """An HBM-bound call: algorithmic bytes over the device time of its
    kernels (the library's per-launch events), the whole call beside it."""
    fn()
    ms, call_ms = _time(fn, reps, flush, rm)
    return {"shape": shape, "ms": round(ms, 4), "call_ms": round(call_ms, 4),
            "GB/s": round(nbytes / ms / 1e6, 1), "frac": round(nbytes / ms / 1e6 / hbm, 4),
            "peak": hbm, "peak_source": f"{peak_src} hbm_gbs", "bytes": nbytes,
            "timing": "kernel device time (per-launch CUDA events)"}


def extras(rm, peaks, peak_src, dev, flush, only=None, small=False):
    """The extra measurements, by group; `only` runs one group (for a
    profiler run of one kernel family on its own workload).  `small` shrinks
    the merge, repack and permute shapes (token counts / 8, / 8 and / 2; still
    larger than L2) so that a multi-pass profiler capture holds at most about
    1 GB on the device; their lines then name the smaller shapes."""
    hbm = peaks["hbm_gbs"]
    groups = {
        "merge": lambda: merge_lines(rm, dev, flush, hbm, peak_src, 8 if small else 1),
        "repack": lambda: repack_line(rm, dev, flush, hbm, peak_src, 8 if small else 1),
        "striped_128k": lambda: striped_lines(rm, dev, flush, peaks, hbm, peak_src, small),
        "llama_16k": lambda: llama_16k_line(rm, flush, peaks, peak_src),
        "tabular_row": lambda: {"tabular_row_fwd": tabular(rm, flush, hbm, peak_src, "row")},
        "tabular_feature": lambda: {"tabular_feature_fwd": tabular(rm, flush, hbm, peak_src,
                                                                   "feature")},
        "usp": lambda: {"usp_16k_fwd_bwd": usp_line(rm, flush, peaks, peak_src)},
        "mesh2d": lambda: {"mesh2d_128k_fwd_bwd": mesh2d_line(rm, flush, peaks, peak_src)},
    }
    out = {}
    for name, fn in groups.items():
        if only is None or name == only:
            out.update(fn())
            torch.cuda.empty_cache()
    return out


EXTRA_GROUPS = ("merge", "repack", "striped_128k", "llama_16k", "tabular_row", "tabular_feature",
                "usp", "mesh2d")


def merge_lines(rm, dev, flush, hbm, peak_src, div=1):
    out = {}
    # LSE merge, striped-128k shapes: per rank 8 fp32 partials [16384, 16, 128] + LSE, 8 ranks
    Lr, H, d, P = 16384 // div, 16, 128, 8
    n = P * Lr
    o_parts = [torch.randn(1, P * Lr, H, d, device=dev) for _ in range(P)]
    lse_parts = [torch.randn(1, H, P * Lr, device=dev) for _ in range(P)]
    o_out = torch.empty(1, P * Lr, H, d, dtype=torch.bfloat16, device=dev)
    lse_out = torch.empty(1, H, P * Lr, device=dev)
    fn = lambda: rm.lse_merge(o_parts, lse_parts, torch.bfloat16, out=o_out, lse_out=lse_out)
    nbytes = P * (P * Lr * H * d * 4 + H * P * Lr * 4) + P * Lr * H * d * 2 + H * P * Lr * 4
    out["lse_merge"] = hbm_row(rm, fn, 10, flush, nbytes, hbm, peak_src,
                               f"8 partials x [1, {n}, 16, 128] fp32 -> bf16")
    # pairwise merge (the running-state form): fp32 O_acc <- merge(O_acc, O_new), in place
    acc, lacc = o_parts[0], lse_parts[0]
    fn = lambda: rm.lse_merge([acc, o_parts[1]], [lacc, lse_parts[1]], torch.float32, out=acc,
                              lse_out=lacc)
    nbytes = 3 * P * Lr * H * d * 4 + 3 * H * P * Lr * 4
    out["lse_merge_pairwise"] = hbm_row(rm, fn, 10, flush, nbytes, hbm, peak_src,
                                        f"2 partials x [1, {n}, 16, 128] fp32 -> fp32 in place")
    return out


def repack_line(rm, dev, flush, hbm, peak_src, div=1):
    # Ulysses repack, 256k-zigzag shapes: Q [8 x 32768, 16, 128] and the fused K|V (8 K heads
    # then 8 V heads) of the same shape, seq -> head, one call each
    Ln = 32768 // div
    x = torch.randn(8, Ln, 16, 128, device=dev).to(torch.bfloat16)
    kv = torch.randn(8, Ln, 16, 128, device=dev).to(torch.bfloat16)
    y = torch.empty(8, 8 * Ln, 2, 128, dtype=torch.bfloat16, device=dev)
    y2 = torch.empty_like(y)
    fn = lambda: (rm.seq_head_repack(x, 8, out=y), rm.seq_head_repack(kv, 8, out=y2))
    nbytes = 2 * (x.numel() + kv.numel()) * 2
    return {"repack": hbm_row(rm, fn, 10, flush, nbytes, hbm, peak_src,
                              f"seq->head Q and fused K|V, each [8, {Ln}, 16, 128] -> "
                              f"[8, {8 * Ln}, 2, 128] bf16")}


def step_line(rm, w, flush, peaks, peak_src, reps):
    """fwd+bwd of workload w (fused ring forward + ring backward on
    global-order operands, as in the headline step, without the repack):
    per-call times, TFLOP/s and the kernels' per-launch rates.  Burst peak:
    each timed call lasts well under a second."""
    q_h, k_h, v_h, do_h = synthetic.attention_inputs(w)
    dev = torch.device("cuda")
    q, kv, do = q_h.to(dev), fused_kv(k_h, v_h).to(dev), do_h.to(dev)
    del q_h, k_h, v_h, do_h
    st = Step(rm, w, q, kv, do, repack=False)
    fwd = lambda: rm.ring_attn_fwd(st.q, st.k, st.v, P=w.P, layout=w.layout, causal=w.causal,
                                   order="global", out=st.o, lse=st.lse)
    bwd = lambda: rm.ring_attn_bwd(st.q, st.k, st.v, st.o, st.lse, st.do, P=w.P, layout=w.layout,
                                   causal=w.causal, order="global", dq=st.dq, dk=st.dk, dv=st.dv,
                                   ws=st.ws)
    fwd()
    bwd()
    _, ms_f = _time(fwd, reps, flush, rm, keep=True)
    recs = list(_RECORDS)
    _, ms_b = _time(bwd, reps, flush, rm, keep=True)
    recs += _RECORDS
    burst = peaks["bf16_tflops"]
    tf_f = flops_fwd(w) / (ms_f * 1e-3) / 1e12
    tf_b = flops_bwd(w) / (ms_b * 1e-3) / 1e12
    tf = (flops_fwd(w) + flops_bwd(w)) / ((ms_f + ms_b) * 1e-3) / 1e12
    kern = {}
    for name, ms in recs:
        kern.setdefault(name, []).append(ms)
    kernels = {}
    for name, v in kern.items():
        e = {"ms": round(statistics.median(v), 4)}
        if name in FLOPS_PER_PAIR:
            e["TFLOP/s"] = round(FLOPS_PER_PAIR[name] * w.d * causal_pairs(w)
                                 / (statistics.median(v) * 1e-3) / 1e12, 2)
            e["frac"] = round(e["TFLOP/s"] / burst, 4)
        kernels[name] = e
    del st, q, kv, do
    return {"workload": f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} d={w.d} N={w.N} P={w.P} "
                        f"{w.layout} causal fwd+bwd", "fwd_ms": round(ms_f, 3),
            "bwd_ms": round(ms_b, 3), "fwd_TFLOP/s": round(tf_f, 2), "bwd_TFLOP/s": round(tf_b, 2),
            "TFLOP/s": round(tf, 2), "frac": round(tf / burst, 4), "fwd_frac": round(tf_f / burst, 4),
            "peak": burst, "peak_source": f"{peak_src} bf16_tflops (burst: calls of under a second)",
            "kernels": kernels}


def striped_lines(rm, dev, flush, peaks, hbm, peak_src, small=False):
    out = {}
    w3 = synthetic.STRIPED_128K
    if small:  # the permute alone, on half the tokens
        q = torch.randn(1, w3.N // 2, w3.Hq, w3.d, device=dev).to(torch.bfloat16)
        o2 = torch.empty_like(q)
        fn = lambda: rm.layout_permute(q, "striped", 8, out=o2)
        out["permute"] = hbm_row(rm, fn, 10, flush, 2 * q.numel() * 2, hbm, peak_src,
                                 f"striped P=8 [1, {w3.N // 2}, 16, 128] bf16")
        return out
    # the causal striped 128k workload, fwd+bwd (the forward alone is its gate)
    out["striped_128k_fwd_bwd"] = step_line(rm, w3, flush, peaks, peak_src, 3)
    torch.cuda.empty_cache()
    # layout permute of the striped 128k Q (global -> rank-major), 2 x 512 MiB
    q = torch.randn(1, w3.N, w3.Hq, w3.d, device=dev).to(torch.bfloat16)
    o2 = torch.empty_like(q)
    fn = lambda: rm.layout_permute(q, "striped", 8, out=o2)
    nbytes = 2 * q.numel() * 2
    out["permute"] = hbm_row(rm, fn, 10, flush, nbytes, hbm, peak_src,
                             "striped P=8 [1, 131072, 16, 128] bf16")
    return out


def llama_16k_line(rm, flush, peaks, peak_src):
    return {"llama_16k_fwd_bwd": step_line(rm, synthetic.LLAMA_ZIGZAG, flush, peaks, peak_src, 10)}


def mesh2d_line(rm, flush, peaks, peak_src):
    """Mesh2D on the causal 128k shapes (B=1, Hq=16, Hkv=8, d=128, N=131072,
    bf16): an 8 x 8 grid of (query chunk, key chunk) tiles of 16384 tokens,
    tiles past the diagonal skipped, partials merged per query chunk."""
    w = synthetic.STRIPED_128K
    g = 8
    q, k, v = (torch.randn(1, w.N, h, w.d, device="cuda").mul_(0.5).to(torch.bfloat16)
               for h in (w.Hq, w.Hkv, w.Hkv))
    do = torch.randn(1, w.N, w.Hq, w.d, device="cuda").to(torch.bfloat16)
    o = torch.empty_like(q)
    lse = torch.empty(1, w.Hq, w.N, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dsc = rm.desc(w.dtype, 1, w.Hq, w.Hkv, w.d, w.N, g, "contiguous", True)
    wsf = torch.empty(rm.mesh2d_workspace_size(dsc, g, g, False), dtype=torch.uint8, device="cuda")
    wsb = torch.empty(rm.mesh2d_workspace_size(dsc, g, g, True), dtype=torch.uint8, device="cuda")
    fwd = lambda: rm.mesh2d_attn_fwd(q, k, v, grid_q=g, grid_k=g, causal=True, out=o, lse=lse,
                                     ws=wsf)
    bwd = lambda: rm.mesh2d_attn_bwd(q, k, v, o, lse, do, grid_q=g, grid_k=g, causal=True, dq=dq,
                                     dk=dk, dv=dv, ws=wsb)
    fwd()
    bwd()
    ms_f = _time(fwd, 3, flush)
    ms_b = _time(bwd, 3, flush)
    tf_f = flops_fwd(w) / (ms_f * 1e-3) / 1e12
    tf = (flops_fwd(w) + flops_bwd(w)) / ((ms_f + ms_b) * 1e-3) / 1e12
    return {"grid": f"{g} x {g} (36 live tiles)", "fwd_ms": round(ms_f, 3), "bwd_ms": round(ms_b, 3),
            "fwd_TFLOP/s": round(tf_f, 2), "TFLOP/s": round(tf, 2),
            "frac": round(tf / peaks["bf16_tflops"], 4),
            "peak_source": f"{peak_src} bf16_tflops (burst: calls of under a second)",
            "note": "fwd: 36 tile launches + 8 merges; bwd: delta, 2 x 36 tile launches (fp32 "
                    "accumulators), 3 converts"}


def usp_line(rm, flush, peaks, peak_src):
    """USP fwd+bwd on the Llama-like 16k workload for a world of 16 virtual
    devices: the selector gives Ulysses 8 x ring 2 (zigzag), global order."""
    w = synthetic.LLAMA_ZIGZAG
    u, p_ring = rm.usp_auto_select(w.Hq, w.Hkv, 16)
    q, k, v, do = (t.cuda() for t in synthetic.attention_inputs(w))
    o = torch.empty_like(q)
    lse = torch.empty(w.B, w.Hq, w.N, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dsc = rm.desc(w.dtype, w.B, w.Hq, w.Hkv, w.d, w.N, p_ring, w.layout, True, order="global")
    wsf = torch.empty(max(rm.usp_workspace_size(dsc, u, False), 256), dtype=torch.uint8,
                      device="cuda")
    wsb = torch.empty(max(rm.usp_workspace_size(dsc, u, True), 256), dtype=torch.uint8,
                      device="cuda")

    def fn():
        rm.usp_attn_fwd(q, k, v, P=p_ring, ulysses=u, layout=w.layout, causal=True,
                        order="global", out=o, lse=lse, ws=wsf)
        rm.usp_attn_bwd(q, k, v, o, lse, do, P=p_ring, ulysses=u, layout=w.layout, causal=True,
                        order="global", dq=dq, dk=dk, dv=dv, ws=wsb)
    fn()
    ms = _time(fn, 5, flush)
    tf = (flops_fwd(w) + flops_bwd(w)) / (ms * 1e-3) / 1e12
    return {"split": f"ulysses {u} x ring {p_ring} ({w.layout})", "ms": round(ms, 4),
            "TFLOP/s": round(tf, 2), "frac": round(tf / peaks["bf16_tflops"], 4),
            "peak_source": f"{peak_src} bf16_tflops (burst: calls of under a second)",
            "note": "includes the 8 repack launches of Q/K/V/O/dO and dQ/dK/dV"}


# exp2 rate of the SFU: 16 results per clock per SM on sm_100 (the documented
# throughput of ex2.approx; a probe on this machine measured 16.0), times the SMs
# and the maximum SM clock.
EX2_PER_CLK_SM = 16


def tabular(rm, flush, hbm, peak_src, axis):
    """The tabular workload.  Row axis (20 sequences of 150000 rows, d = 24
    padded to 32, non-causal fused ring over 8 contiguous shards on strided
    views): TFLOP/s of its 4*d flops per pair against the tensor peak, and
    exponentials per second against the SFU rate (the d = 24 path does only
    96 MMA flops per exponential).  Feature axis (600000 sequences of 5
    tokens): GB/s of its algorithmic traffic (read Q, K, V, write O, LSE)
    against HBM.  `axis` is "row" or "feature"."""
    w = synthetic.TABULAR
    q, k, v = (t.cuda() for t in synthetic.tabular_inputs(w))
    R, F, E, H = w.rows, w.features, w.embed, w.heads
    if axis == "feature":
        fview = lambda x: x.view(w.batch * R, F, H, E // H)
        fo = torch.empty(w.batch * R, F, H, E // H, dtype=torch.bfloat16, device="cuda")
        flse = torch.empty(w.batch * R, H, F, device="cuda")
        fn = lambda: rm.attn_block_fwd(fview(q), fview(k), fview(v), N=F, P=1,
                                       layout="contiguous", causal=False, q_rank=0, kv_rank=0,
                                       out=fo, lse=flse)
        nbytes = 4 * q.numel() * 2 + flse.numel() * 4
        return hbm_row(rm, fn, 10, flush, nbytes, hbm, peak_src,
                       f"{w.batch * R * H} sequences x {F} tokens, d={E // H}")
    view = lambda x: x.view(w.batch, R, F * H, E // H)
    o = torch.empty(w.batch, R, F * H, E // H, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(w.batch, F * H, R, device="cuda")
    fn = lambda: rm.ring_attn_fwd(view(q), view(k), view(v), P=w.P, layout="contiguous",
                                  causal=False, out=o, lse=lse)
    fn()
    ms = _time(fn, 3, flush)
    seqs = w.batch * F * H
    pairs = seqs * R * R
    flops = 4 * (E // H) * pairs
    props = torch.cuda.get_device_properties(0)
    ex2_peak = EX2_PER_CLK_SM * props.multi_processor_count * 1965e6
    ex2_rate = pairs / (ms * 1e-3)
    row = {"shape": f"{seqs} sequences x {R} rows, d={E // H}", "ms": round(ms, 3),
           "TFLOP/s": round(flops / ms / 1e9, 2),
           "exp_per_s": round(ex2_rate / 1e12, 3), "exp_unit": "T exp2/s",
           "exp_frac": round(ex2_rate / ex2_peak, 4),
           "exp_peak_source": f"derived: {EX2_PER_CLK_SM}/clk/SM x {props.multi_processor_count} SMs x 1965 MHz"}
    return row


# ---------------------------------------------------------------------------
# the CPU oracle (baseline / reference arm)
# ---------------------------------------------------------------------------
_INPUTS = {}


def _headline_inputs():
    """The headline workload's inputs (drawn once per process: 17 s of CPU)."""
    if "w" not in _INPUTS:
        _INPUTS["w"] = synthetic.attention_inputs(HEADLINE)
    return _INPUTS["w"]


def sample_desc(n_queries: int) -> str:
    w = HEADLINE
    return (f"oracle ring fwd+bwd (numpy fp64) for the last {n_queries} queries (global positions "
            f"{w.N - n_queries}-{w.N - 1}, virtual rank 0's second zigzag chunk) of query head 0, "
            f"against all {w.N} keys they see in the {w.P} KV shards, N={w.N} zigzag P={w.P}; "
            f"the repack is not part of the sample")


def oracle_sample(n_queries: int = 512):
    """The oracle's ring fwd+bwd for the last `n_queries` queries of query
    head 0 (with KV head 0) of the headline workload: their partials against
    every KV shard in ring order, the LSE merge, the row term, then their
    backward contributions (their dQ, their share of dK / dV) against every
    shard.  Rows of the sequence's end see nearly every key, so the sample is
    the workload's densest part.  Returns (seconds, algorithmic flops)."""
    from oracle import attention as oatt
    from oracle import layouts as olay
    from oracle import merge as omerge
    from oracle import ring as oring
    w = HEADLINE
    q, k, v, do = _headline_inputs()
    f = lambda t: t[:, :, :1].float().numpy().astype(np.float64)
    qs, ks, vs, dos = f(q), f(k), f(v), f(do)
    L, C = w.N // w.P, w.N // (2 * w.P)
    t0 = time.perf_counter()
    perm = lambda x: olay.permute(x, w.layout, w.P)
    qr, kr, vr, dor = perm(qs), perm(ks), perm(vs), perm(dos)
    pos = [olay.rank_positions(w.layout, w.N, w.P, s) for s in range(w.P)]
    r = 0
    j0, j1 = L - n_queries, L  # the end of rank 0's second chunk (2P - 1)
    assert j1 - j0 <= C
    rows = slice(r * L + j0, r * L + j1)
    qpos = pos[r][j0:j1]
    parts = []
    for s in oring.schedule(w.P)[r]:
        cols = slice(s * L, (s + 1) * L)
        parts.append(oatt.attention_forward(qr[:, rows], kr[:, cols], vr[:, cols],
                                            causal=w.causal, q_pos=qpos, k_pos=pos[s]))
    o, lse = omerge.lse_merge([a for a, _ in parts], [b for _, b in parts])
    delta = oatt.delta_from_output(dor[:, rows], o)
    for s in oring.schedule(w.P)[r]:
        cols = slice(s * L, (s + 1) * L)
        oatt.attention_backward_block(qr[:, rows], kr[:, cols], vr[:, cols], dor[:, rows], lse,
                                      delta, causal=w.causal, q_pos=qpos, k_pos=pos[s])
    secs = time.perf_counter() - t0
    # visible pairs: the query at global position t sees t + 1 keys
    pairs = int((qpos + 1).sum())
    return secs, 14.0 * w.d * pairs


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(n_queries: int, reps: int = 3):
    """The oracle on `reps` runs of the sample (about 10-30 s of CPU in all);
    the rate extrapolated to the whole headline step is stated beside it."""
    secs, flops = 0.0, 0.0
    for _ in range(reps):
        s_, f_ = oracle_sample(n_queries)
        secs += s_
        flops += f_
    rate = flops / secs
    step_flops = flops_fwd(HEADLINE) + flops_bwd(HEADLINE)
    return {"value": round(rate / 1e12, 6), "unit": "TFLOP/s", "cores": _cores(),
            "cpu_model": _cpu_model(), "kind": "oracle", "sample": sample_desc(n_queries),
            "runs": reps, "seconds": round(secs, 2),
            "extrapolated_step_s": round(step_flops / rate, 1),
            "extrapolated": "the whole fwd+bwd step at the sample's rate"}


def bench_reference(args, world, rank):
    if rank != 0:
        return None
    for _ in range(args.warmup):
        oracle_sample(args.ref_sample_queries)
    secs, flops = 0.0, 0.0
    for _ in range(args.steps):
        s_, f_ = oracle_sample(args.ref_sample_queries)
        secs += s_
        flops += f_
    value = flops / secs / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": HEADLINE_NAME, "global_batch": 1, "seq_len": HEADLINE.N,
                   "parallelism": "single"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": _cores(),
                         "kind": "oracle",
                         "sample": sample_desc(args.ref_sample_queries) + ", per step"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-sample-queries", type=int, default=512,
                    help="queries in each oracle sample (cpu_baseline and --impl reference)")
    ap.add_argument("--case", choices=EXTRA_GROUPS, default=None,
                    help="run only this group of the extra measurements (no step, no baseline)")
    ap.add_argument("--small", action="store_true",
                    help="with --case: the smaller merge / repack / permute shapes (profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.case:
        from sequence_attention_rm_b200 import rm
        peaks, peak_src = load_peaks()
        dev = torch.device("cuda", 0)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        print(json.dumps({"case": args.case,
                          "extras": extras(rm, peaks, peak_src, dev, flush, only=args.case,
                                           small=args.small)}),
              flush=True)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        line = bench_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_init()
    line = bench_ours(args, world, rank, local)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
