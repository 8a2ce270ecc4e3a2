#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one call of the library on one batch of synthetic input of the
chosen workload (default: the causal 2K-context prefill, B=4 H=16 N=2048
d=128).  The timed region is exactly K steps bracketed by a barrier and a
device synchronisation; each step is timed with CUDA events on the stream it
runs on.  A second pass of steps then has the library record an event pair
just around each step's dominant kernel (fa_set_timing_events), which gives
the roofline's achieved rate.  Rank 0 prints one JSON line.  Under torchrun every rank runs the
same workload on its own GPU (independent (batch, head) partitions, weak
scaling, no data-path collective) and the time is the maximum over ranks.

``--impl reference`` times the fp64 CPU oracle (the deliberately slow
definition) on the host cores, on a bounded sample of the same workload.
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
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from io_aware_exact_35_b200 import inputs  # noqa: E402

METRIC = "bf16 attention TFLOP/s fwd & bwd; decode KV-read GB/s; % of roofline"
DEFAULT_WORKLOAD = "fwd_causal_B4_H16_N2048_d128"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    "fwd": ("fa_fwd.cu", "sm100.cuh"),
    "fwd_varlen": ("fa_fwd.cu", "sm100.cuh"),
    "fwd_fp8": ("fa_fwd.cu", "sm100.cuh"),
    "bwd": ("fa_bwd.cu", "sm100.cuh"),
    "decode": ("fa_decode.cu", "sm100.cuh"),
}


def kernel_sources_sha(kind):
    """Hash of the source files a kernel is built from (traffic figures taken
    by ncu are only reported while this hash still matches)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "io_aware_exact_35_b200", "csrc")
    for name in KERNEL_SOURCES[kind]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key, kind, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on this workload and the kernel's sources have not changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    ent = d.get(kernel_key)
    if not ent or ent.get("source_sha") != kernel_sources_sha(kind):
        return None
    if ent.get("workload") != workload:
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        self.dev = device_index

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            cmd += ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
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
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- workloads
def decode_kernel_key(d, group, paged):
    """Name of the split kernel the library launches for decode: the grouped
    tensor-core kernel with qh query heads per CTA (the whole group up to 16
    heads, else 16 or 8 of them), or the per-head kernel."""
    qh = group if group <= 16 else (16 if group % 16 == 0 else (8 if group % 8 == 0 else 0))
    suffix = ",paged" if paged else ""
    if group > 1 and qh > 0:
        return f"fa_decode_group_mma_kernel<{d},{qh}{suffix}>"
    return f"fa_decode_split_kernel<{d}{suffix}>"


def workload_config(w, parallelism):
    cfg = {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.kv_heads, "N": w.N or None,
           "d": w.d, "causal": w.causal, "parallelism": parallelism}
    if w.page:
        cfg["page_size"] = w.page
    return cfg


def fwd_flops(w):
    f = 4.0 * w.B * w.H * w.N * w.N * w.d
    return f * 0.5 if w.causal else f


def varlen_flops(w, lens):
    """Forward FLOPs of a ragged batch: the fwd convention per sequence."""
    f = sum(4.0 * w.H * L * L * w.d for L in lens)
    return f * 0.5 if w.causal else f


def decode_bytes(w, seqlens):
    """Algorithmic KV bytes: every cached key and value row read once."""
    return float(sum(int(L) for L in seqlens)) * w.kv_heads * w.d * 2 * 2


class Runner:
    """Holds device buffers of one workload and launches one step on demand."""

    def __init__(self, w, dev):
        from io_aware_exact_35_b200 import fa
        self.fa, self.w, self.dev = fa, w, dev
        self.host = inputs.workload_inputs(w)
        if w.kind == "fwd_fp8":  # e4m3 q, k, vt and their descale factors
            self.host, self.fp8_scales = list(self.host[:3]), self.host[3]
        self.dbuf = [t.to(dev) for t in self.host]
        if w.kind == "fwd":
            q, k, v = self.dbuf
            self.o = torch.empty_like(q)
            self.lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
            self.work = fwd_flops(w)
            self.unit, self.kind_bound = "TFLOP/s", "tensor"
            self.launches_per_step = 1
            self.kernel_key = f"fa_fwd_kernel<{w.d},{str(w.causal).lower()}>"
        elif w.kind == "fwd_fp8":
            q8 = self.host[0]
            self.o = torch.empty(q8.shape, dtype=torch.bfloat16, device=dev)
            self.lse = torch.empty(q8.shape[:3], dtype=torch.float32, device=dev)
            self.work = fwd_flops(w)
            self.unit, self.kind_bound = "TFLOP/s", "tensor_fp8"
            self.launches_per_step = 1
            self.kernel_key = f"fa_fwd_kernel<{w.d},{str(w.causal).lower()},e4m3>"
        elif w.kind == "fwd_varlen":
            q, k, v, cu_q, cu_k = self.dbuf
            lens = (self.host[3][1:] - self.host[3][:-1]).tolist()
            self.max_len = max(lens)
            self.o = torch.empty_like(q)
            self.lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=dev)
            self.work = varlen_flops(w, lens)
            self.unit, self.kind_bound = "TFLOP/s", "tensor"
            self.launches_per_step = 1
            self.kernel_key = f"fa_fwd_kernel<{w.d},{str(w.causal).lower()},varlen>"
        elif w.kind == "bwd":
            q, k, v, do = self.dbuf
            self.o, self.lse = fa.fwd(q, k, v, causal=w.causal, scale=w.scale)
            # O and LSE are inputs of the backward too (from the forward pass)
            self.host = list(self.host) + [self.o.cpu(), self.lse.cpu()]
            self.dbuf = list(self.dbuf) + [self.o, self.lse]
            self.dq, self.dk, self.dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            self.ws = torch.empty(fa.bwd_workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8,
                                  device=dev)
            self.work = 2.5 * fwd_flops(w)
            self.unit, self.kind_bound = "TFLOP/s", "tensor"
            self.launches_per_step = 3
            self.kernel_key = f"fa_bwd_kernel<{w.d},{str(w.causal).lower()}>"
        else:
            q, kc, vc, sl = self.dbuf
            lcap = kc.shape[2]
            if w.page:
                # paged cache: pools and page table replace the contiguous caches
                kp, vp, table = inputs.page_cache(*self.host[1:3], self.host[3], w.page,
                                                  w.seed + 1)
                self.host = [self.host[0], kp, vp, table, self.host[3]]
                self.dbuf = [t.to(dev) for t in self.host]
                q = self.dbuf[0]
                lcap = table.shape[1] * w.page
            self.o = torch.empty_like(q)
            self.lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
            self.ws = torch.empty(fa.decode_workspace_size(w.B, w.H, lcap, w.d),
                                  dtype=torch.uint8, device=dev)
            self.work = decode_bytes(w, self.host[-1].tolist())
            self.unit, self.kind_bound = "GB/s", "hbm"
            self.launches_per_step = 2
            self.kernel_key = decode_kernel_key(w.d, w.H // w.kv_heads, bool(w.page))
        # every output of a step, copied back to pinned host memory by the
        # end-to-end measurement
        outs = self.outputs()
        self.out_host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
        self.working_set = sum(t.numel() * t.element_size() for t in self.dbuf)
        self.flush = None
        if self.working_set < 2 * L2_BYTES:
            self.flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def outputs(self):
        """The tensors one step writes (all of them are results)."""
        if self.w.kind == "bwd":
            return [self.dq, self.dk, self.dv]
        return [self.o, self.lse]

    def step(self, bufs=None):
        w, fa = self.w, self.fa
        b = bufs if bufs is not None else self.dbuf
        if w.kind == "fwd":
            fa.fwd(b[0], b[1], b[2], causal=w.causal, scale=w.scale, out=self.o, lse=self.lse)
        elif w.kind == "fwd_fp8":
            qs, ks, vs = self.fp8_scales
            fa.fwd_fp8(b[0], b[1], b[2], qs, ks, vs, causal=w.causal, scale=w.scale, out=self.o,
                       lse=self.lse)
        elif w.kind == "fwd_varlen":
            fa.fwd_varlen(b[0], b[1], b[2], b[3], b[4], self.max_len, causal=w.causal,
                          scale=w.scale, out=self.o, lse=self.lse)
        elif w.kind == "bwd":
            fa.bwd(b[0], b[1], b[2], b[4], b[3], b[5], causal=w.causal, scale=w.scale,
                   dq=self.dq, dk=self.dk, dv=self.dv, workspace=self.ws)
        elif w.page:
            fa.decode_paged(b[0], b[1], b[2], b[3], b[4], scale=w.scale, out=self.o,
                            lse=self.lse, workspace=self.ws)
        else:
            fa.decode(b[0], b[1], b[2], b[3], scale=w.scale, out=self.o, lse=self.lse,
                      workspace=self.ws)
        return self.outputs()

    def value(self, seconds):
        return self.work / seconds / 1e12 if self.unit == "TFLOP/s" else self.work / seconds / 1e9


def barrier(world):
    if world > 1:
        torch.distributed.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(x, world, dev):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(per_rank_value, world):
    """Whole-job throughput: every rank processes the same units (weak
    scaling) and the time is the maximum over ranks, so the job's rate is the
    slowest rank's rate times the number of ranks."""
    return per_rank_value * world


def time_device(r, steps, warmup, world, dev):
    """Kernel-only timing: inputs resident in HBM; events around each step."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        if r.flush is not None:
            r.flush.zero_()
        r.step()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for ev in starts + ends:
        ev.record(stream)  # creates the CUDA event behind it, outside the timed loop
    sampler = ClockSampler(dev.index or 0)
    sampler.start()
    time.sleep(0.3)
    # the sampler's start-up left the GPU idle: bring it back to speed
    for _ in range(min(warmup, 3)):
        if r.flush is not None:
            r.flush.zero_()
        r.step()
    barrier(world)
    t0 = time.perf_counter()
    for i in range(steps):
        if r.flush is not None:
            r.flush.zero_()
        starts[i].record(stream)
        r.step()
        ends[i].record(stream)
    barrier(world)
    wall = time.perf_counter() - t0
    clocks = sampler.stop()
    per = [s.elapsed_time(e) * 1e-3 for s, e in zip(starts, ends)]
    mean_s = max_over_ranks(float(np.mean(per)), world, dev)
    kern_s = time_main_kernel(r, steps, world, dev)
    return mean_s, per, wall, clocks, kern_s


def time_main_kernel(r, steps, world, dev):
    """Mean device time of each step's dominant kernel alone: the library
    records a pair of events just around it (fa_set_timing_events).  A pass
    of its own, after the timed steps, because the two extra event records
    add a few microseconds to a step."""
    stream = torch.cuda.current_stream()
    n = max(3, min(steps, 200))
    kstarts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    kends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for ev in kstarts + kends:
        ev.record(stream)  # creates the CUDA event behind it
    barrier(world)
    for i in range(n):
        if r.flush is not None:
            r.flush.zero_()
        r.fa.set_timing_events(kstarts[i], kends[i])
        r.step()
    r.fa.set_timing_events(None, None)
    barrier(world)
    kern = [s.elapsed_time(e) * 1e-3 for s, e in zip(kstarts, kends)]
    return max_over_ranks(float(np.mean(kern)), world, dev)


def time_e2e(r, steps, warmup, world, dev):
    """End-to-end through the public API: every step copies its inputs from
    pinned host memory to the device, makes the call, and copies its results
    back to pinned host memory.  Steps are pipelined as a user streaming
    batches would run them: inputs are double-buffered on a copy-in stream,
    the calls run on a compute stream and the results go back on a copy-out
    stream, so step k+1's inputs travel while step k computes and its results
    travel back (both directions of the host link at once).  Events order the
    reuse of every buffer; the timed region runs from the first copy in to
    the last copy out."""
    host = [t.pin_memory() for t in r.host]
    dbufs = [[torch.empty_like(t, device=dev) for t in r.host] for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host)
    d2h = sum(t.numel() * t.element_size() for t in r.out_host)
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    comp_done = [torch.cuda.Event() for _ in range(2)]  # buffer k % 2 free again
    in_done = [torch.cuda.Event() for _ in range(2)]
    out_done = torch.cuda.Event()                       # results of the last step read
    state = {"k": 0}

    def one():
        k = state["k"]
        b = k & 1
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(comp_done[b])  # the call of step k-2 has read buffer b
            for hb, db in zip(host, dbufs[b]):
                db.copy_(hb, non_blocking=True)
            in_done[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[b])
            if k >= 1:
                s_comp.wait_event(out_done)    # step k-1's results have left the outputs
            outs = r.step(dbufs[b])
            comp_done[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            for out, oh in zip(outs, r.out_host):
                oh.copy_(out, non_blocking=True)
            out_done.record(s_out)
        state["k"] = k + 1

    for _ in range(max(1, warmup)):
        one()
    torch.cuda.synchronize()
    barrier(world)
    st, en = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    st.record(s_in)
    s_in.wait_event(out_done)  # start from an idle pipeline
    for _ in range(steps):
        one()
    en.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    sec = max_over_ranks(st.elapsed_time(en) * 1e-3 / steps, world, dev)
    return sec, h2d, d2h


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, w, total_budget=150.0, emit=True):
    """The fp64 CPU oracle as it stands, on a bounded sample of the workload."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count() or 1
    host = inputs.workload_inputs(w)
    f64 = inputs.to_f64
    budget = total_budget / max(1, args.steps + args.warmup)  # seconds per step
    rng = np.random.default_rng(w.seed)
    if w.kind == "fwd_varlen":
        q, k, v, cu_q, cu_k = host
        lens = (cu_q[1:] - cu_q[:-1]).tolist()
        group = w.H // w.kv_heads
        seq_heads = [(b, h) for b in range(w.B) for h in range(w.H)]
        L0, c0 = lens[0], int(cu_q[0])
        t0 = time.perf_counter()
        oracle.attention_forward_rows(f64(q[c0:c0 + L0, 0]), f64(k[c0:c0 + L0, 0]),
                                      f64(v[c0:c0 + L0, 0]), w.causal, w.scale,
                                      np.arange(min(64, L0)))
        per_row = (time.perf_counter() - t0) / min(64, L0)
        rows_per_step = int(max(1, budget / max(per_row, 1e-9)))
        sample = (f"up to {rows_per_step} query rows of one (sequence, head) per step, "
                  "rows drawn uniformly")

        def step(i):
            b, h = seq_heads[i % len(seq_heads)]
            L, q0, k0 = lens[b], int(cu_q[b]), int(cu_k[b])
            rows = np.sort(rng.integers(0, L, min(rows_per_step, L)))
            qh = f64(q[q0:q0 + L, h])
            kh, vh = f64(k[k0:k0 + L, h // group]), f64(v[k0:k0 + L, h // group])
            t = time.perf_counter()
            oracle.attention_forward_rows(qh, kh, vh, w.causal, w.scale, rows)
            dt = time.perf_counter() - t
            keys = (rows + 1).sum() if w.causal else rows.size * L
            return dt, 4.0 * keys * w.d, 1.0
        unit = "TFLOP/s"
        scale_out = 1e12
    elif w.kind == "bwd":
        # the oracle's backward of whole (batch, head) problems: it recomputes
        # S and P from q, k, v and forms dV, dP, dS, dQ, dK in fp64
        q, k, v, do = host[:4]
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
        group = w.H // w.kv_heads
        sample = "one whole (batch, head) backward (all N query and key rows) per step"

        def step(i):
            b, h = heads[i % len(heads)]
            args_ = (f64(q[b, h]), f64(k[b, h // group]), f64(v[b, h // group]), f64(do[b, h]))
            t = time.perf_counter()
            oracle.attention_backward(*args_, w.causal, w.scale)
            dt = time.perf_counter() - t
            f = 4.0 * w.N * w.N * w.d * (0.5 if w.causal else 1.0)
            return dt, 2.5 * f, 1.0
        unit = "TFLOP/s"
        scale_out = 1e12
    elif w.kind in ("fwd", "fwd_fp8"):
        if w.kind == "fwd_fp8":  # the oracle takes the real (descaled) values
            q8, k8, vt8, (qs, ks, vs) = host
            q = torch.from_numpy(inputs.fp8_to_f64(q8, qs))
            k = torch.from_numpy(inputs.fp8_to_f64(k8, ks))
            v = torch.from_numpy(inputs.fp8_to_f64(vt8.transpose(-1, -2).contiguous(), vs))
        else:
            q, k, v = (t for t in host[:3])
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
        # rows per step sized from a probe so that a step stays within budget
        b0, h0 = heads[0]
        qh, kh, vh = f64(q[b0, h0]), f64(k[b0, 0]), f64(v[b0, 0])
        t0 = time.perf_counter()
        oracle.attention_forward_rows(qh, kh, vh, w.causal, w.scale, np.arange(min(64, w.N)))
        per_row = (time.perf_counter() - t0) / min(64, w.N)
        rows_per_step = int(max(1, min(w.N, budget / max(per_row, 1e-9))))
        sample = f"{rows_per_step} query rows of one (batch, head) per step, rows drawn uniformly"

        group = w.H // w.kv_heads

        def step(i):
            b, h = heads[i % len(heads)]
            rows = np.sort(rng.integers(0, w.N, rows_per_step))
            qh, kh, vh = f64(q[b, h]), f64(k[b, h // group]), f64(v[b, h // group])
            t = time.perf_counter()
            oracle.attention_forward_rows(qh, kh, vh, w.causal, w.scale, rows)
            dt = time.perf_counter() - t
            keys = (rows + 1).sum() if w.causal else rows.size * w.N
            return dt, 4.0 * keys * w.d, 1.0
        unit = "TFLOP/s"
        scale_out = 1e12
    else:
        q, kc, vc, sl = host
        sample = "one (batch, head) cache prefix per step"

        def step(i):
            b = i % w.B
            h = (i // w.B) % w.H
            L = int(sl[b])
            hk = h // (w.H // w.kv_heads)
            qq, kk, vv = f64(q[b:b + 1, h:h + 1]), f64(kc[b:b + 1, hk:hk + 1, :L]), f64(vc[b:b + 1, hk:hk + 1, :L])
            t = time.perf_counter()
            oracle.decode_forward(qq, kk, vv, [L], w.scale)
            return time.perf_counter() - t, float(L) * w.d * 4, 1.0
        unit = "GB/s"
        scale_out = 1e9
    for i in range(args.warmup):
        step(i)
    tot_t, tot_w = 0.0, 0.0
    for i in range(args.steps):
        dt, work, mult = step(args.warmup + i)
        tot_t += dt * mult
        tot_w += work
    value = tot_w / tot_t / scale_out
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, "cpu"),
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    if emit:
        print(json.dumps(line), flush=True)
    return line


def cpu_baseline(w, seconds=15.0):
    """Oracle timing on the host cores for the JSON line (bounded sample)."""
    ns = argparse.Namespace(steps=6, warmup=1, gpus=1)
    return run_reference(ns, w, total_budget=seconds, emit=False)["cpu_baseline"]


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--skip-baselines", action="store_true",
                    help="profiling runs: skip the end-to-end and CPU-oracle legs")
    ap.add_argument("--no-extra", action="store_true",
                    help="report only the chosen workload (no `workloads` object)")
    ap.add_argument("--B", type=int, default=None,
                    help="profiling runs: override the workload's batch size")
    args = ap.parse_args()
    w = inputs.WORKLOADS[args.workload]
    if args.B is not None:
        import dataclasses
        w = dataclasses.replace(w, B=args.B, name=f"{w.name}[B={args.B}]")
    default_steps = {"fwd": 4000, "bwd": 300, "decode": 800, "fwd_varlen": 1000,
                     "fwd_fp8": 4000}[w.kind]
    if w.name == "fwd_causal_B1_H32_N32768_d128":
        default_steps = 200
    if args.steps is None:
        args.steps = default_steps
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, w)
        return

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=120),
                                             device_id=dev)
    from io_aware_exact_35_b200 import fa
    fa.lib()

    r = Runner(w, dev)
    res = measure(r, args.steps, args.warmup, world, dev, e2e=not args.skip_baselines)
    err = fa.get_device_error()
    line = {
        "metric": METRIC, "value": res["value"], "unit": r.unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
        "ms_per_step_median": res["ms_per_step_median"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if w.kind == "fwd_fp8" else "bf16", "data": "synthetic",
        "config": dict(workload_config(w, f"replicas{world}" if world > 1 else "single"),
                       l2=res["l2"]),
        "roofline": res["roofline"],
        "e2e": res["e2e"],
        "gpu_launches": args.steps * r.launches_per_step,
        "clocks": res["clocks"],
        "device_error": err,
        "wall_s_timed_region": res["wall_s"],
    }
    del r
    if not args.skip_baselines and not args.no_extra and w.name == DEFAULT_WORKLOAD:
        # the other full-size configurations, each timed the same way (device
        # time of whole steps, dominant kernel alone for the roofline)
        line["workloads"] = {}
        for name, steps in EXTRA_WORKLOADS:
            rx = Runner(inputs.WORKLOADS[name], dev)
            rr = measure(rx, steps, args.warmup, world, dev, e2e=False)
            rr["device_error"] = fa.get_device_error()
            rr.pop("e2e", None)
            rr["steps"] = steps
            rr["warmup"] = args.warmup
            rr["unit"] = rx.unit
            line["workloads"][name] = rr
            del rx
            torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.skip_baselines:
        try:
            line["cpu_baseline"] = cpu_baseline(w)
        except Exception as e:  # the baseline is reported, not required
            line["cpu_baseline"] = {"value": None, "error": str(e)[:200]}
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# The other full-size configurations reported beside the default one, with
# their timed steps: the 32K-context forward, the backward, the decode.
EXTRA_WORKLOADS = (("fwd_causal_B1_H32_N32768_d128", 10),
                   ("bwd_causal_B2_H16_N8192_d128", 30),
                   ("decode_B16_H32_d128_L4096-16384", 100))
NOMINAL = {"tensor": 2250.0, "tensor_fp8": 4500.0, "hbm": 8000.0}


def measure(r, steps, warmup, world, dev, e2e=True):
    """Times one workload: the step rate (`value`), the dominant kernel's
    roofline, clocks and (optionally) the end-to-end rate."""
    mean_s, per, wall, clocks, kern_s = time_device(r, steps, warmup, world, dev)
    if e2e:
        e2e_s, h2d, d2h = time_e2e(r, max(3, min(steps, 50)), 2, world, dev)
    else:
        e2e_s, h2d, d2h = float("nan"), 0, 0
    peaks, peak_src = load_peaks()
    if r.kind_bound == "tensor":
        peak = float(peaks["bf16_tflops"])
        src = f"{peak_src} bf16_tflops (burst)"
    elif r.kind_bound == "tensor_fp8":
        # the 8-bit contraction's peak: the measured bf16 peak x the nominal
        # fp8 / bf16 ratio (4.5 / 2.25 PFLOP/s dense)
        peak = 2.0 * float(peaks["bf16_tflops"])
        src = f"{peak_src} bf16_tflops (burst) x 2 (nominal e4m3 / bf16)"
    else:
        peak = float(peaks["hbm_gbs"])
        src = f"{peak_src} hbm_gbs (copy)"
    ach = r.work / kern_s / (1e12 if r.unit == "TFLOP/s" else 1e9)
    roof = {"bound": "hbm" if r.kind_bound == "hbm" else "tensor", "achieved": ach,
            "peak": peak, "unit": r.unit, "frac": ach / peak,
            "traffic": profiled_traffic(r.kernel_key, r.w.kind, r.w.name),
            "peak_source": src, "kernel": r.kernel_key,
            # mean device time of the dominant kernel per step
            "kernel_ms": kern_s * 1e3,
            # against the nominal dense bf16 (2.25 PFLOP/s) / e4m3 / HBM (8 TB/s) figure
            "frac_nominal": ach / NOMINAL[r.kind_bound]}
    return {
        "value": job_value(r.value(mean_s), world),
        "ms_per_step": mean_s * 1e3,
        "ms_per_step_median": float(np.median(per)) * 1e3,
        "roofline": roof,
        "clocks": clocks,
        "e2e": {"value": r.value(e2e_s) * world, "unit": r.unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "l2": "flushed (256 MB write) before every step" if r.flush is not None
              else "inputs larger than L2",
        "wall_s": wall,
    }


if __name__ == "__main__":
    main()
