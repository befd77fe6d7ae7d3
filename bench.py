#!/usr/bin/env python
"""Benchmark of the exact-attention library on B200.

One step = one forward (fa_fwd) plus one backward (fa_bwd) over the
long-context workload: batch 1, 16 heads, 16384 tokens, head_dim 128, bf16,
causal; Q, K, V, dO i.i.d. N(0, 1) from a seeded CPU generator (synthetic).
That step runs every stage of the hot path: tile planning, the TMA/tcgen05
forward with online softmax and the LSE epilogue, the backward preprocess,
the recomputing backward main kernel and the dQ conversion.

Metric: attention TFLOPS of the fwd+bwd step, counting 4*B*Hq*d per visible
(query, key) pair forward and 2.5x that backward (masked work not counted),
whole job over all ranks.  L2 is flushed (256 MB write) before every timed
step; each step is timed with its own CUDA events on the launching stream.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun (N > 1) every rank runs an independent replica (weak scaling,
no collective on the data path); the time is the max over ranks.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from seeded_inputs import (FP8_WORKLOADS, PAGED_WORKLOADS, VARLEN_WORKLOADS,  # noqa: E402
                           WORKLOADS, Workload, make_fp8_inputs, make_paged_inputs, make_qkv,
                           make_varlen_inputs, make_workload_inputs)

METRIC = "attention TFLOPS (fwd, fwd+bwd) on 1 B200 and % of dense FP16/BF16 tensor peak"
MAIN_WORKLOAD = "fwdbwd_1x16384_h16_d128_bf16_causal"
FWD_TABLE = ["fwd_2x2048_h8_d64_fp16", "fwd_2x2048_h8_d64_fp16_causal",
             "fwd_4x4096_h32_d64_fp16_causal", "fwd_2x4096_h32kv8_d128_bf16_causal_win256",
             "fwd_2x4096_h16_d256_bf16_causal"]
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
L2_FLUSH_BYTES = 256 << 20


# ---------------------------------------------------------------- context
def materialised_attention(q, k, v, scale, causal, window):
    """Standard attention with the full score matrix in memory, in plain
    PyTorch (cuBLAS products in the input dtype, softmax in fp32): the
    comparison the pages' speedup claims are made against ("optimizing-
    attention-flash", Quick start; "Что такое FlashAttention…", section
    "Основной механизм простыми словами").  Context for the bench table only;
    the library never calls it.  q [B, Nq, Hq, d], k / v [B, Nk, Hkv, d]."""
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    qh = q.permute(0, 2, 1, 3)
    kh = k.permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    vh = v.permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    scores = torch.matmul(qh, kh.transpose(2, 3)).float().mul_(scale)
    i = torch.arange(Nq, device=q.device).view(-1, 1) + (Nk - Nq)
    j = torch.arange(Nk, device=q.device).view(1, -1)
    wl, wr = window
    right = 0 if causal else wr
    hidden = torch.zeros(Nq, Nk, dtype=torch.bool, device=q.device)
    if right >= 0:
        hidden |= j > i + right
    if wl >= 0:
        hidden |= j < i - wl
    scores.masked_fill_(hidden, float("-inf"))
    probs = torch.softmax(scores, dim=-1).to(q.dtype)
    return torch.matmul(probs, vh).permute(0, 2, 1, 3)


# ---------------------------------------------------------------- counting
def visible_pairs(Nq, Nk, causal, window):
    """Number of (query, key) pairs the mask keeps, per (batch, head)."""
    i = np.arange(Nq, dtype=np.int64)
    ip = i + (Nk - Nq)
    wl, wr = window
    right = 0 if causal else wr
    lo = np.maximum(0, ip - wl) if wl >= 0 else np.zeros_like(ip)
    hi = np.minimum(Nk - 1, ip + right) if right >= 0 else np.full_like(ip, Nk - 1)
    return int(np.maximum(hi - lo + 1, 0).sum())


def fwd_flops(w: Workload):
    """Forward FLOPs: 4 * batch * q_heads * head_dim per visible pair."""
    return 4.0 * w.batch * w.q_heads * w.head_dim * \
        visible_pairs(w.seqlen_q, w.seqlen_k, w.causal, w.window)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# the sources each profiled kernel is compiled from (device code only)
KERNEL_SOURCES = {
    "fa_bwd_main_kernel": ("fa_bwd.cuh", "fa_dropout.cuh", "fa_exp2.cuh", "fa_ptx.cuh"),
    "fa_fwd_kernel": ("fa_fwd.cuh", "fa_dropout.cuh", "fa_exp2.cuh", "fa_ptx.cuh"),
}


def kernel_source_hash(kernel):
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "exact_attention_143_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None
    if it was taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            tr = json.load(f)
    except (OSError, ValueError):
        return None
    ent = tr.get(kernel)
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel):
        return None
    return ent.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.rows = []
        self.proc = None

    def _gpu_id(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            return str(self.dev)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self._gpu_id(), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for k, nm in enumerate(names):
                if r[5 + k].lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- distributed
def dist_setup(args):
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


def dist_max(x, world):
    """Max of x over all ranks (CPU tensor under gloo, CUDA tensor under nccl)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" \
        else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_workload(w: Workload, rank: int) -> Workload:
    """Each rank runs an independent replica of the workload (its own seed)."""
    return Workload(**{**w.__dict__, "seed": w.seed + rank})


def aggregate_tflops(world, flops_per_step, steps, max_total_ms):
    """Whole-job throughput: every rank's work over the slowest rank's time."""
    return world * flops_per_step * steps / (max_total_ms / 1e3) / 1e12


def dist_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- oracle timing
def oracle_sample_rate(w: Workload, budget_s: float):
    """Time the fp64 oracle (fwd + bwd) on a prefix of one head of workload w,
    sized to take about budget_s; returns (TFLOPS, sample description, cores)."""
    import oracle

    def run(T):
        q, k, v, do = make_qkv(1, T, T, 1, 1, w.head_dim, w.dtype, w.seed, with_dout=True)
        f = lambda t: t.float().double().numpy()  # noqa: E731
        t0 = time.perf_counter()
        oracle.attention_fwd(f(q), f(k), f(v), w.softmax_scale, w.causal, w.window)
        oracle.attention_bwd(f(q), f(k), f(v), f(do), w.softmax_scale, w.causal, w.window)
        dt = time.perf_counter() - t0
        flops = 3.5 * 4.0 * w.head_dim * visible_pairs(T, T, w.causal, w.window)
        return dt, flops

    T = min(512, w.seqlen_q)
    dt, flops = run(T)
    # the oracle's cost grows with the pair count, about T^2
    T = int(min(w.seqlen_q, max(T, T * math.sqrt(max(budget_s, 0.1) / max(dt, 1e-3)))))
    T = max(128, T // 128 * 128)
    dt, flops = run(T)
    sample = ("fp64 oracle fwd+bwd on the first %d tokens of one (batch, head) of %s "
              "(%.3g algorithmic GFLOP in %.2f s)" % (T, w.name, flops / 1e9, dt))
    import oracle as _o
    return flops / dt / 1e12, sample, _o.default_threads(), T, dt


# the pages' five benchmark configurations, in order (the sixth workload, d = 256,
# is this library's own addition)
CONFIGS = ["tiny_128_d64_fp16", "fwd_2x2048_h8_d64_fp16", "fwd_2x2048_h8_d64_fp16_causal",
           "fwd_4x4096_h32_d64_fp16_causal", "fwd_2x4096_h32kv8_d128_bf16_causal_win256",
           "fwdbwd_1x16384_h16_d128_bf16_causal"]


def oracle_config_times(budget_s: float):
    """Wall time of the fp64 oracle on every configuration: measured on the whole
    configuration where that fits about budget_s, otherwise on a prefix of one
    (batch, head) and extrapolated.  The oracle materialises every score of a
    (batch, head), so its cost is proportional to B * Hq * Nq * Nk: the full-size
    time is the sample time times that count over the sample's T * T."""
    import oracle
    f = lambda t: t.float().double().numpy()  # noqa: E731
    out = {}
    for name in CONFIGS:
        w = WORKLOADS[name]
        full_units = w.batch * w.q_heads * w.seqlen_q * w.seqlen_k

        def run(B, H, Hk, T, bwd):
            q, k, v, do = make_qkv(B, T, T, H, Hk, w.head_dim, w.dtype, w.seed, with_dout=True)
            qq, kk, vv, dd = f(q), f(k), f(v), f(do)
            t0 = time.perf_counter()
            oracle.attention_fwd(qq, kk, vv, w.softmax_scale, w.causal, w.window)
            t1 = time.perf_counter()
            tb = None
            if bwd:
                oracle.attention_bwd(qq, kk, vv, dd, w.softmax_scale, w.causal, w.window)
                tb = time.perf_counter() - t1
            return t1 - t0, tb

        ent = {}
        if full_units <= 4 * 2048 * 2048 * 8:  # the whole configuration
            tf, tb = run(w.batch, w.q_heads, w.kv_heads, w.seqlen_q, w.backward)
            ent = {"fwd_s": round(tf, 3), "measured": "whole configuration"}
            if tb is not None:
                ent["bwd_s"] = round(tb, 3)
        else:  # a prefix of one (batch, head), then extrapolated
            T = min(w.seqlen_q, 1024)
            tf, tb = run(1, 1, 1, T, w.backward)
            grow = max(1.0, math.sqrt(budget_s / max(tf + (tb or 0.0), 1e-3)))
            T = min(w.seqlen_q, max(T, int(T * grow) // 128 * 128))
            tf, tb = run(1, 1, 1, T, w.backward)
            scale = full_units / float(T * T)
            ent = {"fwd_s": round(tf * scale, 1), "measured": "first %d tokens of one (batch, head): "
                   "fwd %.2f s%s; full size extrapolated by B*Hq*Nq*Nk / T^2 = %.0f"
                   % (T, tf, "" if tb is None else ", bwd %.2f s" % tb, scale)}
            if tb is not None:
                ent["bwd_s"] = round(tb * scale, 1)
        out[name] = ent
    return out


# ---------------------------------------------------------------- our arm
def time_steps(step, K, W, flush, stream, per_step_events=None):
    """Run W warm-up steps, then K steps each bracketed by its own events, with
    an L2 flush before every step (outside the events).  Returns ms per step list."""
    for _ in range(W):
        flush()
        step(None)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    for i in range(K):
        flush()
        evs[i][0].record(stream)
        step(i)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def run_ours(args):
    import exact_attention_143_b200 as fa

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    w = WORKLOADS[args.workload]
    peaks, peak_src = load_peaks()

    # inputs (each rank an independent replica: seed + rank), resident in HBM
    wr = replica_workload(w, rank)
    q, k, v, do = make_workload_inputs(wr, with_dout=True)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty(w.batch, w.q_heads, w.seqlen_q, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    ws = torch.empty(fa.bwd_workspace_size(w.batch, w.seqlen_q, w.q_heads, w.head_dim),
                     dtype=torch.uint8, device=dev)
    flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush = lambda: flush_buf.zero_()  # noqa: E731
    kw = dict(softmax_scale=w.softmax_scale, causal=w.causal, window_size=w.window)

    K, W = args.steps, args.warmup
    main_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
    for a, b in main_ev:  # materialise the events before handing them to the library
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()

    def step(i):
        if i is not None:
            fa.set_bwd_main_events(*main_ev[i])
        else:
            fa.set_bwd_main_events(None, None)
        fa.fa_fwd(qd, kd, vd, out=o, lse=lse, **kw)
        fa.fa_bwd(dod, qd, kd, vd, o, lse, dq=dq, dk=dk, dv=dv, workspace=ws, **kw)

    clocks = ClockSampler(local)
    dist_barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    t_wall0 = time.perf_counter()
    ms = time_steps(step, K, W, flush, stream)
    t_wall = time.perf_counter() - t_wall0
    clk = clocks.stop()
    fa.set_bwd_main_events(None, None)
    dist_barrier(world)
    assert fa.get_device_error(dev) == fa.FA_OK
    main_ms = [a.elapsed_time(b) for a, b in main_ev]

    total_ms = sum(ms)
    total_ms_max = dist_max(total_ms, world)
    f_fwd = fwd_flops(w)
    f_step = 3.5 * f_fwd
    value = aggregate_tflops(world, f_step, K, total_ms_max)
    bwd_main_avg = sum(main_ms) / K
    achieved = 2.5 * f_fwd / (bwd_main_avg / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    traffic = load_traffic("fa_bwd_main_kernel")

    # end to end through the public API with host buffers: every step copies
    # its inputs in from pinned host memory, runs fwd + bwd and copies the
    # gradients back.  The copies run on their own streams against double
    # buffers, so step k's inputs go in while step k-1 computes and step k-2's
    # gradients come out (PCIe is full duplex); the timed region runs from the
    # first copy in to the last copy out.
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hdo = (t.pin_memory() for t in (q, k, v, do))
        hdq, hdk, hdv = (torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (q, k, v))
        ins = [(qd, kd, vd, dod), tuple(torch.empty_like(t) for t in (qd, kd, vd, dod))]
        outs = [(dq, dk, dv), tuple(torch.empty_like(t) for t in (dq, dk, dv))]
        s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))

        def e2e_run(n):
            ev_in = [torch.cuda.Event() for _ in range(n)]
            ev_cmp = [torch.cuda.Event() for _ in range(n)]
            ev_out = [torch.cuda.Event() for _ in range(n)]
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for s_ in (s_in, s_cmp, s_out):
                s_.wait_stream(stream)
            for i in range(n):
                bq, bk, bv, bdo = ins[i % 2]
                gq, gk, gv = outs[i % 2]
                with torch.cuda.stream(s_in):
                    if i >= 2:  # step i - 2, the last reader of this input set, is done
                        s_in.wait_event(ev_cmp[i - 2])
                    for dst, src in ((bq, hq), (bk, hk), (bv, hv), (bdo, hdo)):
                        dst.copy_(src, non_blocking=True)
                    ev_in[i].record(s_in)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(ev_in[i])
                    if i >= 2:  # step i - 2's gradients have left this output set
                        s_cmp.wait_event(ev_out[i - 2])
                    fa.fa_fwd(bq, bk, bv, out=o, lse=lse, **kw)
                    fa.fa_bwd(bdo, bq, bk, bv, o, lse, dq=gq, dk=gk, dv=gv, workspace=ws, **kw)
                    ev_cmp[i].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_cmp[i])
                    for dst, src in ((hdq, gq), (hdk, gk), (hdv, gv)):
                        dst.copy_(src, non_blocking=True)
                    ev_out[i].record(s_out)
            for s_ in (s_in, s_cmp, s_out):
                stream.wait_stream(s_)
            t1.record(stream)
            torch.cuda.synchronize()
            return t0.elapsed_time(t1)

        e2e_run(min(W, 3))  # warm-up
        Ke = max(3, min(K, 20))
        e_ms = dist_max(e2e_run(Ke), world)
        assert fa.get_device_error(dev) == fa.FA_OK
        h2d = sum(t.numel() * t.element_size() for t in (q, k, v, do))
        d2h = sum(t.numel() * t.element_size() for t in (dq, dk, dv))
        e2e = {"value": aggregate_tflops(world, f_step, Ke, e_ms), "unit": "TFLOPS",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": Ke,
               "ms_per_step": e_ms / Ke, "overlap": "copies in / compute / copies out on "
               "three streams, double-buffered"}

    # per-workload forward table (rank 0, N = 1 only): each pages' config alone
    table = {}
    if rank == 0 and world == 1 and not args.no_table:
        for name in FWD_TABLE:
            tw = WORKLOADS[name]
            tq, tk, tv = (t.to(dev) for t in make_workload_inputs(tw, with_dout=False))
            to = torch.empty_like(tq)
            tl = torch.empty(tw.batch, tw.q_heads, tw.seqlen_q, dtype=torch.float32, device=dev)
            tkw = dict(softmax_scale=tw.softmax_scale, causal=tw.causal, window_size=tw.window)
            # 10 warm-ups, then 50 timed launches with L2 flushed before each
            # (the headline figures), and 50 more back to back with L2 warm
            fwd1 = lambda _: fa.fa_fwd(tq, tk, tv, out=to, lse=tl, **tkw)  # noqa: E731
            tms = time_steps(fwd1, 50, 10, flush, stream)
            wms = time_steps(fwd1, 50, 0, lambda: None, stream)
            med = statistics.median(tms)
            tf = fwd_flops(tw) / (med / 1e3) / 1e12
            table[name] = {"fwd_ms_median": round(med, 4), "fwd_ms_min": round(min(tms), 4),
                           "fwd_ms_median_warm_l2": round(statistics.median(wms), 4),
                           "fwd_tflops": round(tf, 1), "frac_of_peak": round(tf / peak, 4)}
            # context: the materialised standard attention on the same inputs
            std1 = lambda _: materialised_attention(tq, tk, tv, tw.softmax_scale,  # noqa: E731
                                                    tw.causal, tw.window)
            sms = time_steps(std1, 5, 2, flush, stream)
            smed = statistics.median(sms)
            table[name].update({"standard_attention_ms_median": round(smed, 4),
                                "speedup_vs_standard": round(smed / med, 2)})
            torch.cuda.empty_cache()
            if tw.head_dim == 256:
                # the head_dim 256 backward (two halves of d per key tile),
                # dO i.i.d. N(0, 1) like the other backward workloads
                tdo = torch.randn(tq.shape, generator=torch.Generator().manual_seed(tw.seed + 1)
                                  ).to(tw.dtype).to(dev)
                fa.fa_fwd(tq, tk, tv, out=to, lse=tl, **tkw)
                tws = torch.empty(fa.bwd_workspace_size(tw.batch, tw.seqlen_q, tw.q_heads, 256),
                                  dtype=torch.uint8, device=dev)
                tdq, tdk, tdv = torch.empty_like(tq), torch.empty_like(tk), torch.empty_like(tv)
                bwd1 = lambda _: fa.fa_bwd(tdo, tq, tk, tv, to, tl, dq=tdq, dk=tdk, dv=tdv,  # noqa: E731
                                           workspace=tws, **tkw)
                bms = time_steps(bwd1, 20, 5, flush, stream)
                bmed = statistics.median(bms)
                btf = 2.5 * fwd_flops(tw) / (bmed / 1e3) / 1e12
                table[name].update({"bwd_ms_median": round(bmed, 4), "bwd_tflops": round(btf, 1),
                                    "bwd_frac_of_peak": round(btf / peak, 4)})
                del tdo, tws, tdq, tdk, tdv
            del tq, tk, tv, to, tl
        # packed variable-length batch (no padding): forward and backward
        for vw in VARLEN_WORKLOADS.values():
            vq, vk, vv, vdo, vcu, lens = make_varlen_inputs(vw)
            vq, vk, vv, vdo, vcu = (t.to(dev) for t in (vq, vk, vv, vdo, vcu))
            mx = max(lens)
            vkw = dict(softmax_scale=vw.softmax_scale, causal=vw.causal)
            vo, vl = fa.fa_fwd_varlen(vq, vk, vv, vcu, vcu, mx, mx, **vkw)
            vws = torch.empty(fa.bwd_workspace_size(len(lens), mx, vw.q_heads, vw.head_dim),
                              dtype=torch.uint8, device=dev)
            vdq, vdk, vdv = torch.empty_like(vq), torch.empty_like(vk), torch.empty_like(vv)
            vf = sum(4.0 * vw.q_heads * vw.head_dim * visible_pairs(n, n, vw.causal, (-1, -1))
                     for n in lens)
            fms_v = time_steps(lambda _: fa.fa_fwd_varlen(vq, vk, vv, vcu, vcu, mx, mx, out=vo,
                                                          lse=vl, **vkw), 10, 3, flush, stream)
            bms_v = time_steps(lambda _: fa.fa_bwd_varlen(vdo, vq, vk, vv, vo, vl, vcu, vcu, mx, mx,
                                                          dq=vdq, dk=vdk, dv=vdv, workspace=vws,
                                                          **vkw), 10, 3, flush, stream)
            fm_v, bm_v = statistics.median(fms_v), statistics.median(bms_v)
            table[vw.name] = {"total_tokens": sum(lens), "fwd_ms_median": round(fm_v, 4),
                              "fwd_tflops": round(vf / (fm_v / 1e3) / 1e12, 1),
                              "bwd_ms_median": round(bm_v, 4),
                              "bwd_tflops": round(2.5 * vf / (bm_v / 1e3) / 1e12, 1)}
            del vq, vk, vv, vdo, vo, vl, vws, vdq, vdk, vdv
        # decode against a paged KV cache: bound by HBM, reported in GB/s of
        # algorithmic traffic (every cached K and V row of every sequence read
        # once, q read and o, lse written once)
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        for pw in PAGED_WORKLOADS.values():
            plens = pw.lengths()
            pq, pkc, pvc, pbt, psl = (t.to(dev) for t in make_paged_inputs(
                pw.n_seqs, pw.Nq, pw.q_heads, pw.kv_heads, pw.head_dim, pw.dtype, pw.page_size,
                plens, pw.seed))
            po = torch.empty_like(pq)
            pl = torch.empty(pw.n_seqs, pw.q_heads, pw.Nq, dtype=torch.float32, device=dev)
            pneed = fa.fa_fwd_paged_workspace_size(pw.n_seqs, pw.Nq, pw.q_heads, pw.kv_heads,
                                                   pw.head_dim, pw.page_size, pbt.shape[1])
            pws = torch.empty(max(pneed, 256), dtype=torch.uint8, device=dev)
            pkw = dict(softmax_scale=pw.softmax_scale, causal=pw.causal)
            pms = time_steps(lambda _: fa.fa_fwd_paged(pq, pkc, pvc, pbt, psl, out=po, lse=pl,
                                                       workspace=pws, **pkw), 20, 3, flush, stream)
            pm = statistics.median(pms)
            kv_bytes = 2 * sum(plens) * pw.kv_heads * pw.head_dim * pkc.element_size()
            io_bytes = (2 * pq.numel() * pq.element_size() + pl.numel() * 4 + psl.numel() * 4 +
                        sum((n + pw.page_size - 1) // pw.page_size for n in plens) * 4)
            gbs = (kv_bytes + io_bytes) / (pm / 1e3) / 1e9
            table[pw.name] = {"cached_tokens": sum(plens), "ms_median": round(pm, 4),
                              "ms_min": round(min(pms), 4),
                              "algorithmic_bytes": kv_bytes + io_bytes,
                              "gb_per_s": round(gbs, 1), "hbm_peak_gb_per_s": hbm,
                              "frac_of_hbm": round(gbs / hbm, 4),
                              "decode_tokens_per_s": round(pw.n_seqs * pw.Nq / (pm / 1e3), 1)}
            del pq, pkc, pvc, pbt, psl, po, pl, pws
        # FP8 (e4m3) forward: counted FLOPs over the e4m3 tensor peak, taken as
        # the measured bf16 rate times the nominal fp8 / bf16 ratio of 2
        for fw in FP8_WORKLOADS.values():
            fq, fk, fv = (t.to(dev) for t in make_fp8_inputs(
                fw.batch, fw.seqlen, fw.seqlen, fw.q_heads, fw.kv_heads, fw.head_dim,
                fw.descales, fw.seed))
            fo = torch.empty(fq.shape, dtype=torch.bfloat16, device=dev)
            fl = torch.empty(fw.batch, fw.q_heads, fw.seqlen, dtype=torch.float32, device=dev)
            fkw = dict(softmax_scale=fw.softmax_scale, causal=fw.causal,
                       descale_q=fw.descales[0], descale_k=fw.descales[1],
                       descale_v=fw.descales[2])
            fms8 = time_steps(lambda _: fa.fa_fwd_fp8(fq, fk, fv, out=fo, lse=fl, **fkw), 20, 3,
                              flush, stream)
            fm8 = statistics.median(fms8)
            ff = 4.0 * fw.batch * fw.q_heads * fw.head_dim * visible_pairs(
                fw.seqlen, fw.seqlen, fw.causal, (-1, -1))
            tf8 = ff / (fm8 / 1e3) / 1e12
            table[fw.name] = {"fwd_ms_median": round(fm8, 4), "fwd_ms_min": round(min(fms8), 4),
                              "fwd_tflops": round(tf8, 1), "fp8_peak_tflops": 2 * peak,
                              "frac_of_fp8_peak": round(tf8 / (2 * peak), 4),
                              "frac_of_bf16_peak": round(tf8 / peak, 4)}
            del fq, fk, fv, fo, fl
        # the main workload with dropout p = 0.1 (keep bits from the in-kernel
        # generator): forward and backward, counted FLOPs as without dropout
        dkw = dict(kw, dropout_p=0.1, seed=1234, offset=0)
        dfms = time_steps(lambda _: fa.fa_fwd(qd, kd, vd, out=o, lse=lse, **dkw), 10, 3, flush,
                          stream)
        dbms = time_steps(lambda _: fa.fa_bwd(dod, qd, kd, vd, o, lse, dq=dq, dk=dk, dv=dv,
                                              workspace=ws, **dkw), 10, 3, flush, stream)
        dfm, dbm = statistics.median(dfms), statistics.median(dbms)
        table[w.name + "_dropout0.1"] = {"fwd_ms_median": round(dfm, 4),
                                         "fwd_tflops": round(f_fwd / (dfm / 1e3) / 1e12, 1),
                                         "bwd_ms_median": round(dbm, 4),
                                         "bwd_tflops": round(2.5 * f_fwd / (dbm / 1e3) / 1e12, 1)}
        # the main workload's forward and backward separately
        fms = time_steps(lambda _: fa.fa_fwd(qd, kd, vd, out=o, lse=lse, **kw), 10, 3, flush,
                         stream)
        bms = time_steps(lambda _: fa.fa_bwd(dod, qd, kd, vd, o, lse, dq=dq, dk=dk, dv=dv,
                                             workspace=ws, **kw), 10, 3, flush, stream)
        fm, bm = statistics.median(fms), statistics.median(bms)
        table[w.name] = {"fwd_ms_median": round(fm, 4),
                         "fwd_tflops": round(f_fwd / (fm / 1e3) / 1e12, 1),
                         "bwd_ms_median": round(bm, 4),
                         "bwd_tflops": round(2.5 * f_fwd / (bm / 1e3) / 1e12, 1),
                         "frac_of_peak_fwd": round(f_fwd / (fm / 1e3) / 1e12 / peak, 4),
                         "frac_of_peak_bwd": round(2.5 * f_fwd / (bm / 1e3) / 1e12 / peak, 4)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, sample, cores, _, _ = oracle_sample_rate(w, args.cpu_seconds)
        cpu = {"value": tf, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "sample": sample,
               "wall_s_per_config": oracle_config_times(args.cpu_seconds / 5.0)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": round(total_ms_max / K, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded N(0,1) Q, K, V, dO)",
            "config": {**w.describe(), "l2": "flushed (256 MB write) before every timed step",
                       "parallelism": "replicas" if world > 1 else "single GPU",
                       "step": "fa_fwd + fa_bwd"},
            "frac_of_peak": round(value / world / peak, 4),
            "roofline": {"bound": "tensor", "kernel": "fa_bwd_main_kernel",
                         "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "peak_source": "%s bf16_tflops (burst)" % peak_src,
                         "frac_of_sustained": round(
                             achieved / float(peaks.get("bf16_tflops_sustained", peak)), 4),
                         "launch_ms_avg": round(bwd_main_avg, 4)},
            "clocks": clk,
            "e2e": e2e,
            "gpu_launches": 4 * K,
            "cpu_baseline": cpu,
            "workloads": table,
            "wall_s_timed_region": round(t_wall, 3),
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    """The fp64 CPU oracle, as it stands, on bounded samples of the same workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    K, W = args.steps, args.warmup
    per_step = max(0.5, args.ref_budget_s / max(1, K + W))
    _, _, cores, T, _ = oracle_sample_rate(w, per_step)
    import oracle
    q, k, v, do = make_qkv(1, T, T, 1, 1, w.head_dim, w.dtype, w.seed, with_dout=True)
    f = lambda t: t.float().double().numpy()  # noqa: E731
    qq, kk, vv, dd = f(q), f(k), f(v), f(do)
    flops = 3.5 * 4.0 * w.head_dim * visible_pairs(T, T, w.causal, w.window)

    def step():
        oracle.attention_fwd(qq, kk, vv, w.softmax_scale, w.causal, w.window)
        oracle.attention_bwd(qq, kk, vv, dd, w.softmax_scale, w.causal, w.window)

    for _ in range(W):
        step()
    t0 = time.perf_counter()
    for _ in range(K):
        step()
    dt = time.perf_counter() - t0
    value = flops * K / dt / 1e12
    sample = ("fp64 oracle fwd+bwd on the first %d tokens of one (batch, head) of %s per step"
              % (T, w.name))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": K, "warmup": W,
        "ms_per_step": dt / K * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) Q, K, V, dO)",
        "config": {**w.describe(), "sample_tokens": T},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }))


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=MAIN_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-table", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target duration of the oracle CPU-baseline sample")
    ap.add_argument("--ref-budget-s", type=float, default=120.0,
                    help="target duration of the whole reference-arm run")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
