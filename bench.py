#!/usr/bin/env python
"""Benchmark of the SPTS prefill layer on B200 (tokens/s per layer, % of roofline).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one pass of the whole hot path over one batch of synthetic input:
for the layer workloads a full SPTS layer (norm, K/V/Q projections, PAP probe
scores, selection, reduced attention, O projection, LTP score, fused
selection, reduced FFN); for ``msdp_32k`` the eight-layer MSDP pipeline with
its four stage prunes.  Each step runs in place on the previous step's
residual stream, so inputs stay resident in HBM; every input (h: 512 MB at
32K, weights: 436 MB) is larger than L2, so no L2 flush is needed.

Multi-GPU: the path does not shard inside one sequence, so N GPUs run N
independent replicas (weak scaling, no data-path collective); the timed
region is bracketed by barriers and the time is the max over ranks.

The default line (``--workload layer_32k``) also carries the metric's second
configuration, the 128K layer, as its ``layer_128k`` object (``--no-128k``
leaves it out), and a few 32K prefills of the 32-layer Table B schedule with
their TTFT ratio against keep 1.0 as ``llama32_32k`` (``--no-schedule``).  Roofline fractions divide by the burst bf16 peak of
MEASURED_PEAKS.json (the timed regions are short and run at full clock); the
sustained fraction is reported beside it.

``cpu_baseline`` and ``--impl reference`` time the CPU oracle (the only other
implementation of this path) in its fp32 timed mode, one whole layer per
step on every host thread, on rank 0 only.
"""

from __future__ import annotations

import argparse
from dataclasses import replace
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

import numpy as np  # noqa: E402
import torch  # noqa: E402

from synthetic import (FUSE_MAXNORM_ADD, FUSE_MULTIPLY, FUSE_NONE, WORKLOADS, keep_rows, make_hidden,  # noqa: E402
                       make_layer_weights, salient_rows)

METRIC = "prefill tokens/s per SPTS layer at 32K/128K on 1 B200; % of roofline"
FUSE_NAMES = {0: "none", 1: "maxnorm_add", 2: "multiply", 3: "std_add", 4: "sequential"}
DEFAULT_STEPS = {"attn_8k": 100, "layer_32k": 20, "layer_128k": 10, "msdp_32k": 10, "layer_small": 100,
                 "llama32": 5}


def progress(msg):
    """One line per phase on stderr (the JSON line stays alone on stdout)."""
    print(f"bench [{time.strftime('%H:%M:%S')}] {msg}", file=sys.stderr, flush=True)


# ---------------------------------------------------------------- peaks
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------- algorithmic work
def layer_work(wl, Nc, k, P, idx_attn, ffn=True):
    """Algorithmic FLOPs per stage and HBM bytes of one layer.

    Positions are ascending and unique, so a query at candidate index i sees
    i + 1 keys; attention counts only those (causal) pairs.  The probe is
    counted twice (row statistics, then column sums)."""
    D, Hq, Hkv, d, F, r = wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r
    d_low = wl.ltp_dout or D
    kv_act = bool(wl.kv_active)
    # active-row keys only: the t-th selected query sees the t + 1 selected keys
    vis = k * (k + 1) / 2.0 if kv_act else float(np.sum(idx_attn.astype(np.float64) + 1.0))
    probe_vis = float(sum(Nc - P + p + 1 for p in range(P)))
    fl = {
        "k_proj_rope": 2.0 * Nc * D * Hkv * d,
        "v_proj": 2.0 * (k if kv_act else Nc) * D * Hkv * d,
        "probe_q_proj": 2.0 * P * D * Hq * d,
        "probe_scores": 2.0 * (2.0 * Hq * d * probe_vis),
        "q_proj_rope": 2.0 * k * D * Hq * d,
        "reduced_attention": 4.0 * Hq * d * vis,
        "o_proj_scatter": 2.0 * k * Hq * d * D,
    }
    if ffn:
        fl.update({"ltp_scores": 2.0 * Nc * (D * r + r * d_low), "gate_up_swiglu": 4.0 * k * D * F,
                   "down_proj_scatter": 2.0 * k * F * D})
    w_bytes = 2.0 * (D * Hq * d * 2 + D * Hkv * d * 2 + (3 * D * F + D * r + r * d_low if ffn else 0))
    kv_rows = (Nc + 2 * k) if kv_act else 2 * Nc             # K (+ gathered K_sel and V_sel) or K and V
    act_bytes = (Nc * D * 4 * 2 * (2 if ffn else 1)          # h read by each norm, written back
                 + Nc * D * 2 * 2 * (2 if ffn else 1)        # normed rows written and read
                 + kv_rows * Hkv * d * 2 * 2                 # K, V written and read
                 + k * Hq * d * 2 * 4                        # Q_sel and O_sel written and read
                 + (k * F * 2 * 2 if ffn else 0))            # SwiGLU activation written and read
    return fl, w_bytes + act_bytes


# ---------------------------------------------------------------- ranks
def max_over_ranks(value, device):
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, ms_max):
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (ms_max / 1000.0)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and throttle reasons while the timed region runs.

    NVML is polled every 10 ms from a thread (read-only queries), so that a
    timed region of ~0.1 s still gets about ten samples; where NVML cannot be
    loaded, nvidia-smi polls every 100 ms instead."""
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    # NVML clock event reason bits, in the order of NAMES
    BITS = (0x8, 0x40, 0x20, 0x4)
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, dev, period_s=0.01):
        import threading
        self.proc = self.thread = None
        self.samples = []                       # (sm MHz, max MHz, set of reasons)
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            mx = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.stop_evt = threading.Event()

            def poll():
                while not self.stop_evt.is_set():
                    try:
                        sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        r = int(reasons(h))
                        self.samples.append((sm, mx, {n for n, b in zip(self.NAMES, self.BITS) if r & b}))
                    except Exception:
                        pass
                    self.stop_evt.wait(period_s)

            self.source = f"NVML every {int(period_s * 1000)} ms"
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        self.out = tempfile.TemporaryFile(mode="w+")
        self.source = "nvidia-smi every 100 ms"
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def _smi_samples(self):
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.seek(0)
        for line in self.out.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm, mx = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            self.samples.append((sm, mx, {n for n, v in zip(self.NAMES, parts[3:7])
                                          if v.lower().startswith("active")}))

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
        elif self.proc is not None:
            self._smi_samples()
        else:
            return None
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        reasons = set().union(*(r for _, _, r in self.samples))
        return {"sm_mhz": statistics.median(s for s, _, _ in self.samples),
                "sm_max_mhz": max(m for _, m, _ in self.samples), "reasons": sorted(reasons),
                "samples": len(self.samples), "source": self.source}


# ---------------------------------------------------------------- the GPU arm
class LayerCase:
    """Inputs and weights of one layer workload, resident on the GPU."""

    def __init__(self, S, wl, dev, layer=0):
        self.S, self.wl = S, wl
        self.h0 = make_hidden(wl).to(dev)
        self.W = {n: t.to(dev) for n, t in make_layer_weights(wl, layer).items()}
        self.pos = torch.arange(wl.N, dtype=torch.int32, device=dev)
        self.sal = salient_rows(wl.N, wl.P, wl.salient_frac, wl.seed).to(dev)
        self.weights = S.layer_weights(self.W)

    def desc(self, k=None):
        wl = self.wl
        return self.S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, wl.k if k is None else k,
                                 fuse=wl.fuse, salient_rows=self.sal if len(self.sal) else None,
                                 salient_shift=wl.salient_shift, ltp_dout=wl.ltp_dout, ltp_top_m=wl.ltp_top_m, seq_pool=0,
                                 kv_active_only=wl.kv_active)


def run_msdp_step(S, wl, h, pos, layers, desc):
    """The MSDP pipeline (stages of two layers, pruning at each boundary) in
    one C-ABI call; h and pos are compacted in place."""
    ks = [keep_rows(r, wl.N) for r in wl.ratios]
    S.spts_msdp_forward(h, pos, desc, layers, 2, ks)
    return h



# The committed ncu summary of each kernel that can dominate a layer, and the
# source file it was captured from.
PROFILED = {"reduced_attention": ("attention_bf16", "attn.cu")}


def captured_traffic(workload: str, kernel: str):
    """DRAM bytes (read + write) per launch of ``kernel``, from the committed
    ncu summary of that kernel on this workload, or None when there is no
    capture for it or the kernel source changed since the capture (the
    summary records a sha256 prefix of the source file)."""
    import hashlib
    import re
    if kernel not in PROFILED:
        return None
    prefix, src_name = PROFILED[kernel]
    summary = os.path.join(ROOT, "profiles", f"{prefix}_{workload}.md")
    src = os.path.join(ROOT, "token_skipping_sparse_b200", "csrc", src_name)
    if not (os.path.exists(summary) and os.path.exists(src)):
        return None
    text = open(summary).read()
    sha = re.search(r"sha256 prefix\s*`([0-9a-f]{16})`", text)
    dram = re.search(r"DRAM read / write per launch \| ([0-9.]+) MB / ([0-9.]+) MB", text)
    if not (sha and dram):
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != sha.group(1):
        return None
    return round((float(dram.group(1)) + float(dram.group(2))) * 1e6)


def layer_config(wl, k, world):
    """The ``config`` object of a layer workload's line (both arms)."""
    return {"workload": wl.name, "N": wl.N, "keep": wl.keep, "k": int(k), "P": wl.P, "Hq": wl.Hq, "Hkv": wl.Hkv,
            "d_head": wl.d, "D": wl.D, "F": wl.F, "ltp_rank": wl.r, "fuse": FUSE_NAMES[wl.fuse],
            "layers_per_step": wl.layers if wl.ratios else 1, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (no flush)", "input": "each step runs on the previous step's output"}


def measure_layer(S, wl, args, rank, world, dev, peaks, e2e=True):
    """Times one layer workload (or the MSDP pipeline) on this rank's GPU:
    the timed region, the dominant kernel inside it, the per-stage split,
    keep 1.0 with the same kernels and the end-to-end rate with host buffers."""
    torch.manual_seed(0)
    msdp = bool(wl.ratios)
    if msdp:
        base = LayerCase(S, wl, dev, 0)
        layer_tensors = [{n: t.to(dev) for n, t in make_layer_weights(wl, i).items()} for i in range(wl.layers)]
        keep_alive = [base, layer_tensors]
        mdesc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, 0, fuse=wl.fuse)
        pos_buf = torch.empty_like(base.pos)

        def step(h, evs=None):
            pos_buf.copy_(base.pos)        # the pipeline compacts positions in place
            return run_msdp_step(S, wl, h, pos_buf, layer_tensors, mdesc)
    else:
        case = LayerCase(S, wl, dev)
        desc = case.desc()
        keep_alive = [case]

        def step(h, evs=None):
            S.spts_layer_forward(h, case.pos, desc, case.weights, events=evs)
            return h

    progress(f"{wl.name}: inputs on the device; {args.warmup} warm-up steps")
    h = (base if msdp else case).h0.clone()
    for _ in range(args.warmup):
        step(h if not msdp else (base.h0.clone()))
    torch.cuda.synchronize()
    S.check_device_status()
    progress(f"{wl.name}: staged passes")

    # ---------------- per-stage breakdown (one layer) and the dominant kernel
    lcase = base if msdp else case
    ldesc = (S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, keep_rows(wl.ratios[0], wl.N), fuse=wl.fuse)
             if msdp else desc)
    hb = lcase.h0.clone()
    idx = torch.empty(ldesc.k, dtype=torch.int32, device=dev)
    evs = S.stage_events()
    S.spts_layer_forward(hb, lcase.pos, ldesc, lcase.weights, outputs={"idx_attn": idx}, events=evs)
    # per-stage median of several staged passes (every kernel on one stream,
    # an event between stages); for the pipeline, of its first layer shape
    reps = 9
    per_rep = []
    for _ in range(reps):
        S.spts_layer_forward(hb, lcase.pos, ldesc, lcase.weights, events=evs)
        torch.cuda.synchronize()
        per_rep.append([evs[i].elapsed_time(evs[i + 1]) for i in range(len(S.LAYER_STAGES))])
    stage_ms = np.median(np.array(per_rep), axis=0)
    del hb
    ffn = wl.F > 0
    fl, nbytes = layer_work(wl, wl.N, ldesc.k, wl.P, idx.cpu().numpy(), ffn)
    kernel_stages = ["k_proj_rope", "v_proj", "q_proj_rope", "reduced_attention", "o_proj_scatter", "ltp_scores",
                     "gate_up_swiglu", "down_proj_scatter"]
    by_name = dict(zip(S.LAYER_STAGES, stage_ms))
    dom = max((s for s in kernel_stages if s in fl), key=lambda s: by_name[s])
    dom_i = S.LAYER_STAGES.index(dom)
    # The dominant kernel is timed again inside the timed region: in every
    # timed step, events on the layer's stream right before and after it
    # (events past the side stream's join, so the production path is kept).
    live = not msdp and dom_i >= 8
    torch.cuda.synchronize()

    # ---------------- timed region
    progress(f"{wl.name}: timed region, {args.steps} steps")
    steps = args.steps
    inputs = [base.h0.clone() for _ in range(1)] if msdp else None
    timed_evs = [None] * steps
    if live:
        for i in range(steps):
            pair = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            for e in pair:  # torch creates the CUDA event at its first record
                e.record()
            timed_evs[i] = [None] * S.LAYER_STAGE_EVENTS
            timed_evs[i][dom_i], timed_evs[i][dom_i + 1] = pair
    sampler = ClockSampler(dev) if rank == 0 else None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    n0 = S.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(h if not msdp else inputs[0], timed_evs[i])
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    launches = S.launch_count() - n0
    clocks = sampler.stop() if sampler else None
    ms_total = max_over_ranks(e0.elapsed_time(e1), dev)
    S.check_device_status()
    ms_step = ms_total / steps
    layers_per_step = wl.layers if msdp else 1
    value = job_throughput(wl.N * layers_per_step * steps, world, ms_total)

    if live:
        dom_ms = float(np.mean([ev[dom_i].elapsed_time(ev[dom_i + 1]) for ev in timed_evs]))
        dom_timing = "CUDA events around the kernel in every timed step, mean"
    else:
        dom_ms = by_name[dom]
        dom_timing = "staged passes of the first layer shape (the pipeline's kernels are not evented), median"
    achieved = fl[dom] / (dom_ms / 1e3) / 1e12
    layer_flops = sum(fl.values())
    if msdp:
        # average layer of the pipeline: each stage's two layers at (|C_s|, k_s); the
        # selected rows of later stages are taken as evenly spread over C_s
        tot_f, tot_b, Nc = 0.0, 0.0, wl.N
        for r_ in wl.ratios:
            k_s = keep_rows(r_, wl.N)
            f_s, b_s = layer_work(wl, Nc, k_s, wl.P, np.linspace(0, Nc - 1, k_s).astype(np.int64), ffn)
            tot_f += 2 * sum(f_s.values())
            tot_b += 2 * b_s
            Nc = k_s
        layer_flops, nbytes = tot_f / wl.layers, tot_b / wl.layers
    ms_layer = ms_step / layers_per_step
    t_roof = {name: max(layer_flops / (peaks[key] * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9)) * 1e3
              for name, key in (("burst", "bf16"), ("sustained", "bf16_sustained"))}

    # ---------------- skipped-prefill speedup over the same kernels at keep 1.0
    progress(f"{wl.name}: timed {ms_step:.3f} ms per step; keep 1.0 and end to end")
    dense = None
    if not msdp and not args.no_dense:
        ddesc = lcase.desc(k=wl.N)
        hd = lcase.h0.clone()
        S.spts_layer_forward(hd, lcase.pos, ddesc, lcase.weights)
        torch.cuda.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        nd = 3
        d0.record()
        for _ in range(nd):
            S.spts_layer_forward(hd, lcase.pos, ddesc, lcase.weights)
        d1.record()
        torch.cuda.synchronize()
        dense_ms = max_over_ranks(d0.elapsed_time(d1) / nd, dev)
        dense = {"keep": 1.0, "ms_per_layer": round(dense_ms, 4),
                 "speedup_of_skipping": round(dense_ms / ms_layer, 3)}
        del hd

    # ---------------- end to end through the C ABI with host buffers
    e2e_res = e2e_f32 = None
    if not msdp and e2e:
        def run_e2e(io_bf16):
            # Consecutive steps are pipelined the way a caller streaming
            # sequences would run them: NBUF device buffers, the H2D copy, the
            # layer call and the D2H copy on three streams, so step i's copies
            # overlap the neighbouring steps' compute (PCIe runs both
            # directions at once).  Every step moves its own input in and its
            # result out.  io_bf16: the residual crosses the boundary in bf16
            # (spts_layer_forward_bf16io), else in fp32 (spts_layer_forward).
            # The timed region covers the same K steps as the device timing,
            # from the first step's H2D to the last step's D2H.
            dt = torch.bfloat16 if io_bf16 else torch.float32
            hh = lcase.h0.to(dt).cpu().pin_memory()
            ho = torch.empty_like(hh).pin_memory()
            NBUF = 3
            ne = steps
            dbuf = [torch.empty_like(lcase.h0, dtype=dt) for _ in range(NBUF)]
            s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
            ev_in = [torch.cuda.Event() for _ in range(NBUF)]
            ev_done = [torch.cuda.Event() for _ in range(NBUF)]
            ev_free = [torch.cuda.Event() for _ in range(NBUF)]
            call = S.spts_layer_forward_bf16io if io_bf16 else S.spts_layer_forward

            def pipelined(n):
                for i in range(n):
                    b = i % NBUF
                    if i >= NBUF:
                        s_in.wait_event(ev_free[b])        # the buffer's previous result is out
                    with torch.cuda.stream(s_in):
                        dbuf[b].copy_(hh, non_blocking=True)
                        ev_in[b].record(s_in)
                    s_cmp.wait_event(ev_in[b])
                    with torch.cuda.stream(s_cmp):
                        call(dbuf[b], lcase.pos, desc, lcase.weights)
                        ev_done[b].record(s_cmp)
                    s_out.wait_event(ev_done[b])
                    with torch.cuda.stream(s_out):
                        ho.copy_(dbuf[b], non_blocking=True)
                        ev_free[b].record(s_out)

            pipelined(NBUF)
            torch.cuda.synchronize()
            x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            x0.record(s_in)
            pipelined(ne)
            x1.record(s_out)                              # after the last step's D2H
            torch.cuda.synchronize()
            e_ms = max_over_ranks(x0.elapsed_time(x1) / ne, dev)
            nbh = hh.numel() * hh.element_size()
            return {"value": round(wl.N * world / (e_ms / 1e3), 1), "unit": "tokens/s", "h2d_bytes_per_step": nbh,
                    "d2h_bytes_per_step": nbh, "ms_per_step": round(e_ms, 4),
                    "boundary": ("bf16 residual (spts_layer_forward_bf16io: fp32 inside, changed rows rounded "
                                 "back to bf16)") if io_bf16 else "fp32 residual (spts_layer_forward)",
                    "pipeline": f"{NBUF} device buffers; H2D, layer call and D2H on separate streams, overlapping "
                                "across consecutive steps"}

        e2e_res = run_e2e(True)
        e2e_f32 = run_e2e(False)

    traffic = captured_traffic(wl.name, dom)
    out = {
        "value": round(value, 1), "unit": "tokens/s", "steps": steps, "ms_per_step": round(ms_step, 4),
        "config": layer_config(wl, ldesc.k, world),
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 1), "peak": peaks["bf16"],
                     "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16"], 4),
                     "traffic": traffic, "algorithmic_flops": fl[dom], "ms": round(dom_ms, 4), "timing": dom_timing,
                     "peak_note": f"{peaks['source']} burst bf16 (cuBLAS 8192^3, best of 10): the timed region is "
                                  "short and runs at full clock; the sustained figure is given beside it",
                     "peak_sustained": peaks["bf16_sustained"],
                     "frac_sustained": round(achieved / peaks["bf16_sustained"], 4)},
        "layer_roofline": {"flops": layer_flops, "hbm_bytes": nbytes, "t_roof_ms": round(t_roof["burst"], 4),
                           "ms_measured": round(ms_layer, 4), "frac": round(t_roof["burst"] / ms_layer, 4),
                           "peak_tflops": peaks["bf16"], "peak_hbm_gbs": peaks["hbm_gbs"],
                           "frac_sustained": round(t_roof["sustained"] / ms_layer, 4),
                           "note": "t_roof = max(flops / bf16 peak, bytes / HBM peak); frac = t_roof / measured"},
        "stages_ms": {k: round(v, 4) for k, v in by_name.items()},
        "stages_timing": "9 staged passes before the timed region, one stream, median",
        "gpu_launches": int(launches),
        "clocks": clocks,
        "e2e": e2e_res,
        "e2e_fp32_boundary": e2e_f32,
        "dense_keep1": dense,
    }
    del keep_alive
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def gpu_arm(args, rank, world, dev):
    import token_skipping_sparse_b200 as S

    wl = WORKLOADS[args.workload]
    peaks = measured_peaks()
    res = measure_layer(S, wl, args, rank, world, dev, peaks, e2e=not args.no_e2e)
    result = {"metric": METRIC, "value": res.pop("value"), "unit": res.pop("unit"), "n_gpus": world,
              "steps": res.pop("steps"), "warmup": args.warmup, "ms_per_step": res.pop("ms_per_step"),
              "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
              "data": "synthetic (seeded N(0,1) hidden states, N(0,0.02) weights)"}
    result.update(res)
    # the metric's second configuration, in the same line
    if args.workload == "layer_32k" and not args.no_128k:
        sub = measure_layer(S, WORKLOADS["layer_128k"], args, rank, world, dev, peaks, e2e=not args.no_e2e)
        result["layer_128k"] = sub
    # the 32-layer Table B schedule at 32K (a few prefills): TTFT against keep 1.0
    if args.workload == "layer_32k" and not args.no_schedule:
        progress("llama32_32k: the 32-layer schedule")
        sargs = argparse.Namespace(**{**vars(args), "workload": "llama32_32k", "steps": 3, "warmup": 1})
        sch = schedule_arm(sargs, rank, world, dev)
        jac = [j["jaccard"] for j in sch["jaccard_consecutive"]]
        result["llama32_32k"] = {
            "what": "32 LLaMA-shaped layers under the Table B schedule, one step = one 32K prefill",
            "steps": sch["steps"], "warmup": sch["warmup"], "ttft_ms": sch["ttft_ms"],
            "ttft_ratio_vs_keep1": sch["ttft_ratio_vs_keep1"], "value": sch["value"], "unit": sch["unit"],
            "roofline_frac": sch["roofline"]["frac"], "layer_roofline_frac": sch["layer_roofline"]["frac"],
            "jaccard_consecutive_mean": round(float(np.mean(jac)), 4) if jac else None,
            "jaccard_consecutive_min": round(float(np.min(jac)), 4) if jac else None,
            "rows_after_prefill": sch["rows_after_prefill"], "gpu_launches": sch["gpu_launches"],
            "clocks": sch["clocks"]}
        torch.cuda.empty_cache()
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        progress("cpu_baseline: one whole layer through the oracle's timed mode")
        result["cpu_baseline"] = cpu_baseline(wl)
    progress("done")
    return result


# ---------------------------------------------------------------- the oracle, timed on the host
def timed_case(wl):
    """Host inputs of the oracle's fp32 timed mode for one layer of ``wl``:
    the same seeded arrays the GPU gets.  For the MSDP pipeline: the first
    layer of stage 1 (all N candidates, k_1 active rows)."""
    k = keep_rows(wl.ratios[0], wl.N) if wl.ratios else wl.k
    h = make_hidden(wl)
    W = {n: t.float() for n, t in make_layer_weights(wl).items()}
    sal = salient_rows(wl.N, wl.P, wl.salient_frac, wl.seed).long()
    return k, h, W, sal, torch.arange(wl.N)


def timed_supported(wl):
    return (not wl.kv_active and not wl.ltp_top_m and not wl.ltp_dout
            and wl.fuse in (FUSE_NONE, FUSE_MAXNORM_ADD, FUSE_MULTIPLY))


def time_oracle_layer(wl, case):
    """Seconds of one whole layer through oracle/timed.py on every host thread."""
    from oracle import timed as T
    k, h, W, sal, pos = case
    t0 = time.perf_counter()
    T.layer_forward(h, pos, W, wl.Hq, wl.Hkv, wl.P, k, wl.fuse, salient_rows=sal, salient_shift=wl.salient_shift,
                    ffn=wl.F > 0)
    return time.perf_counter() - t0


def cpu_baseline(wl):
    """The oracle timed on the host cores: one whole layer of the workload
    (every row, every step of the layer), measured, not scaled."""
    if not timed_supported(wl):
        return {"kind": "oracle", "unavailable": f"{wl.name}: the oracle's timed mode covers the MaxNorm-Add / "
                                                 "Multiply layers (and the attention-only layer) with the L2 "
                                                 "proxy score and all-candidate keys"}
    case = timed_case(wl)
    dt = time_oracle_layer(wl, case)
    threads = torch.get_num_threads()
    what = ("the first layer of MSDP stage 1" if wl.ratios else
            "one attention-only layer (no FFN)" if wl.F == 0 else "one whole layer")
    return {"value": round(wl.N / dt, 2), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{wl.name}: {what} (N = {wl.N} rows, k = {case[0]}), every step in full, through the "
                      f"oracle's fp32 timed mode (oracle/timed.py: plain torch CPU ops) on {threads} host threads; "
                      "measured once, not scaled",
            "seconds": round(dt, 3)}


def schedule_layers(wl):
    """(Nc, k, skipping) of every layer of a Table-B schedule workload."""
    first_skip, ends, budgets, after = wl.schedule
    out, Nc, stage = [], wl.N, 0
    for layer in range(wl.layers):
        skip = layer >= first_skip and stage < len(ends) and layer <= ends[stage]
        k = min(budgets[stage], Nc) if skip else Nc
        out.append((Nc, k, skip))
        if skip and layer == ends[stage]:
            Nc = min(budgets[stage] if stage + 1 < len(ends) else after, Nc)
            stage += 1
    return out


def schedule_arm(args, rank, world, dev):
    """A 32-layer prefill under the Table-B schedule (one step = one full
    prefill of N tokens), its keep-1.0 counterpart (the same layers, every
    token in every layer) for the TTFT ratio, and the Jaccard index of the
    attention sets of consecutive skipping layers (Fig. 3(d))."""
    import token_skipping_sparse_b200 as S

    wl = WORKLOADS[args.workload]
    peaks = measured_peaks()
    first_skip, ends, budgets, after = wl.schedule
    h0 = make_hidden(wl).to(dev)
    pos0 = torch.arange(wl.N, dtype=torch.int32, device=dev)
    Ws = [make_layer_weights(wl, i, device=dev) for i in range(wl.layers)]
    desc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, 0, fuse=wl.fuse, ltp_dout=wl.ltp_dout,
                        kv_active_only=wl.kv_active, ltp_top_m=wl.ltp_top_m)
    ws = S.workspace(S.lib.spts_schedule_forward_workspace(S.C.byref(desc), wl.N))
    h = torch.empty_like(h0)
    pos = torch.empty_like(pos0)

    def step():
        h.copy_(h0)
        pos.copy_(pos0)                   # the schedule compacts h and pos in place
        return S.spts_schedule_forward(h, pos, desc, Ws, first_skip, ends, budgets, after, ws=ws)

    def timed(fn, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(n):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    S.check_device_status(ws)
    sampler = ClockSampler(dev) if rank == 0 else None
    if world > 1:
        torch.distributed.barrier()
    n0 = S.launch_count()
    ms_local = timed(step, args.steps)
    launches = S.launch_count() - n0
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    ms_step = max_over_ranks(ms_local, dev)
    S.check_device_status(ws)
    n_left = step()

    # keep 1.0: the same 32 layers with every token active in every layer
    ddesc = S.layer_desc(wl.D, wl.Hq, wl.Hkv, wl.d, wl.F, wl.r, wl.P, wl.N, fuse=wl.fuse, ltp_dout=wl.ltp_dout,
                         ltp_top_m=wl.ltp_top_m)
    dws = S.workspace(S.lib.spts_layer_forward_workspace(S.C.byref(ddesc), wl.N))
    dW = [S.layer_weights(W) for W in Ws]

    def dense_step():
        h.copy_(h0)
        for W in dW:
            S.lib.spts_layer_forward(S.C.byref(ddesc), S.C.byref(W), h.data_ptr(), pos0.data_ptr(), wl.N, None,
                                     dws.data_ptr(), dws.numel(), S.stream_ptr())

    dense_step()
    S.check_device_status(dws)
    ms_dense = max_over_ranks(timed(dense_step, max(1, min(args.steps, 3))), dev)

    # Fig. 3(d): Jaccard index of consecutive skipping layers' attention sets
    n_sel, sel = S.spts_schedule_forward(h.copy_(h0), pos.copy_(pos0), desc, Ws, first_skip, ends, budgets, after,
                                         selections=True, ws=ws)
    torch.cuda.synchronize()
    sets = [None if x is None else set(x.cpu().numpy().tolist()) for x in sel]
    jac = []
    for layer in range(1, wl.layers):
        a, b = sets[layer - 1], sets[layer]
        if a is not None and b is not None:
            jac.append({"layers": [layer - 1, layer], "jaccard": round(len(a & b) / len(a | b), 4)})

    # algorithmic work of the whole prefill: every layer at its own (Nc, k)
    tot_f = tot_b = 0.0
    for Nc, k, skip in schedule_layers(wl):
        lw = wl if skip else replace(wl, kv_active=False)
        f_l, b_l = layer_work(lw, Nc, k, wl.P, np.arange(Nc - k, Nc) if not skip else np.arange(k), True)
        if not skip:  # full layers run no probe, LTP or selection
            for name in ("probe_q_proj", "probe_scores", "ltp_scores"):
                f_l.pop(name, None)
        tot_f += sum(f_l.values())
        tot_b += b_l
    t_roof_ms = max(tot_f / (peaks["bf16"] * 1e12), tot_b / (peaks["hbm_gbs"] * 1e9)) * 1e3
    achieved = tot_f / (ms_step / 1e3) / 1e12
    return {
        "metric": "prefill tokens/s of the 32-layer Table-B schedule on 1 B200; TTFT ratio vs keep 1.0",
        "value": round(job_throughput(wl.N * args.steps, world, ms_step * args.steps), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) hidden states, N(0,0.02) weights drawn on the GPU)",
        "config": {"workload": wl.name, "N": wl.N, "layers": wl.layers, "first_skip": first_skip,
                   "stage_ends": list(ends), "budgets": list(budgets), "after_last": after, "P": wl.P,
                   "fuse": "multiply", "ltp_dout": wl.ltp_dout, "ltp_top_m": wl.ltp_top_m,
                   "kv_active_only": bool(wl.kv_active), "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (no flush)"},
        "roofline": {"bound": "tensor", "kernel": "whole prefill (all kernels)", "achieved": round(achieved, 1),
                     "peak": peaks["bf16"], "unit": "TFLOP/s",
                     "frac": round(achieved / peaks["bf16"], 4), "traffic": None,
                     "peak_note": f"{peaks['source']} burst bf16",
                     "frac_sustained": round(achieved / peaks["bf16_sustained"], 4)},
        "layer_roofline": {"flops": tot_f, "hbm_bytes": tot_b, "t_roof_ms": round(t_roof_ms, 3),
                           "ms_measured": round(ms_step, 3), "frac": round(t_roof_ms / ms_step, 4)},
        "ttft_ms": {"schedule": round(ms_step, 3), "keep_1": round(ms_dense, 3)},
        "ttft_ratio_vs_keep1": round(ms_dense / ms_step, 3),
        "rows_after_prefill": int(n_left),
        "jaccard_consecutive": jac,
        "gpu_launches": int(launches),
        "clocks": clocks,
    }


def attention_arm(args, rank, world, dev):
    """spts_reduced_attention alone on a workload's shapes: seeded bf16
    N(0,1) Q/K/V, positions 0..N-1, the selected rows a seeded random subset
    with the last P kept.  For profiling one kernel at a size that holds about
    a gigabyte on the device (the whole 128K layer holds several)."""
    import token_skipping_sparse_b200 as S
    wl = WORKLOADS[args.workload]
    peaks = measured_peaks()
    g = torch.Generator().manual_seed(wl.seed + 11)
    k = wl.k
    sel = torch.cat([torch.sort(torch.randperm(wl.N - wl.P, generator=g)[:k - wl.P]).values,
                     torch.arange(wl.N - wl.P, wl.N)]).to(torch.int32)
    q = torch.randn(k, wl.Hq, wl.d, generator=g).to(torch.bfloat16).to(dev)
    kk = torch.randn(wl.N, wl.Hkv, wl.d, generator=g).to(torch.bfloat16).to(dev)
    vv = torch.randn(wl.N, wl.Hkv, wl.d, generator=g).to(torch.bfloat16).to(dev)
    pos = torch.arange(wl.N, dtype=torch.int32, device=dev)
    qpos = sel.to(dev)
    o = torch.empty_like(q)
    for _ in range(args.warmup):
        S.spts_reduced_attention(q, qpos, kk, vv, pos, out=o)
    torch.cuda.synchronize()
    S.check_device_status()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        S.spts_reduced_attention(q, qpos, kk, vv, pos, out=o)
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    flops = 4.0 * wl.Hq * wl.d * float((sel.to(torch.float64) + 1.0).sum())
    ach = flops / (ms / 1e3) / 1e12
    return {"metric": "reduced attention TFLOP/s (kernel alone)", "value": round(ach, 1), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) Q/K/V, random selection)",
            "config": {"workload": wl.name, "kernel": "reduced_attention", "N": wl.N, "k": k, "Hq": wl.Hq,
                       "Hkv": wl.Hkv, "d_head": wl.d},
            "roofline": {"bound": "tensor", "achieved": round(ach, 1), "peak": peaks["bf16"], "unit": "TFLOP/s",
                         "frac": round(ach / peaks["bf16"], 4), "traffic": None}}


# Free candidates above which spts_select_topk runs on the grid (given a
# workspace); the library's own threshold, checked against its source in the
# host tests.
TOPK_GRID_MIN = 20480


def topk_arm(args, rank, world, dev):
    """spts_select_topk alone on a workload's candidate count: the FFN-set
    selection of the layer (MaxNorm-Add fusion of two seeded positive score
    vectors, k of them kept with the last P forced, the fused scores written
    out).  Up to 20K free candidates one CTA runs it, above that the grid
    path.  The calls are queued behind a sleep kernel so that the timed
    region holds their device time back to back, not the host's time to
    issue them (a few microseconds of kernels per call)."""
    import token_skipping_sparse_b200 as S
    wl = WORKLOADS[args.workload]
    peaks = measured_peaks()
    g = torch.Generator().manual_seed(wl.seed + 12)
    N, k = wl.N, wl.k
    s_a = -torch.log1p(-torch.rand(N, generator=g)) * (wl.P * wl.Hq / N)   # sums to about P·Hq, like PAP scores
    s_b = 26.0 + 2.0 * torch.randn(N, generator=g)                           # LTP row norms at these inits
    s_a, s_b = s_a.float().to(dev), s_b.abs().float().to(dev)
    ws = S.workspace(int(S.lib.spts_select_topk_workspace(N)))
    call = lambda: S.spts_select_topk(s_a, k, wl.P, s_b=s_b, mode=FUSE_MAXNORM_ADD, fused=True, ws=ws)  # noqa: E731
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    S.check_device_status()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(20_000_000)       # ~10 ms of device time while the calls are queued behind it
    e0.record()
    for _ in range(args.steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    nbytes = 3 * N * 4 + k * 4           # two score vectors read, the fused scores and k indices written
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"metric": "top-k selection time (kernel alone)", "value": round(ms * 1e3, 2), "unit": "us",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded exponential and |N(26, 2)| score vectors)",
            "config": {"workload": wl.name, "kernel": "select_topk", "Nc": N, "k": k, "force_tail": wl.P,
                       "fuse": "maxnorm_add", "path": "grid" if N - wl.P > TOPK_GRID_MIN else "one CTA"},
            "roofline": {"bound": "latency", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 5), "traffic": None,
                         "note": f"{nbytes / 1e6:.2f} MB per call: far below what HBM time would matter for; the "
                                 "call is bound by its passes' latency (launches, block-wide scans)"}}


def reference_arm(args):
    """The oracle (fp32 timed mode) on the host cores: one whole layer per
    step, on the GPU arm's workload, config, metric and unit."""
    wl = WORKLOADS[args.workload]
    if wl.schedule or not timed_supported(wl):
        return {"impl": "reference", "workload": wl.name,
                "unavailable": f"{wl.name}: outside the oracle's timed mode (a 32-layer schedule, or a scoring variant "
                               "it does not cover); parity against the oracle is tested at small and sampled sizes"}
    case = timed_case(wl)
    for _ in range(args.warmup):
        time_oracle_layer(wl, case)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time_oracle_layer(wl, case)
    wall = time.perf_counter() - t0
    ms = 1000.0 * wall / args.steps
    v = round(wl.N / (ms / 1000.0), 2)
    threads = torch.get_num_threads()
    what = ("the first layer of MSDP stage 1" if wl.ratios else
            "one attention-only layer (no FFN)" if wl.F == 0 else "one whole layer")
    cb = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
          "sample": f"{wl.name}: {what} per step (N = {wl.N}, k = {case[0]}), every step of the layer in full, "
                    f"through the oracle's fp32 timed mode on {threads} host threads; not scaled",
          "seconds": round(ms / 1000.0, 3)}
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": layer_config(wl, case[0], args.gpus), "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="layer_32k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-128k", action="store_true", help="time only the 32K layer in the default line")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffer) measurement")
    ap.add_argument("--no-schedule", action="store_true", help="leave the 32-layer schedule out of the default line")
    ap.add_argument("--kernel", default=None, choices=["attention", "topk"],
                    help="time one kernel alone on the workload's shapes (for profiling)")
    args = ap.parse_args()
    if args.steps is None:
        base = args.workload.rsplit("_", 1)[0]  # a variant takes its base workload's count
        args.steps = (DEFAULT_STEPS.get(args.workload, DEFAULT_STEPS.get(base, 50)) if args.impl == "ours" else 3)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args)), flush=True)
        return 0

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=dev)
    try:
        if args.kernel == "attention":
            res = attention_arm(args, rank, world, dev)
        elif args.kernel == "topk":
            res = topk_arm(args, rank, world, dev)
        elif WORKLOADS[args.workload].schedule:
            res = schedule_arm(args, rank, world, dev)
        else:
            res = gpu_arm(args, rank, world, dev)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
