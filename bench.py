#!/usr/bin/env python
"""Benchmark of the gated delta rule chunked forward on B200.

One step = the whole prefill hot path over one batch of the headline workload
(bf16 q/k/v, B=4, H=16, T=4096, K=V=128, fp32 gates/state/output): the gate
preparation followed by the chunked forward (WY transform, inter-chunk state
recurrence and chunk output in one kernel).  Prints one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun: every rank processes its own batch of the same
shape (independent problems, no data-path collective: weak scaling); the
timed region is bracketed by barriers and the max over ranks is reported.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN chunk-fwd tokens/s (H=16,K=V=128,T=4096) and % of roofline on 1 B200"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def chunk_algorithmic(B, T, H, K, V, n_seq, qkv_bytes=2, o_bytes=4, h0=False, C=64):
    """Algorithmic bytes and FLOPs of one chunked forward: every input and output
    touched once (q, k, v, g, beta in; o, h_T out; h0 in if given); FLOPs of the
    dense per-chunk tiles, 2C(3K+2V) + 6KV per token-head."""
    th = B * T * H
    by = th * ((2 * K + V) * qkv_bytes + 8 + V * o_bytes) + n_seq * H * K * V * 4 * (2 if h0 else 1)
    fl = th * (2 * C * (3 * K + 2 * V) + 6 * K * V)
    return by, fl


def decode_algorithmic(n, M, H, G, P, N):
    """State read + written once, the x and ba rows read once, o written once."""
    by = n * H * N * P * 4 * 2 + n * (M * H * P + M * G * N + G * N) * 2 + n * (M * H + H) * 2 \
        + n * H * P * 2
    fl = n * H * (M * 5 * N * P + 2 * N * P)
    return by, fl


# Sources the tensor-core chunk kernel is built from: a committed ncu summary
# stays valid while these are unchanged.
CHUNK_KERNEL_SOURCES = ("chunk_tc.cuh", "tc_ptx.cuh", "common.cuh", "chunk_simt.cuh")


def kernel_source_sha(files=CHUNK_KERNEL_SOURCES):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_71_b200", "csrc")
    for fn in sorted(files):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(name):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    s = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", txt)
    if not m or not s or s.group(1) != kernel_source_sha():
        return None
    return float(m.group(1))


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while running."""

    BAD = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
           "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
           "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
           "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
           "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.ok = False
        self.samples, self.reasons = [], set()
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = str(e)

    def _handle(self, idx):
        nv = self.nv
        try:
            uuid = str(torch.cuda.get_device_properties(idx).uuid)
            return nv.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
        except Exception:
            pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if ids and idx < len(ids):
            v = ids[idx]
            if v.startswith("GPU-"):
                return nv.nvmlDeviceGetHandleByUUID(v)
            return nv.nvmlDeviceGetHandleByIndex(int(v))
        return nv.nvmlDeviceGetHandleByIndex(idx)

    def _poll(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, attr in self.BAD.items():
                    if r & getattr(nv, attr):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._poll, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, dev) -> float:
    """Max of a per-rank scalar over the process group (nccl: dev is the rank's
    GPU; gloo: a CPU device)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_units(n_units: int, rank: int, world: int):
    """Contiguous, balanced split of n_units independent units over ranks."""
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


# ----------------------------------------------------------- CPU baseline

def cpu_baseline(inp, target_s=12.0):
    """The fp64 oracle, as it stands, on a bounded sample of the workload: whole
    (batch, head) chains over the full sequence, as many as take about target_s
    seconds on all host cores (the whole batch when it is cheaper than that).
    Reported in the workload's tokens/s."""
    import oracle
    q, k, v = inp["q"], inp["k"], inp["v"]
    B, T, H, K = q.shape
    cores = os.cpu_count() or 1
    a, b = inp["a"], inp["b"]
    beta, g = oracle.gate_prep(a, b, inp["A_log"], inp["dt_bias"])
    beta, g = torch.from_numpy(beta), torch.from_numpy(g)
    # calibrate on one short chain
    t0 = time.perf_counter()
    oracle.gdn_fwd(q[:1, :256, :1], k[:1, :256, :1], v[:1, :256, :1], g[:1, :256, :1],
                   beta[:1, :256, :1], n_threads=1)
    per_tokhead = (time.perf_counter() - t0) / 256
    # whole chains over the full sequence, as many as fit the time target
    Ts = T
    want = int(target_s * cores / (T * per_tokhead))
    n_chains = max(min(cores, B * H), min(B * H, want))
    Bs, Hs = (1, n_chains) if n_chains < H else (min(B, -(-n_chains // H)), H)
    sl = lambda x: x[:Bs, :Ts, :Hs].contiguous()
    t0 = time.perf_counter()
    oracle.gdn_fwd(sl(q), sl(k), sl(v), sl(g), sl(beta), n_threads=cores)
    dt = time.perf_counter() - t0
    tok_heads = Bs * Hs * Ts
    return {"value": tok_heads / H / dt, "unit": UNIT, "cores": oracle.last_threads,
            "kind": "oracle",
            "sample": f"fp64 oracle on {Bs * Hs} of {B * H} (batch, head) chains x {Ts} tokens "
                      f"({tok_heads} token-heads, {dt:.1f} s); tokens/s = token-heads/s / H"}


# ---------------------------------------------------- other chunk workloads

def time_chunk_workload(gdn, I, w, dev, stream, world, peaks, src, n_iter=20):
    """Times gdn.chunk_fwd alone on one chunk workload at full size (inputs
    resident in HBM, gates prepared once), with the roofline of its algorithmic
    bytes; the per-call time is the mean over n_iter back-to-back calls."""
    inp = I.chunk_inputs(w)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    B, T, H, K, V = w.B, w.T, w.H, w.K, w.V
    n_seq = w.n_seq_varlen if w.n_seq_varlen else B
    beta, g = gdn.gate_prep(d["a"], d["b"], d["A_log"], d["dt_bias"])
    o = torch.empty(B, T, H, V, device=dev)
    hT = torch.empty(n_seq, H, K, V, device=dev)
    ws = torch.empty(max(1, gdn.chunk_fwd_workspace_size(n_seq, B * T, H, K, V, w.dtype)),
                     dtype=torch.uint8, device=dev)

    def call():
        gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, h0=d["h0"], cu_seqlens=d["cu_seqlens"],
                      out=o, hT=hT, workspace=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n_iter):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / n_iter
    by, fl = chunk_algorithmic(B, T, H, K, V, n_seq, h0=w.h0)
    ach = by / (ms * 1e-3) / 1e9
    lens = None
    if d["cu_seqlens"] is not None:
        cu = inp["cu_seqlens"].tolist()
        lens = [cu[i + 1] - cu[i] for i in range(n_seq)]
    del d, o, hT, ws
    return {"workload": w.name, "metric": "tokens/s", "value": B * T * world / (ms * 1e-3),
            "ms_per_step": ms, "n_seq": n_seq, "lengths": lens, "calls_timed": n_iter,
            "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                         "algorithmic_bytes": by, "algorithmic_flops": fl,
                         "peak_source": src}}


# ------------------------------------------------------------------- ours

def run_ours(args):
    import gated_delta_rule_71_b200 as gdn
    from gated_delta_rule_71_b200 import inputs as I
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = I.BF16_B4_T4096
    inp = I.chunk_inputs(w)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    B, T, H, K, V = w.B, w.T, w.H, w.K, w.V
    stream = torch.cuda.current_stream(dev)
    beta = torch.empty(B, T, H, device=dev)
    g = torch.empty(B, T, H, device=dev)
    o = torch.empty(B, T, H, V, device=dev)
    hT = torch.empty(B, H, K, V, device=dev)

    def step(ev=None):
        gdn.gate_prep(d["a"], d["b"], d["A_log"], d["dt_bias"], beta=beta, g=g)
        if ev is not None:
            ev[0].record(stream)
        gdn.chunk_fwd(d["q"], d["k"], d["v"], g, beta, out=o, hT=hT)
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e0.record(stream)
        for i in range(args.steps):
            step(kev[i])
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps
    k_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in kev) / args.steps, world, dev)
    launches_per_step = 2  # gate_prep + chunk_fwd (dense batch: no schedule kernel)

    by, fl = chunk_algorithmic(B, T, H, K, V, B)
    peaks, src = load_peaks()
    achieved = by / (k_ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": profiled_traffic("chunk_fwd.bf16_B4_H16_T4096.txt"),
            "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs, copy)" if src == "measured"
            else "fallback 6.65 TB/s",
            "kernel": "chunk_fwd", "kernel_ms": round(k_ms, 4),
            "algorithmic_bytes": by, "algorithmic_flops": fl,
            "tensor_tflops": round(fl / (k_ms * 1e-3) / 1e12, 1)}

    if args.headline_only:
        # the headline step alone (for profiler captures: few launches, <1 GB held)
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": B * T * world / (ms * 1e-3), "unit": UNIT,
                              "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                              "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                              "config": {"workload": w.name, "sections": "headline only"},
                              "roofline": roof, "gpu_launches": launches_per_step * args.steps,
                              "clocks": clk.summary()}), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    # --- end to end through the public API with host buffers
    pin = {k: (v.pin_memory() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    o_host = torch.empty(B, T, H, V, pin_memory=True)
    h_host = torch.empty(B, H, K, V, pin_memory=True)
    names = ("q", "k", "v", "a", "b", "A_log", "dt_bias")
    h2d = sum(pin[n].numel() * pin[n].element_size() for n in names)
    d2h = o_host.numel() * 4 + h_host.numel() * 4
    n_e2e = max(3, min(args.steps, 20))

    def e2e_step():
        x = {n: pin[n].to(dev, non_blocking=True) for n in names}
        bt, gt = gdn.gate_prep(x["a"], x["b"], x["A_log"], x["dt_bias"])
        oo, hh = gdn.chunk_fwd(x["q"], x["k"], x["v"], gt, bt)
        o_host.copy_(oo, non_blocking=True)
        h_host.copy_(hh, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    f1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, dev) / n_e2e

    # --- decode step (Gated Delta Product, n=256 M=2 H=32 G=16 P=N=128)
    dw = I.GDP_DECODE
    dd = {k: v.to(dev) for k, v in I.decode_inputs(dw).items()}
    dargs = (dw.M, dw.H, dw.G, dw.P, dw.N)
    od = torch.empty(dw.n, dw.H, dw.P, dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        gdn.gdp_decode_step(dd["x"], dd["ba"], dd["A_log"], dd["dt_bias"], dd["state"], *dargs,
                            out=od)
    n_dec = max(5, args.steps)
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for _ in range(n_dec):
        gdn.gdp_decode_step(dd["x"], dd["ba"], dd["A_log"], dd["dt_bias"], dd["state"], *dargs,
                            out=od)
    d1.record(stream)
    torch.cuda.synchronize()
    dec_ms = max_over_ranks(d0.elapsed_time(d1), world, dev) / n_dec
    dby, dfl = decode_algorithmic(dw.n, *dargs)
    dach = dby / (dec_ms * 1e-3) / 1e9

    # --- the decode token of a layer in one launch (conv update + decode step) against
    # the same two launches apart, on the decode workload with a W=4 SiLU convolution
    Cd = dw.M * dw.H * dw.P + dw.M * dw.G * dw.N + dw.G * dw.N
    lcv = {k: v.to(dev) for k, v in I.conv_decode_inputs(dw.n, Cd, 4, dw.n, seed=1011).items()}
    lx = dd["x"].reshape(dw.n, Cd)
    lba = dd["ba"].reshape(dw.n, -1)
    lws = torch.zeros(gdn.gdp_decode_layer_step_workspace_size(dw.n, dw.G), dtype=torch.uint8,
                      device=dev)
    ly = torch.empty_like(lx)

    def layer_fused():
        gdn.gdp_decode_layer_step(lx, lba, lcv["w"], lcv["conv_state"], dd["A_log"], dd["dt_bias"],
                                  dd["state"], *dargs, conv_bias=lcv["bias"], out=od, workspace=lws)

    def layer_two():
        gdn.conv1d_update(lx, lcv["w"], lcv["conv_state"], lcv["bias"], activation=True, out=ly)
        gdn.gdp_decode_step(ly, lba, dd["A_log"], dd["dt_bias"], dd["state"], *dargs, out=od)

    lay_ms = {}
    for nm, fn in (("fused", layer_fused), ("two_launches", layer_two)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        d0.record(stream)
        for _ in range(n_dec):
            fn()
        d1.record(stream)
        torch.cuda.synchronize()
        lay_ms[nm] = max_over_ranks(d0.elapsed_time(d1), world, dev) / n_dec
    lay_by = dby + dw.n * Cd * 3 * 2 * 2 + Cd * 4 * 4 + Cd * 4
    lay_ach = lay_by / (lay_ms["fused"] * 1e-3) / 1e9

    # --- short convolution (ZzCompute item 1) over the layer's q/k/v channels, and its
    # one-token update at the decode row width
    cw = I.CONV_B4_T4096
    ci = I.conv_inputs(cw)
    cx, cwt, cb = ci["x"].to(dev), ci["w"].to(dev), ci["bias"].to(dev)
    cy = torch.empty_like(cx)
    for _ in range(3):
        gdn.conv1d_fwd(cx, cwt, cb, activation=True, out=cy)
    n_cv = max(5, args.steps)
    torch.cuda.synchronize()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for _ in range(n_cv):
        gdn.conv1d_fwd(cx, cwt, cb, activation=True, out=cy)
    c1.record(stream)
    torch.cuda.synchronize()
    conv_ms = max_over_ranks(c0.elapsed_time(c1), world, dev) / n_cv
    conv_by = 2 * cx.numel() * cx.element_size() + cwt.numel() * 4 + cb.numel() * 4
    conv_ach = conv_by / (conv_ms * 1e-3) / 1e9
    ui = {k: v.to(dev) for k, v in I.conv_decode_inputs(I.CONV_DECODE_N, I.CONV_DECODE_C, cw.W,
                                                        I.CONV_DECODE_N).items()}
    uy = torch.empty_like(ui["x"])
    for _ in range(3):
        gdn.conv1d_update(ui["x"], ui["w"], ui["conv_state"], ui["bias"], activation=True, out=uy)
    torch.cuda.synchronize()
    c0.record(stream)
    for _ in range(n_cv):
        gdn.conv1d_update(ui["x"], ui["w"], ui["conv_state"], ui["bias"], activation=True, out=uy)
    c1.record(stream)
    torch.cuda.synchronize()
    upd_ms = max_over_ranks(c0.elapsed_time(c1), world, dev) / n_cv
    upd_by = (2 * ui["x"].numel() * 2 + 2 * ui["conv_state"].numel() * 2
              + ui["w"].numel() * 4 + ui["bias"].numel() * 4)

    # --- Gated Delta Product prefill: the decode step's heads over a 4096-token prompt
    pw = I.GDP_PREFILL
    pin_ = {k: v.to(dev) for k, v in I.prefill_inputs(pw).items()}
    pargs = (pw.M, pw.H, pw.G, pw.P, pw.N)
    pws = torch.empty(gdn.gdp_prefill_workspace_size(pw.B, pw.B * pw.T, pw.M, pw.H, pw.P, pw.N),
                      dtype=torch.uint8, device=dev)

    def prefill():
        return gdn.gdp_prefill(pin_["x"], pin_["ba"], pin_["A_log"], pin_["dt_bias"], *pargs,
                               workspace=pws)

    for _ in range(3):
        prefill()
    n_pf = max(3, min(args.steps, 20))
    torch.cuda.synchronize()
    c0.record(stream)
    for _ in range(n_pf):
        prefill()
    c1.record(stream)
    torch.cuda.synchronize()
    pf_ms = max_over_ranks(c0.elapsed_time(c1), world, dev) / n_pf
    pf_rows = pw.B * pw.T
    pf_by = (pin_["x"].numel() + pin_["ba"].numel()) * 2 + pf_rows * pw.H * pw.P * 4 \
        + pw.B * pw.H * pw.N * pw.P * 4
    pf_ach = pf_by / (pf_ms * 1e-3) / 1e9

    # --- the packed variable-length batch and the long single sequence, each at full
    # size (their own tokens/s and roofline; not part of the headline step)
    extra = {}
    for key, wl in (("varlen", I.VARLEN_8x32768), ("long", I.LONG_T131072)):
        extra[key] = time_chunk_workload(gdn, I, wl, dev, stream, world, peaks, src,
                                         n_iter=max(3, min(args.steps, 20)))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp)

    if rank == 0:
        tokens = B * T * world
        line = {
            "metric": METRIC, "value": tokens / (ms * 1e-3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "B": B, "T": T, "H": H, "K": K, "V": V, "chunk": 64,
                       "global_batch": B * world, "seq_len": T, "parallelism": f"replica{world}",
                       "step": "gate_prep + chunk_fwd", "qkv": "bf16", "gates_state_o": "fp32",
                       "l2": "inputs exceed L2 (342 MB touched per step > 126 MB)"},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": UNIT, "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "path": "pinned host -> gate_prep -> chunk_fwd -> pinned host (o, h_T)"},
            "gpu_launches": launches_per_step * args.steps,  # timed region of the headline step
            "clocks": clk.summary(),
            "decode": {"workload": dw.name, "metric": "requests/s",
                       "value": dw.n * world / (dec_ms * 1e-3), "ms_per_step": dec_ms,
                       "roofline": {"bound": "hbm", "achieved": round(dach, 1),
                                    "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                    "frac": round(dach / peaks["hbm_gbs"], 4),
                                    "algorithmic_bytes": dby}},
            "decode_layer": {"workload": dw.name + " + conv W4 SiLU", "metric": "requests/s",
                             "value": dw.n * world / (lay_ms["fused"] * 1e-3),
                             "ms_per_step": lay_ms["fused"],
                             "two_launches_ms": lay_ms["two_launches"],
                             "path": "gdp_decode_layer_step (one launch) vs gdn_conv1d_update + "
                                     "gdp_decode_step",
                             "roofline": {"bound": "hbm", "achieved": round(lay_ach, 1),
                                          "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                          "frac": round(lay_ach / peaks["hbm_gbs"], 4),
                                          "algorithmic_bytes": lay_by}},
            "conv1d": {"workload": cw.name, "metric": "tokens/s",
                       "value": cw.B * cw.T * world / (conv_ms * 1e-3), "ms_per_step": conv_ms,
                       "roofline": {"bound": "hbm", "achieved": round(conv_ach, 1),
                                    "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                    "frac": round(conv_ach / peaks["hbm_gbs"], 4),
                                    "algorithmic_bytes": conv_by},
                       "update": {"workload": f"n{I.CONV_DECODE_N} C{I.CONV_DECODE_C} W{cw.W} bf16",
                                  "ms_per_step": upd_ms,
                                  "achieved_gbs": round(upd_by / (upd_ms * 1e-3) / 1e9, 1),
                                  "algorithmic_bytes": upd_by}},
            "varlen": extra["varlen"],
            "long": extra["long"],
            "gdp_prefill": {"workload": pw.name, "metric": "tokens/s",
                            "value": pf_rows * world / (pf_ms * 1e-3), "ms_per_step": pf_ms,
                            "path": "gdp_decode_prepare over the prompt, the chunked kernel over "
                                    "its T*M copies, last-copy gather",
                            "roofline": {"bound": "hbm", "achieved": round(pf_ach, 1),
                                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                         "frac": round(pf_ach / peaks["hbm_gbs"], 4),
                                         "algorithmic_bytes": pf_by}},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------- reference

def run_reference(args):
    """The oracle, as it stands, on the host cores: each step is a bounded sample
    of the headline workload (whole chains, one per core, over a sequence prefix)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from gated_delta_rule_71_b200 import inputs as I
    w = I.BF16_B4_T4096
    inp = I.chunk_inputs(w)
    B, T, H = w.B, w.T, w.H
    cores = os.cpu_count() or 1
    beta, g = oracle.gate_prep(inp["a"], inp["b"], inp["A_log"], inp["dt_bias"])
    beta, g = torch.from_numpy(beta), torch.from_numpy(g)
    heads = min(H, cores)
    Ts = 256
    sl = lambda x: x[:1, :Ts, :heads].contiguous()
    q, k, v, gg, bb = (sl(x) for x in (inp["q"], inp["k"], inp["v"], g, beta))

    def step():
        oracle.gdn_fwd(q, k, v, gg, bb, n_threads=cores)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    val = Ts * heads / H / dt
    sample = (f"fp64 oracle, per step {heads} (batch 0, head) chains x first {Ts} tokens of the "
              f"headline workload; tokens/s = token-heads/s / H")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "B": B, "T": T, "H": H, "K": w.K, "V": w.V, "chunk": 64},
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": oracle.last_threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="time the headline step only (for profiler captures)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
