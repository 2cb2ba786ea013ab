#!/usr/bin/env python
"""Throughput of exact IO-aware attention on B200, one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one GQA training step of attention: forward then backward on
B=1, Hq=32, Hkv=8, N=8192, d=128, causal, bf16, called as a user calls it
(fa_fwd, then fa_bwd: D preprocess, dK/dV, and dQ as a programmatic dependent
of dK/dV); per-kernel durations for the roofline come from a second pass of
the same steps with one entry point per launch.  ``value`` is whole-job
fwd+bwd TFLOP/s with the inputs resident in HBM, FLOPs counted as
4 B Hq Nq Nk d / 2 for the causal forward and 2.5x that for the backward.
The split-KV decode workload (B=64, Hq=32, Hkv=8, Nk_max=32768 with a ragged
second half, d=128, bf16) is timed in the same run and reported as HBM GB/s
under ``decode``.  Every input is synthetic and seeded; each step touches
more bytes than the 126 MB L2 holds, so no explicit flush is done.

Under torchrun (N > 1) every rank runs the same per-GPU workload on its own
GPU (weak scaling; the work shards by (b, h_kv) with no data exchange), the
timed region is bracketed by barriers, and the max over ranks is reported.
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

METRIC = "attention fwd/bwd bf16 TFLOP/s & % of B200 dense peak; decode HBM GB/s"
DENSE_BF16_DATASHEET_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def attn_flops(B, Hq, Nq, Nk, d, causal):
    """Nominal forward FLOPs: two matmuls of 2 FLOPs per multiply-add, halved when causal."""
    f = 4.0 * B * Hq * Nq * Nk * d
    return f * 0.5 if causal else f


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's
    source has not changed since the counters were taken (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        t = json.load(f).get(kernel)
    if not t:
        return None
    try:
        if source_hash(t["sources"]) != t["source_hash"]:
            return None
    except OSError:
        return None
    return t["dram_bytes_per_launch"]


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x10: "sync_boost",
    }

    def __init__(self, index, period=0.01):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period, self._stop = period, threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = get_r(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_init(torch):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(torch, world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(torch, world, x: float, device="cuda") -> float:
    """The slowest rank's value (timings are reported as the max over ranks)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, flops_per_rank, ms_per_step_max):
    """Whole-job TFLOP/s: every rank runs the same per-GPU work (weak scaling)."""
    return world * flops_per_rank / (ms_per_step_max * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args):
    import torch

    import exact_io_aware_80_b200 as fa
    import workloads
    from exact_io_aware_80_b200 import _lib

    world, rank, local = dist_init(torch)
    dev = torch.device("cuda", local)
    _lib.load()
    peaks, peaks_kind = load_peaks()

    w = workloads.get(3)
    if args.seq:
        import dataclasses
        w = dataclasses.replace(w, Nq=args.seq, Nk=args.seq)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.Nq, w.d
    q, k, v, do = workloads.workload_inputs(w, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, N, device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, Hq, N), device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    dt = _lib.FA_BF16
    ptrs = [t.data_ptr() for t in (q, k, v, o, do, lse, dq, dk, dv, ws)]
    bargs = ptrs + [B, Hq, Hkv, N, N, d, 1, w.scale, dt, sh]

    def fwd():
        _lib.fa_fwd(ptrs[0], ptrs[1], ptrs[2], ptrs[3], ptrs[5], B, Hq, Hkv, N, N, d, 1, w.scale, dt, sh)

    def step(ev=None):
        """The training step as a user runs it: fa_fwd, then fa_bwd (preprocess, dK/dV, and dQ
        launched as a programmatic dependent of dK/dV, so it fills the SMs dK/dV's tail frees)."""
        if ev:
            ev[0].record(stream)
        fwd()
        if ev:
            ev[1].record(stream)
        _lib.fa_bwd(*bargs)
        if ev:
            ev[2].record(stream)

    def step_per_kernel(ev):
        """The same launches one entry point at a time, with an event between every two: the
        per-kernel durations behind the roofline (dQ here starts after dK/dV has finished)."""
        ev[0].record(stream)
        fwd()
        ev[1].record(stream)
        _lib.fa_bwd_preprocess(*bargs)
        ev[2].record(stream)
        _lib.fa_bwd_dkdv(*bargs)
        ev[3].record(stream)
        _lib.fa_bwd_dq(*bargs)
        ev[4].record(stream)

    K, W = args.steps, args.warmup
    for _ in range(W):
        step()
    torch.cuda.synchronize(dev)
    if fa.device_status() != 0:
        raise RuntimeError("kernel status word set during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    evk = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(torch, world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        t0.record(stream)
        for i in range(K):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(torch, world)
        # per-kernel pass under the same starting conditions as the timed steps: the GPU idles
        # briefly (its power management recovers from the timed steps), then W warm-up and K
        # measured steps
        time.sleep(0.5)
        for _ in range(W):
            step()
        for i in range(K):
            step_per_kernel(evk[i])
        torch.cuda.synchronize(dev)
    barrier(torch, world)
    ms = t0.elapsed_time(t1)
    ms_max = max_over_ranks(torch, world, ms)
    if fa.device_status() != 0:
        raise RuntimeError("kernel status word set during the timed region")
    fwd_ms_step = statistics.fmean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.fmean(e[1].elapsed_time(e[2]) for e in evs)
    per = {name: statistics.fmean(e[j].elapsed_time(e[j + 1]) for e in evk)
           for j, name in enumerate(("fwd", "bwd_preprocess", "bwd_dkdv", "bwd_dq"))}

    F = attn_flops(B, Hq, N, N, d, True)
    ms_step = ms_max / K
    value = job_throughput(world, F * 3.5, ms_step)
    fwd_tflops = F / (fwd_ms_step * 1e-3) / 1e12
    bwd_tflops = 2.5 * F / (bwd_ms * 1e-3) / 1e12

    # roofline of the kernel with the largest share of the step
    timed_region_s = ms / 1e3
    peak_key = "bf16_tflops_sustained" if timed_region_s >= 2.0 else "bf16_tflops"
    peak = float(peaks.get(peak_key, FALLBACK_PEAKS[peak_key]))
    # FLOPs each kernel must execute: fwd 2 GEMMs (F), dK/dV 4 GEMMs (2F), dQ 3 GEMMs (1.5F)
    kflops = {"fwd": F, "bwd_dkdv": 2.0 * F, "bwd_dq": 1.5 * F}
    dom = max(kflops, key=lambda n: per[n])
    kname = {"fwd": "fwd_sm100_kernel", "bwd_dkdv": "bwd_dkdv_sm100_kernel", "bwd_dq": "bwd_dq_sm100_kernel"}[dom]
    achieved = kflops[dom] / (per[dom] * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": kname, "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic_for(kname),
                "peak_source": f"{peaks_kind} {peak_key}",
                "algorithmic_flops_per_launch": kflops[dom], "avg_launch_ms": round(per[dom], 4)}

    decode = None if args.no_decode else run_decode(args, torch, fa, _lib, workloads, dev, stream, world, peaks,
                                                    peaks_kind)
    fp8 = None if args.no_fp8 else run_fp8(args, torch, fa, _lib, workloads, w, q, k, v, dev, stream, world, peaks,
                                           peaks_kind)
    sparse = None if args.no_sparse else run_blocksparse(args, torch, fa, _lib, workloads, w, q, k, v, dev, stream,
                                                         world, peaks, peaks_kind)
    drop = None if args.no_dropout else run_dropout(args, torch, fa, _lib, w, q, k, v, do, dev, stream, world)
    ringl = None if args.no_ring else run_ring_local(args, torch, w, q, k, v, dev, stream, world)
    mha = None if args.no_mha else run_mha_prefill(args, torch, fa, _lib, workloads, dev, stream, world, peaks,
                                                   peaks_kind)
    longc = None if args.no_long else run_long_context(args, torch, fa, _lib, workloads, dev, stream, world, peaks,
                                                       peaks_kind)
    e2e = run_e2e(args, torch, fa, w, q, k, v, do, dev, stream, world, F) if not args.no_e2e else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(q, k, v, do, w)

    touched = sum(t.numel() * t.element_size() for t in (q, k, v, o, do, dq, dk, dv, lse, ws))
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"GQA training step: fwd+bwd, B=1 Hq=32 Hkv=8 Nq=Nk={N} d=128 causal bf16",
                   "global_batch": B * world, "seq_len": N, "parallelism": f"replicas x{world} (weak)",
                   "l2": f"no flush: each step touches {touched / 2**20:.0f} MiB (> 126 MB L2 at N=8192)",
                   "flops_convention": "fwd 4*B*Hq*N*N*d/2 (causal); bwd 2.5x fwd"},
        "parts": {"fwd_ms": round(fwd_ms_step, 4), "fwd_tflops": round(fwd_tflops, 1),
                  "fwd_frac_of_datasheet_2250": round(fwd_tflops / DENSE_BF16_DATASHEET_TFLOPS, 4),
                  "fwd_frac_of_measured": round(fwd_tflops / peak, 4),
                  "bwd_ms": round(bwd_ms, 4), "bwd_tflops": round(bwd_tflops, 1),
                  "bwd_frac_of_datasheet_2250": round(bwd_tflops / DENSE_BF16_DATASHEET_TFLOPS, 4),
                  "bwd_frac_of_measured": round(bwd_tflops / peak, 4),
                  "per_kernel_ms": {kk: round(vv, 4) for kk, vv in per.items()},
                  "per_kernel_note": "K more steps after a 0.5 s idle and W warm-up steps, one entry point "
                                     "per launch with an event between launches (the timed steps call fa_bwd, "
                                     "whose dQ launch overlaps the end of dK/dV)"},
        "decode": decode,
        "fp8": fp8,
        "blocksparse": sparse,
        "dropout": drop,
        "ring_local": ringl,
        "mha_prefill": mha,
        "long_context": longc,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 4 * K,
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_decode(args, torch, fa, _lib, workloads, dev, stream, world, peaks, peaks_kind):
    w = workloads.get(5)
    if args.decode_b:
        import dataclasses
        w = dataclasses.replace(w, B=args.decode_b)
    q, kc, vc, sl = workloads.workload_inputs(w, device=dev)
    sld = sl.to(dev)
    B, Hq, Hkv, Nmax, d = w.B, w.Hq, w.Hkv, w.Nk, w.d
    S = fa.fa_decode_num_splits(B, Hkv, Nmax, d, 0)
    ws = torch.empty(fa.fa_decode_workspace_bytes(B, Hq, S, d), device=dev, dtype=torch.uint8)
    o = torch.empty(B, 1, Hq, d, device=dev, dtype=torch.bfloat16)
    lse = torch.empty(B, Hq, 1, device=dev, dtype=torch.float32)
    sh = stream.cuda_stream

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        _lib.fa_decode_splitkv(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), sld.data_ptr(), B, Hq, Hkv, Nmax, d,
                               w.scale, S, ws.data_ptr(), _lib.FA_BF16, sh)
        if ev:
            ev[1].record(stream)
        _lib.fa_decode_combine(ws.data_ptr(), o.data_ptr(), lse.data_ptr(), sld.data_ptr(), B, Hq, S, d,
                               _lib.FA_BF16, sh)
        if ev:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    barrier(torch, world)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(K):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(torch, world)
    ms = max_over_ranks(torch, world, t0.elapsed_time(t1)) / K
    if fa.device_status() != 0:
        raise RuntimeError("kernel status word set during decode")
    split_ms = statistics.fmean(e[0].elapsed_time(e[1]) for e in evs)
    comb_ms = statistics.fmean(e[1].elapsed_time(e[2]) for e in evs)
    kv_bytes = int(sl.to(torch.int64).sum()) * Hkv * d * 2 * 2
    q_bytes = B * Hq * d * 2
    part_bytes = B * Hq * S * (d + 1) * 4
    split_bytes = kv_bytes + q_bytes + part_bytes
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    gbs_step = world * (kv_bytes + q_bytes + B * Hq * d * 2) / (ms * 1e-3) / 1e9
    gbs_split = split_bytes / (split_ms * 1e-3) / 1e9
    return {"workload": f"split-KV decode: B={B} Hq=32 Hkv=8 Nq=1 Nk_max=32768 (b>={B // 2} ragged U[1024,32768]) "
                        "d=128 bf16",
            "num_splits": S, "ms_per_step": round(ms, 4), "split_ms": round(split_ms, 4),
            "combine_ms": round(comb_ms, 4), "kv_bytes": kv_bytes, "value": round(gbs_step, 1), "unit": "GB/s",
            "frac_of_measured_hbm": round(gbs_step / hbm, 4), "frac_of_8000": round(gbs_step / 8000.0, 4),
            "roofline": {"bound": "hbm", "kernel": "decode_split_kernel", "achieved": round(gbs_split, 1),
                         "peak": hbm, "unit": "GB/s", "frac": round(gbs_split / hbm, 4),
                         "traffic": traffic_for("decode_split_kernel"), "peak_source": f"{peaks_kind} hbm_gbs",
                         "algorithmic_bytes_per_launch": split_bytes},
            "gpu_launches": 2 * K}


def run_fp8(args, torch, fa, _lib, workloads, w, q, k, v, dev, stream, world, peaks, peaks_kind):
    """FP8 forward on the same GQA inputs: E4M3 quantization (Q, K rotated) + the fp8 forward kernel."""
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.Nq, w.d
    sh = stream.cuda_stream
    signs = workloads.rotation_signs(d, 1000 * w.id + 9, device=dev)
    nb = (N + 127) // 128
    npad = (N + 15) // 16 * 16
    q8 = torch.empty(B, N, Hq, d, device=dev, dtype=torch.uint8)
    k8 = torch.empty(B, N, Hkv, d, device=dev, dtype=torch.uint8)
    v8t = torch.empty(B, Hkv, d, npad, device=dev, dtype=torch.uint8)
    qs = torch.empty(B, Hq, nb, device=dev, dtype=torch.float32)
    ks = torch.empty(B, Hkv, nb, device=dev, dtype=torch.float32)
    vs = torch.empty(B, Hkv, device=dev, dtype=torch.float32)
    vws = torch.empty(fa.fa_fp8_v_workspace_bytes(B, Hkv, N), device=dev, dtype=torch.uint8)
    o = torch.empty(B, N, Hq, d, device=dev, dtype=torch.bfloat16)
    lse = torch.empty(B, Hq, N, device=dev, dtype=torch.float32)
    dt = _lib.FA_BF16

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        _lib.fa_fp8_quantize_qkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), q8.data_ptr(), k8.data_ptr(), v8t.data_ptr(),
                                 qs.data_ptr(), ks.data_ptr(), vs.data_ptr(), signs.data_ptr(), vws.data_ptr(), B, Hq,
                                 Hkv, N, N, d, dt, sh)
        if ev:
            ev[1].record(stream)
        _lib.fa_fwd_fp8(q8.data_ptr(), qs.data_ptr(), k8.data_ptr(), ks.data_ptr(), v8t.data_ptr(), vs.data_ptr(),
                        o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N, d, 1, w.scale, 1, dt, sh)
        if ev:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    barrier(torch, world)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(K):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(torch, world)
    ms = max_over_ranks(torch, world, t0.elapsed_time(t1)) / K
    if fa.device_status() != 0:
        raise RuntimeError("kernel status word set during the fp8 section")
    quant_ms = statistics.fmean(e[0].elapsed_time(e[1]) for e in evs)
    fwd_ms = statistics.fmean(e[1].elapsed_time(e[2]) for e in evs)
    F = attn_flops(B, Hq, N, N, d, True)
    key = "bf16_tflops_sustained" if ms * K >= 2000 else "bf16_tflops"
    peak = 2.0 * float(peaks.get(key, FALLBACK_PEAKS[key]))  # e4m3 dense rate = 2x bf16 (nominal ratio)
    ach = F / (fwd_ms * 1e-3) / 1e12
    # quantizers: Q, K read once, V twice (amax, then encode), codes written once
    qbytes = (2 * (q.numel() + k.numel() + 2 * v.numel()) + q.numel() + k.numel() + v8t.numel() +
              4 * (qs.numel() + ks.numel() + vs.numel()))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    return {"workload": f"FP8 (E4M3) forward, Q/K rotated: B={B} Hq={Hq} Hkv={Hkv} N={N} d={d} causal, bf16 in/out",
            "ms_per_step": round(ms, 4), "quantize_ms": round(quant_ms, 4), "fwd_ms": round(fwd_ms, 4),
            "fwd_tflops": round(ach, 1), "value": round(world * F / (ms * 1e-3) / 1e12, 1), "unit": "TFLOP/s",
            "quantize": {"bytes": qbytes, "gbs": round(qbytes / (quant_ms * 1e-3) / 1e9, 1),
                         "frac_of_measured_hbm": round(qbytes / (quant_ms * 1e-3) / 1e9 / hbm, 4),
                         "launches": 2, "traffic": traffic_for("quant_kernel + v_quant_kernel")},
            "roofline": {"bound": "tensor", "kernel": "fwd_sm100_kernel (F8)", "achieved": round(ach, 1),
                         "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                         "traffic": traffic_for("fwd_sm100_kernel (F8)"),
                         "peak_source": f"{peaks_kind} {key} x 2 (nominal e4m3 / bf16 ratio)",
                         "algorithmic_flops_per_launch": F},
            "gpu_launches": 3 * K}


def run_blocksparse(args, torch, fa, _lib, workloads, w, q, k, v, dev, stream, world, peaks, peaks_kind):
    """Block-sparse forward on the same GQA inputs: causal, local window of 8 key blocks + the first block."""
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.Nq, w.d
    nb = (N + 127) // 128
    window = 8
    bm = workloads.block_mask_local(B, Hq, nb, nb, window=window, sink=1).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, N, device=dev, dtype=torch.float32)
    sh = stream.cuda_stream

    def step():
        _lib.fa_fwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), bm.data_ptr(),
                                B, Hq, Hkv, N, N, d, 1, w.scale, _lib.FA_BF16, sh)

    for _ in range(args.warmup):
        step()
    K = args.steps
    barrier(torch, world)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(K):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(torch, world)
    ms = max_over_ranks(torch, world, t0.elapsed_time(t1)) / K
    if fa.device_status() != 0:
        raise RuntimeError("kernel status word set during the block-sparse section")
    # FLOPs of the visible pairs (4 d per pair): per query block I, causal diagonal block plus full blocks
    pairs = 0
    for I in range(nb):
        js = set(range(max(0, I - window + 1), I + 1)) | {0}
        for J in js:
            pairs += 128 * 129 // 2 if J == I else 128 * 128
    F = 4.0 * d * pairs * B * Hq
    key = "bf16_tflops_sustained" if ms * K >= 2000 else "bf16_tflops"
    peak = float(peaks.get(key, FALLBACK_PEAKS[key]))
    ach = F / (ms * 1e-3) / 1e12
    dense = attn_flops(B, Hq, N, N, d, True)
    return {"workload": f"block-sparse forward, causal, local window {window} blocks + first block (128 x 128 blocks): "
                        f"B={B} Hq={Hq} Hkv={Hkv} N={N} d={d} bf16",
            "density_vs_causal": round(F / dense, 4), "ms_per_step": round(ms, 4),
            "value": round(world * ach, 1), "unit": "TFLOP/s (visible pairs)",
            "roofline": {"bound": "tensor", "kernel": "fwd_sm100_kernel (SPARSE)", "achieved": round(ach, 1),
                         "peak": peak, "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                         "traffic": traffic_for("fwd_sm100_kernel (SPARSE)"),
                         "peak_source": f"{peaks_kind} {key}", "algorithmic_flops_per_launch": F},
            "gpu_launches": K}


def run_dropout(args, torch, fa, _lib, w, q, k, v, do, dev, stream, world):
    """The GQA training step with dropout p = 0.1 (mask regenerated in the backward kernels)."""
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.Nq, w.d
    p_drop, seed = 0.1, 0x5EED
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, N, device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, Hq, N), device=dev, dtype=torch.uint8)
    sh = stream.cuda_stream

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        _lib.fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N,
                            d, 1, w.scale, p_drop, seed, 0, _lib.FA_BF16, sh)
        if ev:
            ev[1].record(stream)
        _lib.fa_bwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), B, Hq, Hkv, N, N, d, 1,
                            w.scale, p_drop, seed, 0, _lib.FA_BF16, sh)
        if ev:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    barrier(torch, world)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(K):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(torch, world)
    ms = max_over_ranks(torch, world, t0.elapsed_time(t1)) / K
    if fa.device_status() != 0:
        raise RuntimeError("kernel status word set during the dropout section")
    fwd_ms = statistics.fmean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.fmean(e[1].elapsed_time(e[2]) for e in evs)
    F = attn_flops(B, Hq, N, N, d, True)
    return {"workload": f"GQA training step with dropout p={p_drop}: B={B} Hq={Hq} Hkv={Hkv} N={N} d={d} causal bf16",
            "ms_per_step": round(ms, 4), "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4),
            "value": round(world * 3.5 * F / (ms * 1e-3) / 1e12, 1), "unit": "TFLOP/s",
            "fwd_tflops": round(F / (fwd_ms * 1e-3) / 1e12, 1),
            "bwd_tflops": round(2.5 * F / (bwd_ms * 1e-3) / 1e12, 1), "gpu_launches": 4 * K}


def run_ring_local(args, torch, w, q, k, v, dev, stream, world):
    """Ring attention forward (context parallelism) for 4 virtual ranks run one after another on this GPU."""
    from exact_io_aware_80_b200 import ring
    W = 4
    for _ in range(args.warmup):
        ring.ring_attention_fwd_local(q, k, v, W, True, w.scale)
    K = max(1, args.steps // 2)
    barrier(torch, world)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(K):
        ring.ring_attention_fwd_local(q, k, v, W, True, w.scale)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(torch, world)
    ms = max_over_ranks(torch, world, t0.elapsed_time(t1)) / K
    F = attn_flops(w.B, w.Hq, w.Nq, w.Nk, w.d, True)
    return {"workload": f"ring attention forward, {W} virtual ranks on one GPU (no communication), causal: "
                        f"B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.Nq} d={w.d} bf16",
            "ms_per_step": round(ms, 4), "value": round(world * F / (ms * 1e-3) / 1e12, 1), "unit": "TFLOP/s",
            "gpu_launches": K * (W * (W + 1) - 1)}  # W(W+1)/2 forward launches, one merge fewer (rank 0 copies)


def _peak_for(peaks, region_ms):
    key = "bf16_tflops_sustained" if region_ms >= 2000 else "bf16_tflops"
    return float(peaks.get(key, FALLBACK_PEAKS[key])), key


def run_mha_prefill(args, torch, fa, _lib, workloads, dev, stream, world, peaks, peaks_kind):
    """MHA prefill forward, B=4, H=16, N=2048, d=128 bf16, causal and non-causal.  Its four tensors
    (Q, K, V, O: 128 MiB) are about the size of L2, so L2 is flushed (a 256 MiB write) before every
    timed launch and each launch is timed alone with CUDA events on the launching stream."""
    w = workloads.get(2)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.Nq, w.d
    q, k, v = workloads.workload_inputs(w, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, N, device=dev, dtype=torch.float32)
    flush = torch.empty(256 << 20, device=dev, dtype=torch.uint8)
    sh = stream.cuda_stream
    out = {"workload": f"MHA prefill forward: B={B} Hq=Hkv={Hq} Nq=Nk={N} d={d} bf16",
           "l2": "flushed before every timed launch (256 MiB write, outside the timed events)"}
    total_ms = 0.0
    for causal in (False, True):
        def launch():
            _lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N, d,
                        int(causal), w.scale, _lib.FA_BF16, sh)

        for _ in range(args.warmup):
            launch()
        K = args.steps
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        barrier(torch, world)
        torch.cuda.synchronize(dev)
        for e0, e1 in evs:
            flush.fill_(1)
            e0.record(stream)
            launch()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(torch, world)
        if fa.device_status() != 0:
            raise RuntimeError("kernel status word set during the MHA prefill section")
        ms = max_over_ranks(torch, world, statistics.fmean(e0.elapsed_time(e1) for e0, e1 in evs))
        total_ms += ms * K
        F = attn_flops(B, Hq, N, N, d, causal)
        ach = F / (ms * 1e-3) / 1e12
        peak, key = _peak_for(peaks, ms * K)
        out["causal" if causal else "noncausal"] = {
            "ms": round(ms, 4), "value": round(world * ach, 1), "unit": "TFLOP/s",
            "frac_of_datasheet_2250": round(ach / DENSE_BF16_DATASHEET_TFLOPS, 4),
            "roofline": {"bound": "tensor", "kernel": "fwd_sm100_kernel", "achieved": round(ach, 1), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(ach / peak, 4), "traffic": None,
                         "peak_source": f"{peaks_kind} {key}", "algorithmic_flops_per_launch": F},
            "gpu_launches": K}
    return out


def run_long_context(args, torch, fa, _lib, workloads, dev, stream, world, peaks, peaks_kind):
    """Long-context GQA step, B=1, Hq=32, Hkv=8, N=16384, d=128 bf16 causal: forward + the three
    backward launches, timed per launch like the headline step (each step touches ~650 MiB, more
    than L2, so no flush)."""
    w = workloads.get(4)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.Nq, w.d
    q, k, v, do = workloads.workload_inputs(w, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, N, device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, Hq, N), device=dev, dtype=torch.uint8)
    sh = stream.cuda_stream
    dt = _lib.FA_BF16
    bargs = [t.data_ptr() for t in (q, k, v, o, do, lse, dq, dk, dv, ws)] + [B, Hq, Hkv, N, N, d, 1, w.scale, dt, sh]

    def fwd():
        _lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N, d, 1,
                    w.scale, dt, sh)

    def step(ev=None):  # as a user runs it: fa_fwd, then the one-call fa_bwd
        if ev:
            ev[0].record(stream)
        fwd()
        if ev:
            ev[1].record(stream)
        _lib.fa_bwd(*bargs)
        if ev:
            ev[2].record(stream)

    def step_per_kernel(ev):  # one entry point per launch, an event between launches
        ev[0].record(stream)
        fwd()
        ev[1].record(stream)
        _lib.fa_bwd_preprocess(*bargs)
        ev[2].record(stream)
        _lib.fa_bwd_dkdv(*bargs)
        ev[3].record(stream)
        _lib.fa_bwd_dq(*bargs)
        ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    K = max(3, args.steps // 2)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    evk = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    barrier(torch, world)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(K):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(torch, world)
    time.sleep(0.5)  # per-kernel pass from the same starting conditions as the timed steps
    for _ in range(args.warmup):
        step()
    for i in range(K):
        step_per_kernel(evk[i])
    torch.cuda.synchronize(dev)
    barrier(torch, world)
    if fa.device_status() != 0:
        raise RuntimeError("kernel status word set during the long-context section")
    ms_total = t0.elapsed_time(t1)
    ms = max_over_ranks(torch, world, ms_total) / K
    per = {name: statistics.fmean(e[j].elapsed_time(e[j + 1]) for e in evk)
           for j, name in enumerate(("fwd", "bwd_preprocess", "bwd_dkdv", "bwd_dq"))}
    F = attn_flops(B, Hq, N, N, d, True)
    fwd_ms = statistics.fmean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.fmean(e[1].elapsed_time(e[2]) for e in evs)
    peak, key = _peak_for(peaks, ms_total)
    kflops = {"fwd": F, "bwd_dkdv": 2.0 * F, "bwd_dq": 1.5 * F}
    dom = max(kflops, key=lambda n: per[n])
    kname = {"fwd": "fwd_sm100_kernel", "bwd_dkdv": "bwd_dkdv_sm100_kernel", "bwd_dq": "bwd_dq_sm100_kernel"}[dom]
    ach = kflops[dom] / (per[dom] * 1e-3) / 1e12
    fwd_t, bwd_t = F / (fwd_ms * 1e-3) / 1e12, 2.5 * F / (bwd_ms * 1e-3) / 1e12
    traffic8192 = traffic_for(kname)
    traffic8192 = None if traffic8192 is None else int(traffic8192 * N / 8192)
    return {"workload": f"long-context GQA step: fwd+bwd, B={B} Hq={Hq} Hkv={Hkv} Nq=Nk={N} d={d} causal bf16",
            "ms_per_step": round(ms, 4), "value": round(world * 3.5 * F / (ms * 1e-3) / 1e12, 1), "unit": "TFLOP/s",
            "fwd_ms": round(fwd_ms, 4), "fwd_tflops": round(fwd_t, 1),
            "fwd_frac_of_datasheet_2250": round(fwd_t / DENSE_BF16_DATASHEET_TFLOPS, 4),
            "bwd_ms": round(bwd_ms, 4), "bwd_tflops": round(bwd_t, 1),
            "bwd_frac_of_datasheet_2250": round(bwd_t / DENSE_BF16_DATASHEET_TFLOPS, 4),
            "per_kernel_ms": {kk: round(vv, 4) for kk, vv in per.items()},
            "roofline": {"bound": "tensor", "kernel": kname, "achieved": round(ach, 1), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(ach / peak, 4), "traffic": traffic8192,
                         "traffic_basis": "the N=8192 figure x N / 8192 (each input is read once per launch)",
                         "peak_source": f"{peaks_kind} {key}", "algorithmic_flops_per_launch": kflops[dom],
                         "avg_launch_ms": round(per[dom], 4)},
            "gpu_launches": 4 * K}


def run_e2e(args, torch, fa, w, q, k, v, do, dev, stream, world, F):
    """Same step through the public Python API with host buffers: every step uploads q, k, v, dO from
    pinned host memory, runs the forward and backward, and downloads dQ, dK, dV, all inside the timed
    region.  Uploads, kernels and downloads run on three streams with two device buffer sets, so the
    copies of neighbouring steps overlap the current step's kernels (events keep a buffer set from
    being refilled before its kernels and download are done)."""
    hq, hk, hv, hdo = (t.cpu().pin_memory() for t in (q, k, v, do))
    h_out = [tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (q, k, v)) for _ in range(2)]
    bufs = []
    for _ in range(2):
        bufs.append({"q": torch.empty_like(q), "k": torch.empty_like(k), "v": torch.empty_like(v),
                     "do": torch.empty_like(do), "dq": torch.empty_like(q), "dk": torch.empty_like(k),
                     "dv": torch.empty_like(v),
                     "ws": torch.empty(fa.fa_bwd_workspace_bytes(w.B, w.Hq, w.Nq), device=dev, dtype=torch.uint8)})
    up, comp, down = (torch.cuda.Stream(device=dev) for _ in range(3))
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    downloaded = [torch.cuda.Event() for _ in range(2)]
    seen = [False, False]

    def step(i):
        b = i % 2
        d = bufs[b]
        with torch.cuda.stream(up):
            if seen[b]:
                up.wait_event(computed[b])  # the kernels of step i - 2 have read these inputs
            d["q"].copy_(hq, non_blocking=True)
            d["k"].copy_(hk, non_blocking=True)
            d["v"].copy_(hv, non_blocking=True)
            d["do"].copy_(hdo, non_blocking=True)
            uploaded[b].record(up)
        with torch.cuda.stream(comp):
            comp.wait_event(uploaded[b])
            if seen[b]:
                comp.wait_event(downloaded[b])  # step i - 2's gradients have left these buffers
            o, lse = fa.attention_fwd(d["q"], d["k"], d["v"], causal=True)
            fa.attention_bwd(d["q"], d["k"], d["v"], o, d["do"], lse, causal=True, workspace=d["ws"], dq=d["dq"],
                             dk=d["dk"], dv=d["dv"])
            computed[b].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(computed[b])
            for host, dev_t in zip(h_out[b], (d["dq"], d["dk"], d["dv"])):
                host.copy_(dev_t, non_blocking=True)
            downloaded[b].record(down)
        seen[b] = True

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    barrier(torch, world)
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    up.wait_stream(down)  # the timed region starts after the warm-up's last download
    t0.record(up)
    for i in range(K):
        step(args.warmup + i)
    t1.record(down)  # after every step's download (and, through the events, every kernel)
    torch.cuda.synchronize(dev)
    barrier(torch, world)
    ms = max_over_ranks(torch, world, t0.elapsed_time(t1)) / K
    if fa.device_status() != 0:
        raise RuntimeError("kernel status word set during the end-to-end section")
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v, do))
    d2h = sum(t.numel() * t.element_size() for t in (q, k, v))
    return {"value": round(world * 3.5 * F / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelining": "uploads, kernels and downloads on three streams, two device buffer sets"}


def cpu_baseline(q, k, v, do, w):
    """The fp64 oracle as it stands, on the host cores, on a bounded sample of the
    same workload: KV group 0 (4 query heads) of the GQA training step, fwd + bwd."""
    import numpy as np

    import oracle
    G = w.Hq // w.Hkv
    qs = q[:, :, :G].float().cpu().numpy().astype(np.float64)
    ks = k[:, :, :1].float().cpu().numpy().astype(np.float64)
    vs = v[:, :, :1].float().cpu().numpy().astype(np.float64)
    dos = do[:, :, :G].float().cpu().numpy().astype(np.float64)
    threads = _blas_threads()
    t = time.perf_counter()
    oracle.attention_fwd(qs, ks, vs, True, w.scale)
    oracle.attention_bwd(qs, ks, vs, dos, True, w.scale)
    dt = time.perf_counter() - t
    flops = 3.5 * attn_flops(1, G, w.Nq, w.Nk, w.d, True)
    return {"value": round(flops / dt / 1e12, 5), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"KV group 0 ({G} query heads) of the GQA training step, fwd+bwd, {dt:.1f} s",
            "seconds": round(dt, 2)}


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:  # noqa: BLE001
        pass
    return os.cpu_count()


# ---------------------------------------------------------------------------
# reference arm: the fp64 oracle on the host cores
# ---------------------------------------------------------------------------
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle
    import workloads
    w = workloads.get(3)
    q, k, v, do = workloads.workload_inputs(w)
    # one query head and its KV head of the GQA training step, fwd + bwd, per step
    qs, ks, vs, dos = (t[:, :, :1].float().numpy().astype(np.float64) for t in (q, k, v, do))
    del torch

    def step():
        oracle.attention_fwd(qs, ks, vs, True, w.scale)
        oracle.attention_bwd(qs, ks, vs, dos, True, w.scale)

    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t) / args.steps
    flops = 3.5 * attn_flops(1, 1, w.Nq, w.Nk, w.d, True)
    val = flops / dt / 1e12
    threads = _blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(val, 5), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "GQA training step: fwd+bwd, B=1 Hq=32 Hkv=8 Nq=Nk=8192 d=128 causal bf16 inputs",
                   "sample": "one query head with its KV head per step", "global_batch": 1, "seq_len": w.Nq,
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": round(val, 5), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": "one query head with its KV head of the GQA training step, fwd+bwd"},
        "e2e": {"value": round(val, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode section (profiling runs)")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 forward section (profiling runs)")
    ap.add_argument("--no-sparse", action="store_true", help="skip the block-sparse section (profiling runs)")
    ap.add_argument("--no-dropout", action="store_true", help="skip the dropout section (profiling runs)")
    ap.add_argument("--no-ring", action="store_true", help="skip the one-GPU ring-attention section")
    ap.add_argument("--no-mha", action="store_true", help="skip the MHA prefill section (B=4 H=16 N=2048)")
    ap.add_argument("--no-long", action="store_true", help="skip the long-context section (N=16384)")
    ap.add_argument("--decode-b", type=int, default=0,
                    help="override B of the decode workload (profiling runs on a smaller case)")
    ap.add_argument("--seq", type=int, default=0,
                    help="override N of the training-step workload (profiling runs on a smaller case)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
