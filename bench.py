#!/usr/bin/env python
"""Throughput of the B200 TTT-Linear scan, as one JSON line.

Headline workload: the per-token fp32 scan at d = 64 (B=4, H=4, T=2048, q and k
L2-normalised, eps = 1e-6); one step is one pass with the simplified gradient
plus one pass with the LayerNorm-Jacobian gradient over the same inputs.
The metric is head-tokens per second (B*H*T per pass) and the fraction of the
binding roofline of the dominant kernel. On one GPU the other d = 64 workloads
(mini-batch bf16 at three shapes, the per-token bf16-input pass, and the
streaming decode step over 16384 heads) are measured too and reported under
``by_workload``.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one rank per GPU) every rank scans its own batch of the
headline workload (weak scaling; heads are independent, nothing is exchanged)
and the slowest rank's device time is reported. ``--impl reference`` times the
CPU oracle on the host cores instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "TTT-Linear scan head-tokens/sec at d=64 on 1 B200; % of binding roofline"
L2_FLUSH_BYTES = 256 << 20      # > 126 MB L2
PROFILE_TRAFFIC = ROOT / "profiles" / "dram_traffic.json"


def _peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"),
                    sm_max_mhz=d.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                sm_max_mhz=1965.0, source="fallback")


def _csrc_hash() -> str:
    h = hashlib.sha256()
    csrc = ROOT / "test_sequence_layers_02_b200" / "csrc"
    for p in sorted(csrc.glob("*")) + sorted((ROOT / "include").glob("*.h")):
        h.update(p.name.encode())
        h.update(p.read_bytes())
    return h.hexdigest()[:16]


# The files each kernel's binary is built from: the translation unit that
# instantiates it and everything that unit includes, plus (for every kernel)
# the launcher that sets its parameters, the public header and the build flags.
_KERNEL_SOURCES = {
    "scan_cluster": ["cluster.cu", "scan_cluster.cuh", "scan_simt.cuh", "launch.h", "common.cuh"],
    "scan_simt": ["simt_f32.cu", "simt_bf16.cu", "scan_simt.cuh", "launch.h", "common.cuh"],
    # one translation unit holds both
    "scan_tc": ["scan_tc.cuh", "sm100.cuh", "decode.cuh", "scan_simt.cuh", "launch.h", "common.cuh"],
    "decode_step": ["scan_tc.cuh", "sm100.cuh", "decode.cuh", "scan_simt.cuh", "launch.h",
                    "common.cuh"],
}


def _kernel_hash(kernel_key: str) -> str:
    pkg = ROOT / "test_sequence_layers_02_b200"
    files = sorted(set(_KERNEL_SOURCES[kernel_key] + ["ttt_scan.cu"]))
    paths = [pkg / "csrc" / f for f in files] + [pkg / "build.py", ROOT / "include" / "ttt_scan.h"]
    h = hashlib.sha256()
    for p in paths:
        h.update(p.name.encode())
        h.update(p.read_bytes())
    return h.hexdigest()[:16]


def _traffic(kernel_key: str, head_tokens_per_launch: int):
    """DRAM bytes (read + write) per launch from the committed ncu capture of
    that kernel, scaled from its case by head-tokens; None if that kernel's
    sources changed since the capture."""
    if not PROFILE_TRAFFIC.exists():
        return None
    d = json.loads(PROFILE_TRAFFIC.read_text())
    e = d.get("kernels", {}).get(kernel_key)
    if e is None:
        return None
    if "sources_hash" in e:
        if e["sources_hash"] != _kernel_hash(kernel_key):
            return None
    elif d.get("csrc_hash") != _csrc_hash():
        return None
    return round(e["bytes_per_head_token"] * head_tokens_per_launch)


# ---------------------------------------------------------------------------
# Workloads
# ---------------------------------------------------------------------------

class Job:
    """One workload resident on the device, with its step function."""

    def __init__(self, name: str, device, seed_offset: int = 0):
        import torch
        from test_sequence_layers_02_b200 import ttt_scan
        from test_sequence_layers_02_b200.workloads import WORKLOADS, make_workload
        self.w = w = WORKLOADS["2s" if name == "2" else name]
        self.name = name
        self.passes = ([dict(lnjac=False), dict(lnjac=True)] if name == "2"
                       else [dict(lnjac=w.lnjac)])
        inp = make_workload(w, seed=w.seed + seed_offset) if seed_offset else make_workload(w)
        self.inp = inp
        self.mask_np = inp.get("mask")

        def dev(key):
            a = inp.get(key)
            if a is None:
                return None
            if w.in_bf16 and key in ("q", "k", "v", "eta_logit", "gate_logit"):
                return torch.from_numpy(inp[key + "_bf16"].view(np.int16)).view(torch.bfloat16).to(device)
            return torch.from_numpy(np.ascontiguousarray(a)).to(device)

        self.t = {k: dev(k) for k in ("q", "k", "v", "eta_logit", "gate_logit", "W0", "gamma", "beta")}
        self.t["mask"] = None if self.mask_np is None else torch.from_numpy(self.mask_np).to(device)
        self.out_dtype = torch.bfloat16 if w.out_bf16 else torch.float32
        t = self.t
        self.o = torch.empty(t["q"].shape, dtype=self.out_dtype, device=device)
        self.W_T = torch.empty(t["W0"].shape, dtype=torch.float32, device=device)
        self.scan = ttt_scan.scan

    @property
    def head_tokens_per_step(self) -> int:
        return self.w.head_tokens * len(self.passes)

    def step(self):
        """One step: every pass over the resident inputs. Independent passes (the
        two gradient forms of workload 2) run concurrently on their own streams."""
        import torch
        t, w = self.t, self.w
        if len(self.passes) == 1:
            self.scan(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"],
                      t["gamma"], t["beta"], eps=w.eps, minibatch=w.minibatch, b=w.b,
                      mask=t["mask"], out_dtype=self.out_dtype, o=self.o, W_T=self.W_T,
                      **self.passes[0])
            return
        main = torch.cuda.current_stream()
        if not hasattr(self, "streams"):
            self.streams = [torch.cuda.Stream() for _ in self.passes]
            self.outs = [(torch.empty_like(self.o), torch.empty_like(self.W_T)) for _ in self.passes]
        start = torch.cuda.Event()
        start.record(main)
        for st, ps, (o, wt) in zip(self.streams, self.passes, self.outs):
            st.wait_event(start)
            self.scan(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"],
                      t["gamma"], t["beta"], eps=w.eps, minibatch=w.minibatch, b=w.b,
                      mask=t["mask"], out_dtype=self.out_dtype, o=o, W_T=wt, stream=st, **ps)
        for st in self.streams:
            ev = torch.cuda.Event()
            ev.record(st)
            main.wait_event(ev)

    def launches_per_step(self) -> int:
        return len(self.passes)

    # --- algorithmic work per step -------------------------------------------------
    def flops_per_step(self) -> float:
        w = self.w
        d, b = w.d, w.b
        if not w.minibatch:
            return 6.0 * d * d * w.head_tokens * len(self.passes)
        f_upd = 6.0 * d * d + 2.0 * d * (b + 1)
        f_skip = 2.0 * d * d
        frac = 1.0 if self.mask_np is None else float(self.mask_np.mean())
        return w.head_tokens * (frac * f_upd + (1 - frac) * f_skip)

    def bytes_per_step(self) -> float:
        w = self.w
        d, T = w.d, w.T
        ie = 2 if w.in_bf16 else 4
        oe = 2 if w.out_bf16 else 4
        state = 2.0 * d * d * 4 * w.heads
        if self.mask_np is None:
            per_tok = 3 * d * ie + 2 * ie + d * oe
            return (per_tok * w.head_tokens + state) * len(self.passes)
        # SKIP chunks need only q, the gate logit and the output (plus the mask byte)
        upd_tok = 3 * d * ie + 2 * ie + d * oe
        skip_tok = d * ie + ie + d * oe
        total = 0.0
        n_chunks = self.mask_np.shape[1]
        for bi in range(w.B):
            for c in range(n_chunks):
                ntok = min(w.b, T - c * w.b)
                total += w.H * ntok * (upd_tok if self.mask_np[bi, c] else skip_tok)
        total += self.mask_np.size * w.H
        return total + state

    def bound(self):
        return "hbm" if self.w.minibatch else "alu"

    def kernel_key(self) -> str:
        from test_sequence_layers_02_b200 import ttt_scan
        w = self.w
        k = ttt_scan.kernel_choice(w.B, w.H, w.T, w.d, minibatch=w.minibatch, lnjac=w.lnjac,
                                   in_bf16=w.in_bf16, out_bf16=w.out_bf16, b=w.b)
        return {ttt_scan.KERNEL_CUDA_CORE: "scan_simt",
                ttt_scan.KERNEL_CUDA_CORE_CLUSTER: "scan_cluster",
                ttt_scan.KERNEL_TENSOR_CORE: "scan_tc"}[k]


class DecodeJob:
    """The streaming decode step over many heads, W updated in place each step."""

    def __init__(self, name: str, device):
        import torch
        from test_sequence_layers_02_b200 import ttt_scan
        from test_sequence_layers_02_b200.workloads import DECODE_WORKLOADS, make_workload
        self.w = w = DECODE_WORKLOADS[name]
        self.name = name
        self.passes = [dict(lnjac=w.lnjac)]
        inp = make_workload(w)
        self.inp = inp
        self.mask_np = None

        def dev(key):
            a = inp.get(key)
            if a is None:
                return None
            if w.in_bf16 and key in ("q", "k", "v", "eta_logit", "gate_logit"):
                a = torch.from_numpy(inp[key + "_bf16"].view(np.int16)).view(torch.bfloat16)
            else:
                a = torch.from_numpy(np.ascontiguousarray(a))
            if key in ("q", "k", "v", "eta_logit", "gate_logit"):
                a = a[:, :, 0].contiguous()
            return a.to(device)

        self.t = {k: dev(k) for k in ("q", "k", "v", "eta_logit", "gate_logit", "W0", "gamma", "beta")}
        self.out_dtype = torch.bfloat16 if w.out_bf16 else torch.float32
        self.o = torch.empty(self.t["q"].shape, dtype=self.out_dtype, device=device)
        self.step_fn = ttt_scan.decode_step

    @property
    def head_tokens_per_step(self) -> int:
        return self.w.heads

    def step(self):
        t, w = self.t, self.w
        self.step_fn(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"], t["gamma"],
                     t["beta"], eps=w.eps, lnjac=w.lnjac, out_dtype=self.out_dtype, o=self.o)

    def launches_per_step(self) -> int:
        return 1

    def flops_per_step(self) -> float:
        return 6.0 * self.w.d * self.w.d * self.w.heads

    def bytes_per_step(self) -> float:
        w = self.w
        d = w.d
        ie = 2 if w.in_bf16 else 4
        oe = 2 if w.out_bf16 else 4
        per_head = 2 * d * d * 4 + 3 * d * ie + 2 * ie + d * oe
        return float(per_head * w.heads + 2 * w.H * d * 4)

    def bound(self):
        return "hbm"

    def kernel_key(self) -> str:
        return "decode_step"


def _flush(buf):
    buf.fill_(1.0)


def _time_job(job, steps, warmup, flush_buf):
    """Device time of `steps` steps (events around each step, L2 flushed between)."""
    import torch
    for _ in range(warmup):
        _flush(flush_buf)
        job.step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    evs = []
    for _ in range(steps):
        _flush(flush_buf)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        job.step()
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    from test_sequence_layers_02_b200 import ttt_scan
    rc = ttt_scan.check_device_status()
    if rc != ttt_scan.TTT_OK:
        raise RuntimeError(f"device status {ttt_scan.status_string(rc)}")
    return [a.elapsed_time(b) / 1e3 for a, b in evs]


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every
    few milliseconds while the timed region runs (read-only queries)."""

    REASONS = {
        "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
        "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
        "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
        "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
        "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.dev = device_index
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._nvml = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            props = torch.cuda.get_device_properties(self.dev)
            bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def _run(self):
        import pynvml
        h = self._h
        bits = {nm: getattr(pynvml, attr, 0) for nm, attr in self.REASONS.items()}
        while not self._stop.is_set():
            try:
                self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                for nm, bit in bits.items():
                    if bit and (r & bit):
                        self.reasons.add(nm)
            except Exception:
                break
            time.sleep(self.period)

    def __enter__(self):
        try:
            import pynvml
            self._h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        except Exception:
            self._h = None
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if getattr(self, "thread", None) is not None:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples),
                "sm_mhz_min": min(self.samples), "source": "NVML, 2 ms polling"}


def _fp32_peak(device):
    """Measured FFMA throughput (TFLOP/s) of this device with the library's probe."""
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    props = torch.cuda.get_device_properties(device)
    blocks, threads, iters = props.multi_processor_count * 8, 256, 4000
    sink = torch.empty(blocks * threads, dtype=torch.float32, device=device)
    ttt_scan.probe_ffma(blocks, threads, 200, sink)
    torch.cuda.synchronize()
    best = 0.0
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fl = ttt_scan.probe_ffma(blocks, threads, iters, sink)
        e1.record()
        torch.cuda.synchronize()
        best = max(best, fl / (e0.elapsed_time(e1) / 1e3) / 1e12)
    return best, props.multi_processor_count


def _roofline(job, per_launch_s, peaks, fp32_meas_tflops, n_sm):
    launches = job.launches_per_step()
    if job.bound() == "alu":
        flops = job.flops_per_step() / launches
        achieved = flops / per_launch_s / 1e12
        peak = n_sm * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12
        return {"bound": "alu", "achieved": round(achieved, 3), "peak": round(peak, 2),
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "traffic": _traffic(job.kernel_key(), job.w.head_tokens),
                "algorithmic_flops_per_launch": flops,
                "peak_basis": f"{n_sm} SM x 128 FP32 lanes x 2 x {peaks['sm_max_mhz']:.0f} MHz",
                "fp32_probe_tflops": round(fp32_meas_tflops, 2),
                "frac_of_probe": round(achieved / fp32_meas_tflops, 4),
                "kernel": job.kernel_key()}
    byts = job.bytes_per_step() / launches
    achieved = byts / per_launch_s / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": _traffic(job.kernel_key(), job.w.head_tokens), "kernel": job.kernel_key(),
            "algorithmic_bytes_per_launch": round(byts),
            "peak_basis": f"{peaks['source']} HBM copy bandwidth"}


def _oracle_pass(w, inp, passes, heads, threads):
    """One oracle run over the sampled heads (OpenMP over heads), every pass."""
    import oracle
    f64 = lambda a: None if a is None else np.asarray(a, dtype=np.float64)
    sel = lambda a: None if a is None else f64(a[:, :heads] if a.ndim >= 3 else a)
    rows = heads if heads < w.H else w.H
    for ps in passes:
        mode = (1 if w.minibatch else 0) | (2 if ps["lnjac"] else 0)
        m = inp.get("mask")
        if heads >= w.H:
            oracle.forward(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["eta_logit"]),
                           f64(inp["gate_logit"]), f64(inp["W0"]), f64(inp["gamma"]),
                           f64(inp["beta"]), eps=w.eps, mode=mode, b=w.b, mask=m, nthreads=threads)
        else:
            oracle.forward(sel(inp["q"][:1]), sel(inp["k"][:1]), sel(inp["v"][:1]),
                           sel(inp["eta_logit"][:1]), sel(inp["gate_logit"][:1]),
                           sel(inp["W0"][:1]), f64(inp["gamma"][:rows]), f64(inp["beta"][:rows]),
                           eps=w.eps, mode=mode, b=w.b, mask=None if m is None else m[:1],
                           nthreads=threads)


def _cpu_baseline(job, min_seconds=8.0):
    """The oracle, as it stands, on the host cores: head-tokens/s over the whole workload."""
    w = job.w
    cores = len(os.sched_getaffinity(0))
    used = min(cores, w.heads)
    t0 = time.perf_counter()
    reps = 0
    while True:
        _oracle_pass(w, job.inp, job.passes, w.heads, used)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= 8:
            break
    return {"value": job.head_tokens_per_step * reps / el, "unit": "head-tokens/s",
            "cores": used, "kind": "oracle",
            "sample": f"whole workload {job.name} ({w.heads} heads x T={w.T} x {len(job.passes)} "
                      f"pass(es)) x {reps} rep(s), fp64, OpenMP over heads, {el:.1f} s"}


def _e2e(job, steps, device):
    """Same metric through the public API, end to end. Every step copies that
    step's inputs from pinned host memory to the device (once: the passes share
    them), runs the passes on their own streams as the device-timed step does,
    copies every pass's results (o, W_T) back to pinned host memory as soon as
    that pass ends, and waits for them on the host."""
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    t = job.t
    w = job.w
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in t.items()}
    dev = {k: (None if v is None else torch.empty_like(v)) for k, v in t.items()}
    n = len(job.passes)
    o_h = [torch.empty(t["q"].shape, dtype=job.out_dtype).pin_memory() for _ in range(n)]
    wt_h = [torch.empty(t["W0"].shape, dtype=torch.float32).pin_memory() for _ in range(n)]
    o_d = [torch.empty_like(t["q"], dtype=job.out_dtype) for _ in range(n)]
    wt_d = [torch.empty_like(t["W0"]) for _ in range(n)]
    streams = [torch.cuda.Stream(device) for _ in range(n)]
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = sum(o.numel() * o.element_size() + x.numel() * x.element_size()
              for o, x in zip(o_h, wt_h))

    def step():
        main = torch.cuda.current_stream(device)
        for k, v in host.items():
            if v is not None:
                dev[k].copy_(v, non_blocking=True)
        for i, ps in enumerate(job.passes):
            st = streams[i]
            st.wait_stream(main)
            ttt_scan.scan(dev["q"], dev["k"], dev["v"], dev["eta_logit"], dev["gate_logit"],
                          dev["W0"], dev["gamma"], dev["beta"], eps=w.eps,
                          minibatch=w.minibatch, b=w.b, mask=dev["mask"],
                          out_dtype=job.out_dtype, o=o_d[i], W_T=wt_d[i], stream=st, **ps)
            with torch.cuda.stream(st):
                o_h[i].copy_(o_d[i], non_blocking=True)
                wt_h[i].copy_(wt_d[i], non_blocking=True)
            main.wait_stream(st)
        rc = ttt_scan.check_device_status(main)   # synchronises: the results are on the host
        if rc != ttt_scan.TTT_OK:
            raise ttt_scan.TTTScanError(rc, "device")

    step()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
    torch.cuda.synchronize()
    el = time.perf_counter() - t0
    return {"value": job.head_tokens_per_step * steps / el, "unit": "head-tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(el / steps * 1e3, 3)}


def _workload_desc(job):
    w = job.w
    if isinstance(job, DecodeJob):
        return (f"TTT-Linear decode step {job.name}: one token per head, W [B,H,d,d] fp32 "
                f"updated in place, LN-Jacobian gradient, bf16 in, bf16 out, B={w.B} H={w.H} "
                f"d={w.d}")
    mode = "mini-batch b=%d" % w.b if w.minibatch else "per-token"
    grad = "simplified + LN-Jacobian gradients" if len(job.passes) == 2 else (
        "LN-Jacobian gradient" if w.lnjac else "simplified gradient")
    dt = ("bf16 in" if w.in_bf16 else "fp32 in") + (", bf16 out" if w.out_bf16 else ", fp32 out")
    extra = ", SKIP/UPDATE mask ~ Bernoulli(0.5)" if w.mask_p else ""
    return (f"TTT-Linear scan workload {job.name}: {mode}, {grad}, {dt}, B={w.B} H={w.H} "
            f"T={w.T} d={w.d}{extra}")


def shard_rows(B: int, world: int, rank: int) -> tuple:
    """Contiguous block of batch rows owned by `rank` when a batch is split over
    `world` ranks (heads and masks follow their batch row, so nothing crosses
    ranks)."""
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def weak_scaling_value(units_per_rank: float, t_local: float, world: int, dist=None):
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    t_max = t_local
    if world > 1:
        import torch
        dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
        tt = torch.tensor([t_local], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        t_max = float(tt.item())
    return units_per_rank * world / t_max, t_max


def run_ours(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    from test_sequence_layers_02_b200 import build, ttt_scan
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    ttt_scan.lib()
    peaks = _peaks()
    flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    fp32_tflops, n_sm = _fp32_peak(device)

    job = Job(args.workload, device, seed_offset=1000 * rank)
    # --- headline: timed region ---
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        step_times = _time_job(job, args.steps, args.warmup, flush_buf)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    total = sum(step_times)
    value, t_max = weak_scaling_value(job.head_tokens_per_step * args.steps, total, world,
                                      dist if world > 1 else None)
    per_launch = total / (args.steps * job.launches_per_step())
    roof = _roofline(job, per_launch, peaks, fp32_tflops, n_sm)
    e2e = _e2e(job, max(2, min(args.steps, 5)), device)
    if world > 1:
        ev = torch.tensor([e2e["value"]], dtype=torch.float64, device=device)
        dist.all_reduce(ev, op=dist.ReduceOp.MIN)
        e2e["value"] = float(ev.item()) * world
    by_workload = {}
    if world == 1 and not args.headline_only:
        for name in args.extra:
            ej = DecodeJob(name, device) if name == "dec" else Job(name, device)
            ts = _time_job(ej, max(3, min(args.steps, 10)), args.warmup, flush_buf)
            tot = sum(ts)
            pl = tot / (len(ts) * ej.launches_per_step())
            by_workload[name] = {
                "workload": _workload_desc(ej),
                "value": ej.head_tokens_per_step * len(ts) / tot, "unit": "head-tokens/s",
                "ms_per_step": round(tot / len(ts) * 1e3, 4),
                "roofline": _roofline(ej, pl, peaks, fp32_tflops, n_sm),
                "chain_step_ns": round(pl / max(1, ej.w.n_chunks if ej.w.minibatch else ej.w.T) * 1e9, 2),
                "gpu_launches": ej.launches_per_step() * len(ts)}
            del ej
            torch.cuda.empty_cache()
    cpu = _cpu_baseline(job) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None
    if rank == 0:
        w = job.w
        line = {
            "metric": METRIC, "value": value, "unit": "head-tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t_max / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic (seeded numpy PCG64; no dataset)",
            "config": {"workload": _workload_desc(job), "B": w.B, "H": w.H, "T": w.T, "d": w.d,
                       "head_tokens_per_step": job.head_tokens_per_step,
                       "l2": "flushed between timed steps (256 MB device write, untimed)",
                       "passes": ("the two gradient forms run as two concurrent launches "
                                  "(one stream each) over the same resident inputs"
                                  if len(job.passes) == 2 else "one launch"),
                       "parallelism": f"heads sharded across {world} rank(s), no collective"},
            "roofline": roof,
            # the passes of a step run concurrently, so one chain step takes the
            # step time over the sequence length
            "chain_step_ns": round(t_max / args.steps / w.T * 1e9, 2),
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": job.launches_per_step() * args.steps,
            "clocks": clk.summary(),
            "fp32_probe_tflops": round(fp32_tflops, 2),
            "by_workload": by_workload,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The oracle (CPU, fp64) on the headline workload, as the reference arm (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from test_sequence_layers_02_b200.workloads import WORKLOADS, make_workload
    w = WORKLOADS["2s"]
    inp = make_workload(w)
    cores = len(os.sched_getaffinity(0))
    passes = [dict(lnjac=False), dict(lnjac=True)]
    # one step = both gradient forms over a sample of the heads, sized so that a
    # step takes about a second on this host (the full run stays within minutes)
    heads = min(w.heads, cores)
    t0 = time.perf_counter()
    _oracle_pass(w, inp, passes, heads, min(cores, heads))
    first = time.perf_counter() - t0
    if first > 3.0 and heads > 1:
        heads = max(1, int(heads * 3.0 / first))
    used = min(cores, heads)
    for _ in range(args.warmup):
        _oracle_pass(w, inp, passes, heads, used)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_pass(w, inp, passes, heads, used)
    el = time.perf_counter() - t0
    value = 2 * heads * w.T * args.steps / el
    sample = f"{heads} of {w.heads} heads x T={w.T} x 2 gradient forms per step, fp64"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "head-tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded numpy PCG64; no dataset)",
            "config": {"workload": "TTT-Linear scan workload 2: per-token, simplified + LN-Jacobian "
                                   "gradients, fp32 inputs, B=4 H=4 T=2048 d=64",
                       "sample": sample},
            "cpu_baseline": {"value": value, "unit": "head-tokens/s", "cores": used,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "head-tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


PROFILE_CASES = {
    # kernel -> (make_inputs kwargs, scan kwargs)
    "tc": (dict(B=4, H=16, T=8192, d=64, seed=7, random_affine=True, in_bf16=True),
           dict(eps=1e-6, minibatch=True, lnjac=True, b=16, out_bf16=True)),
    "simt": (dict(B=4, H=4, T=2048, d=64, seed=2, qk_l2norm=True),
             dict(eps=1e-6, minibatch=False, lnjac=True, b=16, out_bf16=False, single_cta=True)),
    "cluster": (dict(B=4, H=4, T=2048, d=64, seed=2, qk_l2norm=True),
                dict(eps=1e-6, minibatch=False, lnjac=True, b=16, out_bf16=False)),
    "decode": (None, None),
}


def run_profile_case(name: str):
    """One warm-up launch and one more launch of a scan kernel on a fixed
    case, for profiler captures (no timing)."""
    import torch
    from test_sequence_layers_02_b200 import build, ttt_scan
    from test_sequence_layers_02_b200.workloads import make_inputs
    build.build()
    if name == "decode":
        job = DecodeJob("dec", torch.device("cuda"))
        for _ in range(2):
            job.step()
        rc = ttt_scan.check_device_status()
        print(f"profile case {name}: status {ttt_scan.status_string(rc)}")
        if rc != ttt_scan.TTT_OK:
            raise SystemExit(1)
        return
    mk, kw = PROFILE_CASES[name]
    inp = make_inputs(**mk)
    bf = mk.get("in_bf16", False)

    def dev(key):
        a = inp.get(key)
        if a is None:
            return None
        if bf and key in ("q", "k", "v", "eta_logit", "gate_logit"):
            return torch.from_numpy(inp[key + "_bf16"].view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(np.ascontiguousarray(a)).cuda()

    t = {k: dev(k) for k in ("q", "k", "v", "eta_logit", "gate_logit", "W0", "gamma", "beta")}
    kw = dict(kw)
    out_dtype = torch.bfloat16 if kw.pop("out_bf16") else torch.float32
    for _ in range(2):
        ttt_scan.scan(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"], t["gamma"],
                      t["beta"], out_dtype=out_dtype, **kw)
    rc = ttt_scan.check_device_status()
    print(f"profile case {name}: status {ttt_scan.status_string(rc)}")
    if rc != ttt_scan.TTT_OK:
        raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="2", help="headline workload id (default 2)")
    ap.add_argument("--extra", nargs="*", default=["3", "4", "4pt", "5", "dec"],
                    help="other workloads measured on one GPU (by_workload)")
    ap.add_argument("--headline-only", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES),
                    help="run one kernel on a fixed case for a profiler capture and exit")
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args.profile_case)
        return
    if args.warmup < 3:
        print("note: at least 3 warm-up steps are required; using 3", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
