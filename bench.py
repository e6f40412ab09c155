#!/usr/bin/env python
"""Throughput of the B200 TTT-Linear scan, as one JSON line.

Headline workload: workload 5, the largest single-GPU configuration (the long
gated mini-batch scan: B=2, H=32, T=32768, d=64, b=16, bf16 inputs, fp32 state,
a SKIP/UPDATE mask ~ Bernoulli(0.5) per chunk, LN-Jacobian gradient) on the
tcgen05 kernel. The metric is head-tokens per second (B*H*T per step) and the
fraction of the binding roofline of the kernel. On one GPU every other
workload is measured too and reported under ``by_workload`` with its own
roofline, CPU-oracle baseline and end-to-end figure: 1 (d = 16, per-token),
2 (per-token fp32, both gradient forms), 3 and 4 (mini-batch on tensor cores),
4pt (workload 4's per-token pass) and dec (the streaming decode step).

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
import sys
import threading
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "TTT-Linear scan head-tokens/sec at d=64 on 1 B200; % of binding roofline"
HEADLINE = "5"
EXTRA = ["1", "2", "3", "4", "4pt", "dec", "bwd2", "bwd3"]
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


# The files each kernel's binary is built from: the translation unit that
# instantiates it and everything that unit includes, plus (for every kernel)
# the launcher that sets its parameters, the public header and the build flags.
_KERNEL_SOURCES = {
    "scan_cluster": ["cluster.cu", "scan_cluster.cuh", "scan_simt.cuh", "launch.h", "common.cuh"],
    "scan_simt": ["simt.cu", "scan_simt.cuh", "launch.h", "common.cuh"],
    # one translation unit holds the tensor-core and decode kernels
    "scan_tc": ["scan_tc.cuh", "sm100.cuh", "decode.cuh", "scan_simt.cuh", "launch.h", "common.cuh"],
    "scan_tc_many": ["tc_many.cu", "scan_tc_many.cuh", "sm100.cuh", "launch.h", "common.cuh"],
    "decode_step": ["scan_tc.cuh", "sm100.cuh", "decode.cuh", "scan_simt.cuh", "launch.h",
                    "common.cuh"],
    "scan_bwd": ["backward.cu", "scan_bwd.cuh", "scan_simt.cuh", "abi_util.h", "common.cuh"],
}
# Captures: a kernel may have several (e.g. the tensor-core kernel with and
# without a SKIP/UPDATE mask); each names the kernel whose sources it covers.
_CAPTURE_KERNEL = {"scan_tc_masked": "scan_tc", "scan_simt_4pt": "scan_simt",
                   "scan_bwd_pertoken": "scan_bwd", "scan_bwd_minibatch": "scan_bwd"}


def _tc_takes_many(heads: int) -> bool:
    """Whether the tensor-core launcher picks its three-CTAs-per-SM kernel for
    this many heads: where that saves a wave, (waves at three per SM) * 1.5 <
    (waves at two per SM), the rule of the launcher in ttt_scan.cu."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    waves2 = -(-heads // (2 * sms))
    waves3 = -(-heads // (3 * sms))
    return 3 * waves3 < 2 * waves2


def _code_only(text: str) -> str:
    """C/C++ source without its comments (a comment edit leaves the binary alone)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def _kernel_hash(kernel_key: str) -> str:
    """Hash of what a kernel's binary is built from: its sources and includes
    (with ttt_scan.cu where that unit builds or configures it), the public
    header (comments stripped) and the compiler flags."""
    from test_sequence_layers_02_b200 import build
    kernel_key = _CAPTURE_KERNEL.get(kernel_key, kernel_key)
    pkg = ROOT / "test_sequence_layers_02_b200"
    # ttt_scan.cu builds the tensor-core and decode kernels and encodes the
    # tensor maps; the other kernels are objects of their own
    own = ["ttt_scan.cu"] if kernel_key in ("scan_tc", "scan_tc_many", "decode_step") else []
    files = sorted(set(_KERNEL_SOURCES[kernel_key] + own))
    paths = [pkg / "csrc" / f for f in files] + [ROOT / "include" / "ttt_scan.h"]
    h = hashlib.sha256()
    for p in paths:
        h.update(p.name.encode())
        h.update(_code_only(p.read_text()).encode())
    h.update(" ".join(build.NVCC_FLAGS).replace(str(ROOT), "").encode())
    return h.hexdigest()[:16]


def _traffic(capture_key: str, head_tokens_per_launch: int):
    """DRAM bytes (read + write) per launch from the committed ncu capture,
    scaled from its case by head-tokens; None if the kernel's sources changed
    since the capture (or it was never captured)."""
    if not PROFILE_TRAFFIC.exists():
        return None
    d = json.loads(PROFILE_TRAFFIC.read_text())
    e = d.get("kernels", {}).get(capture_key)
    if e is None or e.get("sources_hash") != _kernel_hash(capture_key):
        return None
    return round(e["bytes_per_head_token"] * head_tokens_per_launch)


# ---------------------------------------------------------------------------
# Workloads
# ---------------------------------------------------------------------------

def _dev_inputs(inp, w, device, decode=False):
    import torch

    def dev(key):
        a = inp.get(key)
        if a is None:
            return None
        if w.in_bf16 and key in ("q", "k", "v", "eta_logit", "gate_logit"):
            a = torch.from_numpy(inp[key + "_bf16"].view(np.int16)).view(torch.bfloat16)
        else:
            a = torch.from_numpy(np.ascontiguousarray(a))
        if decode and key in ("q", "k", "v", "eta_logit", "gate_logit"):
            a = a[:, :, 0].contiguous()
        return a.to(device)

    t = {k: dev(k) for k in ("q", "k", "v", "eta_logit", "gate_logit", "W0", "gamma", "beta")}
    m = inp.get("mask")
    t["mask"] = None if m is None else torch.from_numpy(np.ascontiguousarray(m)).to(device)
    return t


class Job:
    """One scan workload resident on the device, with its step function."""

    decode = False

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
        self.t = _dev_inputs(inp, w, device)
        self.out_dtype = torch.bfloat16 if w.out_bf16 else torch.float32
        self.outs = [(torch.empty(self.t["q"].shape, dtype=self.out_dtype, device=device),
                      torch.empty(self.t["W0"].shape, dtype=torch.float32, device=device))
                     for _ in self.passes]
        self.scan = ttt_scan.scan
        self.streams = None

    @property
    def head_tokens_per_step(self) -> int:
        return self.w.head_tokens * len(self.passes)

    def _call(self, t, ps, o, wt, stream=None):
        w = self.w
        return self.scan(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"],
                         t["gamma"], t["beta"], eps=w.eps, minibatch=w.minibatch, b=w.b,
                         mask=t["mask"], out_dtype=self.out_dtype, o=o, W_T=wt, stream=stream,
                         **ps)

    def step(self):
        """One step: every pass over the resident inputs. Independent passes (the
        two gradient forms of workload 2) run concurrently on their own streams."""
        import torch
        if len(self.passes) == 1:
            self._call(self.t, self.passes[0], *self.outs[0])
            return
        main = torch.cuda.current_stream()
        if self.streams is None:
            self.streams = [torch.cuda.Stream() for _ in self.passes]
        start = torch.cuda.Event()
        start.record(main)
        for st, ps, (o, wt) in zip(self.streams, self.passes, self.outs):
            st.wait_event(start)
            self._call(self.t, ps, o, wt, stream=st)
        for st in self.streams:
            ev = torch.cuda.Event()
            ev.record(st)
            main.wait_event(ev)

    def launches_per_step(self) -> int:
        return len(self.passes)

    def steps_per_chain(self) -> int:
        """Dependent steps of one head's recurrence (chunks, or tokens)."""
        return self.w.n_chunks if self.w.minibatch else self.w.T

    # --- algorithmic work per step -------------------------------------------------
    def update_fraction(self) -> float:
        return 1.0 if self.mask_np is None else float(self.mask_np.mean())

    def flops_per_step(self) -> float:
        w = self.w
        d, b = w.d, w.b
        if not w.minibatch:
            return 6.0 * d * d * w.head_tokens * len(self.passes)
        f_upd = 6.0 * d * d + 2.0 * d * (b + 1)
        f_skip = 2.0 * d * d
        frac = self.update_fraction()
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
        return "hbm" if (self.w.minibatch or self.w.d == 16) else "alu"

    def kernel_key(self) -> str:
        from test_sequence_layers_02_b200 import ttt_scan
        w = self.w
        k = ttt_scan.kernel_choice(w.B, w.H, w.T, w.d, minibatch=w.minibatch, lnjac=w.lnjac,
                                   in_bf16=w.in_bf16, out_bf16=w.out_bf16, b=w.b)
        return {ttt_scan.KERNEL_CUDA_CORE: "scan_simt",
                ttt_scan.KERNEL_CUDA_CORE_CLUSTER: "scan_cluster",
                ttt_scan.KERNEL_TENSOR_CORE: "scan_tc"}[k]

    def capture_key(self) -> str:
        k = self.kernel_key()
        if k == "scan_tc" and _tc_takes_many(self.w.B * self.w.H):
            return "scan_tc_many"
        if k == "scan_tc" and self.mask_np is not None:
            return "scan_tc_masked"
        if k == "scan_simt" and self.name == "4pt":
            return "scan_simt_4pt"
        return k

    # --- end to end ------------------------------------------------------------------
    def e2e_setup(self):
        """Pinned host copies of the inputs and of every pass's outputs."""
        import torch
        self.h_in = {k: (None if v is None else v.cpu().pin_memory()) for k, v in self.t.items()}
        self.h_out = [(torch.empty(self.t["q"].shape, dtype=self.out_dtype).pin_memory(),
                       torch.empty(self.t["W0"].shape, dtype=torch.float32).pin_memory())
                      for _ in self.passes]
        h2d = sum(v.numel() * v.element_size() for v in self.h_in.values() if v is not None)
        d2h = sum(o.numel() * o.element_size() + x.numel() * x.element_size()
                  for o, x in self.h_out)
        return h2d * len(self.passes), d2h

    def e2e_step(self):
        """Every pass through the public call with host buffers: the call copies
        its inputs in, scans and copies o and W_T back before returning."""
        for ps, (o, wt) in zip(self.passes, self.h_out):
            self._call(self.h_in, ps, o, wt)


class DecodeJob:
    """The streaming decode step over many heads, W updated in place each step."""

    decode = True

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
        self.t = _dev_inputs(inp, w, device, decode=True)
        self.out_dtype = torch.bfloat16 if w.out_bf16 else torch.float32
        self.o = torch.empty(self.t["q"].shape, dtype=self.out_dtype, device=device)
        self.step_fn = ttt_scan.decode_step

    @property
    def head_tokens_per_step(self) -> int:
        return self.w.heads

    def _call(self, t, W, o):
        w = self.w
        return self.step_fn(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], W,
                            t["gamma"], t["beta"], eps=w.eps, lnjac=w.lnjac,
                            out_dtype=self.out_dtype, o=o)

    def step(self):
        self._call(self.t, self.t["W0"], self.o)

    def launches_per_step(self) -> int:
        return 1

    def steps_per_chain(self) -> int:
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

    def capture_key(self) -> str:
        return "decode_step"

    def e2e_setup(self):
        import torch
        self.h_in = {k: (None if v is None else v.cpu().pin_memory()) for k, v in self.t.items()}
        self.h_o = torch.empty(self.t["q"].shape, dtype=self.out_dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in self.h_in.values() if v is not None)
        d2h = self.h_o.numel() * self.h_o.element_size() + \
            self.h_in["W0"].numel() * self.h_in["W0"].element_size()
        return h2d, d2h

    def e2e_step(self):
        """The public call with host buffers: the state W goes in and comes back
        updated, with the token's inputs in and o out."""
        self._call(self.h_in, self.h_in["W0"], self.h_o)


class BwdJob:
    """The backward pass of a scan workload (gradients of <dO, o> + <dW_T, W_T>
    for every input), from the forward's chunk snapshots; the forward runs once
    before timing, outside the timed region."""

    decode = False
    BWD_OF = {"bwd2": "2j", "bwd3": "3"}

    def __init__(self, name: str, device):
        import torch
        from test_sequence_layers_02_b200 import ttt_scan
        from test_sequence_layers_02_b200.workloads import WORKLOADS, make_workload
        self.name = name
        self.w = w = WORKLOADS[self.BWD_OF[name]]
        self.passes = [dict(lnjac=w.lnjac)]
        self.inp = make_workload(w)
        self.mask_np = self.inp.get("mask")
        self.t = _dev_inputs(self.inp, w, device)
        t = self.t
        rng = np.random.default_rng(w.seed + 77)
        self.t["dO"] = torch.from_numpy(
            rng.standard_normal((w.B, w.H, w.T, w.d), dtype=np.float32)).to(device)
        self.t["dW_T"] = torch.from_numpy(
            (0.1 * rng.standard_normal((w.B, w.H, w.d, w.d))).astype(np.float32)).to(device)
        self.kw = dict(eps=w.eps, minibatch=w.minibatch, lnjac=w.lnjac, b=w.b)
        _, _, self.t["W_chunks"] = ttt_scan.scan(
            t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"], t["gamma"],
            t["beta"], mask=t["mask"], want_chunks=True, force_simt=True,
            out_dtype=torch.float32, **self.kw)
        self.ws = torch.empty(ttt_scan.backward_workspace_bytes(w.B, w.H, w.d), dtype=torch.uint8,
                              device=device)
        self.bwd = ttt_scan.scan_backward
        torch.cuda.synchronize()

    @property
    def head_tokens_per_step(self) -> int:
        return self.w.head_tokens

    def _call(self, t):
        return self.bwd(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["gamma"],
                        t["beta"], t["W_chunks"], t["dO"], t["dW_T"], mask=t["mask"],
                        workspace=self.ws, **self.kw)

    def step(self):
        self.out = self._call(self.t)

    def launches_per_step(self) -> int:
        return 2  # the per-head kernel and the gamma / beta reduction

    def steps_per_chain(self) -> int:
        return self.w.T

    def update_fraction(self) -> float:
        return 1.0 if self.mask_np is None else float(self.mask_np.mean())

    def flops_per_step(self) -> float:
        # per head-token: the forward recomputed from W_s (W_s k, W_s q: 4 d^2),
        # D_e k (2 d^2), W_s^T dy, W_s^T dz, D_e^T G (6 d^2), the rank-2 update of
        # D (4 d^2); the O(b d) Gram terms are left out
        return 16.0 * self.w.d * self.w.d * self.w.head_tokens

    def bytes_per_step(self) -> float:
        w = self.w
        d = w.d
        ie = 2 if w.in_bf16 else 4
        per_tok = 3 * d * ie + 2 * ie + d * 4 + 3 * d * 4 + 2 * 4   # inputs, dO; dq, dk, dv, dlogits
        snaps = (w.n_chunks + 1) * d * d * 4 * w.heads               # W_chunks
        return float(per_tok * w.head_tokens + snaps + 2 * d * d * 4 * w.heads)

    def bound(self):
        return "alu"

    def kernel_key(self) -> str:
        return "scan_bwd"

    def capture_key(self) -> str:
        return "scan_bwd_minibatch" if self.w.minibatch else "scan_bwd_pertoken"

    def e2e_setup(self):
        """Pinned host copies of the inputs (with the forward's snapshots and dO)
        and of the gradients."""
        import torch
        self.h_in = {k: (None if v is None else v.cpu().pin_memory()) for k, v in self.t.items()}
        self.d_in = {k: (None if v is None else torch.empty_like(v)) for k, v in self.t.items()}
        out = self._call(self.t)
        self.h_out = {k: (None if v is None else torch.empty(v.shape, dtype=v.dtype).pin_memory())
                      for k, v in out.items()}
        h2d = sum(v.numel() * v.element_size() for v in self.h_in.values() if v is not None)
        d2h = sum(v.numel() * v.element_size() for v in self.h_out.values() if v is not None)
        return h2d, d2h

    def e2e_step(self):
        """Inputs in, the public backward call, every gradient back to the host."""
        import torch
        for k, v in self.h_in.items():
            if v is not None:
                self.d_in[k].copy_(v, non_blocking=True)
        out = self._call(self.d_in)
        for k, v in out.items():
            if v is not None:
                self.h_out[k].copy_(v, non_blocking=True)
        torch.cuda.current_stream().synchronize()


def _make_job(name, device, seed_offset=0):
    if name == "dec":
        return DecodeJob(name, device)
    if name in BwdJob.BWD_OF:
        return BwdJob(name, device)
    return Job(name, device, seed_offset)


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
    """Binding roofline of the job's kernel: HBM for the mini-batch, decode and
    d = 16 kernels, FP32 FMA (plain ALU arithmetic) for the per-token d = 64 ones."""
    launches = job.launches_per_step()
    head_tokens = job.head_tokens_per_step // launches
    traffic = _traffic(job.capture_key(), head_tokens)
    if job.bound() == "alu":
        flops = job.flops_per_step() / launches
        achieved = flops / per_launch_s / 1e12
        peak = n_sm * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12
        return {"bound": "alu", "achieved": round(achieved, 3), "peak": round(peak, 2),
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                "algorithmic_flops_per_launch": flops,
                "peak_basis": f"{n_sm} SM x 128 FP32 lanes x 2 x {peaks['sm_max_mhz']:.0f} MHz",
                "fp32_probe_tflops": round(fp32_meas_tflops, 2),
                "frac_of_probe": round(achieved / fp32_meas_tflops, 4),
                "kernel": job.kernel_key()}
    byts = job.bytes_per_step() / launches
    achieved = byts / per_launch_s / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": traffic, "kernel": job.kernel_key(),
            "algorithmic_bytes_per_launch": round(byts),
            "peak_basis": f"{peaks['source']} HBM copy bandwidth"}


# ---------------------------------------------------------------------------
# The oracle on the host cores (CPU baseline and reference arm)
# ---------------------------------------------------------------------------

def _oracle_heads(job, heads, threads):
    """One oracle run over the first `heads` heads of the workload (in batch-row
    order, OpenMP over heads), every pass (the backward job: the oracle's
    backward, one head after another)."""
    import oracle
    w, inp = job.w, job.inp
    if isinstance(job, BwdJob):
        rows = max(1, -(-heads // w.H))
        hh = min(heads, w.H)
        f64 = lambda a: None if a is None else np.asarray(a, dtype=np.float64)
        sel = lambda a: None if a is None else f64(a[:rows, :hh])
        m = inp.get("mask")
        oracle.backward(sel(inp["q"]), sel(inp["k"]), sel(inp["v"]), sel(inp["eta_logit"]),
                        sel(inp["gate_logit"]), sel(inp["W0"]), f64(inp["gamma"][:hh]),
                        f64(inp["beta"][:hh]), sel(job.t["dO"].cpu().numpy()),
                        sel(job.t["dW_T"].cpu().numpy()), eps=w.eps,
                        mode=(1 if w.minibatch else 0) | (2 if w.lnjac else 0), b=w.b,
                        mask=None if m is None else m[:rows])
        return rows * hh
    f64 = lambda a: None if a is None else np.asarray(a, dtype=np.float64)
    rows = max(1, -(-heads // w.H))
    hh = min(heads, w.H)
    # the decode workload's inputs hold one token per head already ([B, H, 1, ...])
    sel = lambda a: None if a is None else f64(a[:rows, :hh])
    m = inp.get("mask")
    for ps in job.passes:
        mode = (1 if w.minibatch else 0) | (2 if ps["lnjac"] else 0)
        oracle.forward(sel(inp["q"]), sel(inp["k"]), sel(inp["v"]), sel(inp["eta_logit"]),
                       sel(inp["gate_logit"]), sel(inp["W0"]), f64(inp["gamma"][:hh]),
                       f64(inp["beta"][:hh]), eps=w.eps, mode=mode, b=w.b,
                       mask=None if m is None else m[:rows], nthreads=threads)
    return rows * hh


def _oracle_sample(job, budget_s):
    """Time the oracle, as it stands, on a bounded sample of the workload: whole
    heads (all T tokens of each), as many as fill about `budget_s` seconds on the
    host's cores. Returns (head-tokens/s, cores, sample description)."""
    w = job.w
    cores = len(os.sched_getaffinity(0))
    T = 1 if job.decode else w.T
    heads = min(w.heads, cores)
    while True:
        # grow the sample (whole rows of heads) until it fills the budget
        t0 = time.perf_counter()
        done = _oracle_heads(job, heads, min(cores, heads))
        el = time.perf_counter() - t0
        if el >= 0.5 * budget_s or done >= w.heads:
            break
        heads = min(w.heads, max(2 * heads, int(heads * budget_s / max(el, 1e-3))))
    reps, ht = 1, done * T * len(job.passes)
    while el < budget_s and done >= w.heads and reps < 1000000:
        t1 = time.perf_counter()
        _oracle_heads(job, heads, min(cores, heads))
        el += time.perf_counter() - t1
        reps += 1
    used = 1 if isinstance(job, BwdJob) else min(cores, done)   # the backward oracle is serial
    sample = (f"{done} of {w.heads} heads x T={T} x {len(job.passes)} pass(es) x {reps} rep(s) "
              f"of workload {job.name}, fp64, OpenMP over heads on {used} of {cores} host cores, "
              f"{el:.1f} s")
    return ht * reps / el, used, sample


def _cpu_baseline(job, budget_s):
    v, cores, sample = _oracle_sample(job, budget_s)
    return {"value": v, "unit": "head-tokens/s", "cores": cores, "kind": "oracle",
            "sample": sample}


def _e2e(job, steps):
    """The same metric through the public call with HOST buffers: every step
    copies that step's inputs from pinned host memory, runs the kernel and
    copies the results (o, W_T, or the decode state W) back before the call
    returns."""
    import torch
    h2d, d2h = job.e2e_setup()
    job.e2e_step()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(steps):
        job.e2e_step()
    torch.cuda.synchronize()
    el = time.perf_counter() - t0
    return {"value": job.head_tokens_per_step * steps / el, "unit": "head-tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(el / steps * 1e3, 3)}


def _workload_desc(job):
    w = job.w
    if isinstance(job, BwdJob):
        mode = "mini-batch b=%d" % w.b if w.minibatch else "per-token"
        dt = "bf16 in" if w.in_bf16 else "fp32 in"
        extra = ", SKIP/UPDATE mask" if w.mask_p else ""
        return (f"TTT-Linear scan backward ({job.name}: the gradients of workload "
                f"{job.BWD_OF[job.name]}): {mode}, LN-Jacobian gradient, {dt}, fp32 gradients, "
                f"B={w.B} H={w.H} T={w.T} d={w.d}{extra}")
    if job.decode:
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


def _measure(job, steps, warmup, flush_buf, peaks, fp32_tflops, n_sm):
    ts = _time_job(job, steps, warmup, flush_buf)
    tot = sum(ts)
    per_launch = tot / (len(ts) * job.launches_per_step())
    return {
        "workload": _workload_desc(job),
        "value": job.head_tokens_per_step * len(ts) / tot, "unit": "head-tokens/s",
        "ms_per_step": round(tot / len(ts) * 1e3, 4),
        "roofline": _roofline(job, per_launch, peaks, fp32_tflops, n_sm),
        # the passes of a step run concurrently: one dependent step of a head's
        # chain takes the step time over the chain's length
        "chain_step_ns": round(tot / len(ts) / job.steps_per_chain() * 1e9, 2),
        "update_fraction": round(job.update_fraction(), 4) if not job.decode else None,
        "gpu_launches": job.launches_per_step() * len(ts)}, tot


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

    job = _make_job(args.workload, device, 1000 * rank)
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
    e2e = _e2e(job, max(2, min(args.steps, 5)))
    if world > 1:
        ev = torch.tensor([e2e["value"]], dtype=torch.float64, device=device)
        dist.all_reduce(ev, op=dist.ReduceOp.MIN)
        e2e["value"] = float(ev.item()) * world
    by_workload = {}
    if world == 1 and not args.headline_only:
        for name in args.extra:
            if name == args.workload:
                continue
            ej = _make_job(name, device)
            entry, _ = _measure(ej, max(3, min(args.steps, 10)), args.warmup, flush_buf, peaks,
                                fp32_tflops, n_sm)
            entry["e2e"] = _e2e(ej, 3)
            if not args.no_cpu_baseline:
                entry["cpu_baseline"] = _cpu_baseline(ej, args.cpu_budget_extra)
            by_workload[name] = entry
            del ej
            torch.cuda.empty_cache()
    cpu = (_cpu_baseline(job, args.cpu_budget)
           if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None)
    if rank == 0:
        w = job.w
        line = {
            "metric": METRIC, "value": value, "unit": "head-tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t_max / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.in_bf16 else "f32",
            "data": "synthetic (seeded numpy PCG64; no dataset)",
            "config": {"workload": _workload_desc(job), "B": w.B, "H": w.H, "T": w.T, "d": w.d,
                       "head_tokens_per_step": job.head_tokens_per_step,
                       "l2": "flushed between timed steps (256 MB device write, untimed)",
                       "passes": ("the two gradient forms run as two concurrent launches "
                                  "(one stream each) over the same resident inputs"
                                  if len(job.passes) == 2 else "one launch"),
                       "parallelism": f"heads sharded across {world} rank(s), no collective"},
            "roofline": roof,
            "chain_step_ns": round(t_max / args.steps / job.steps_per_chain() * 1e9, 2),
            "update_fraction": None if job.decode else round(job.update_fraction(), 4),
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


class _HostJob:
    """A workload's host inputs only (the reference arm needs no GPU)."""

    def __init__(self, name):
        from test_sequence_layers_02_b200.workloads import WORKLOADS, make_workload
        self.w = WORKLOADS["2s" if name == "2" else name]
        self.name = name
        self.decode = False
        self.passes = ([dict(lnjac=False), dict(lnjac=True)] if name == "2"
                       else [dict(lnjac=self.w.lnjac)])
        self.inp = make_workload(self.w)


def run_reference(args):
    """The oracle (CPU, fp64) on the headline workload, as the reference arm
    (rank 0 only): every step is a bounded sample of whole heads, sized so that
    a step takes a few seconds on this host."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    job = _HostJob(args.workload)
    w = job.w
    cores = len(os.sched_getaffinity(0))
    heads = min(w.heads, cores)
    t0 = time.perf_counter()
    _oracle_heads(job, heads, min(cores, heads))
    first = time.perf_counter() - t0
    if first > args.ref_step_s and heads > 1:
        heads = max(1, int(heads * args.ref_step_s / first))
    used = min(cores, heads)
    for _ in range(args.warmup):
        _oracle_heads(job, heads, used)
    t0 = time.perf_counter()
    done = 0
    for _ in range(args.steps):
        done = _oracle_heads(job, heads, used)
    el = time.perf_counter() - t0
    value = done * w.T * len(job.passes) * args.steps / el
    sample = (f"{done} of {w.heads} heads x T={w.T} x {len(job.passes)} pass(es) per step, fp64, "
              f"OpenMP over heads on {used} of {cores} host cores")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "head-tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded numpy PCG64; no dataset)",
            "config": {"workload": _workload_desc(job), "sample": sample},
            "cpu_baseline": {"value": value, "unit": "head-tokens/s", "cores": used,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "head-tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


PROFILE_CASES = {
    # name -> (make_inputs kwargs, scan kwargs)
    "tc": (dict(B=4, H=16, T=8192, d=64, seed=7, random_affine=True, in_bf16=True),
           dict(eps=1e-6, minibatch=True, lnjac=True, b=16, out_bf16=True)),
    # workload 5's kind of launch (mask ~ Bernoulli(0.5), one CTA per SM) at a
    # quarter of its length: inputs 268 MB > L2
    "tc_masked": (dict(B=2, H=32, T=8192, d=64, seed=5, random_affine=True, in_bf16=True,
                       mask_p=0.5, b=16),
                  dict(eps=1e-6, minibatch=True, lnjac=True, b=16, out_bf16=True)),
    # workload 4's mini-batch launch at its full size (384 heads: the kernel
    # built for three CTAs per SM); inputs 302 MB > L2
    "tc_many": (dict(B=16, H=24, T=2048, d=64, seed=4, random_affine=True, in_bf16=True),
                dict(eps=1e-6, minibatch=True, lnjac=True, b=16, out_bf16=True)),
    # workload 4's per-token pass at its full size (384 heads, one CTA per head)
    "simt_4pt": (dict(B=16, H=24, T=2048, d=64, seed=4, random_affine=True, in_bf16=True),
                 dict(eps=1e-6, minibatch=False, lnjac=True, b=16, out_bf16=False)),
    "simt": (dict(B=4, H=4, T=2048, d=64, seed=2, qk_l2norm=True),
             dict(eps=1e-6, minibatch=False, lnjac=True, b=16, out_bf16=False, single_cta=True)),
    "cluster": (dict(B=4, H=4, T=2048, d=64, seed=2, qk_l2norm=True),
                dict(eps=1e-6, minibatch=False, lnjac=True, b=16, out_bf16=False)),
    "decode": (None, None),
    # the backward pass at workload 2's shape, a quarter of its length (per-token,
    # LN Jacobian, fp32) and at workload 3's shape, a quarter of its length
    # (mini-batch, bf16 inputs); the forward's snapshots are taken first
    "bwd2": (dict(B=4, H=4, T=512, d=64, seed=2, qk_l2norm=True),
             dict(eps=1e-6, minibatch=False, lnjac=True, b=16)),
    "bwd3": (dict(B=8, H=12, T=1024, d=64, seed=3, random_affine=True, in_bf16=True),
             dict(eps=1e-6, minibatch=True, lnjac=True, b=16)),
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

    class _W:
        in_bf16 = mk.get("in_bf16", False)

    t = _dev_inputs(inp, _W, torch.device("cuda"))
    if name.startswith("bwd"):
        _, _, Wc = ttt_scan.scan(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"],
                                 t["gamma"], t["beta"], mask=t["mask"], want_chunks=True,
                                 force_simt=True, out_dtype=torch.float32, **kw)
        dO = torch.randn(t["q"].shape, dtype=torch.float32, device="cuda")
        for _ in range(2):
            ttt_scan.scan_backward(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"],
                                   t["gamma"], t["beta"], Wc, dO, None, mask=t["mask"], **kw)
        rc = ttt_scan.check_device_status()
        print(f"profile case {name}: status {ttt_scan.status_string(rc)}")
        if rc != ttt_scan.TTT_OK:
            raise SystemExit(1)
        return
    kw = dict(kw)
    out_dtype = torch.bfloat16 if kw.pop("out_bf16") else torch.float32
    for _ in range(2):
        ttt_scan.scan(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"], t["gamma"],
                      t["beta"], mask=t["mask"], out_dtype=out_dtype, **kw)
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
    ap.add_argument("--workload", default=HEADLINE, help="headline workload id (default 5)")
    ap.add_argument("--extra", nargs="*", default=EXTRA,
                    help="other workloads measured on one GPU (by_workload)")
    ap.add_argument("--headline-only", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of oracle work for the headline's CPU baseline")
    ap.add_argument("--cpu-budget-extra", type=float, default=3.0,
                    help="seconds of oracle work for each other workload's CPU baseline")
    ap.add_argument("--ref-step-s", type=float, default=4.0,
                    help="reference arm: about this many seconds of oracle work per step")
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
