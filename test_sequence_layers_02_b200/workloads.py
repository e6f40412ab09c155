"""Seeded synthetic inputs for the TTT-Linear scan.

This module only draws and stores numbers; it holds none of the scan's
arithmetic, and both the CUDA path's tests/benchmark and the CPU oracle take
their inputs from it.

Recipe (numpy PCG64, seed = workload id, draws in the order q, k, v, eta_logit,
gate_logit, W0, gamma, beta, mask; each draw is float32):

* q, k, v, eta_logit, gate_logit ~ N(0, 1); the gate is [B, H, T], or
  [B, H, T, d] for the per-channel gate.
* W0 ~ N(0, 0.02^2) -- the small initialisation of "Edifice.Recurrent.TTT",
  section "Paper-Faithful Implementation" (0.02 read as the standard deviation).
* gamma = 1, beta = 0, or per head gamma ~ N(1, 0.1^2), beta ~ N(0, 0.1^2).
* Optionally q and k are L2-normalised per token as x / (||x||_2 + 1e-6), the
  normalisation of cortex_rust src/layers/ttt.rs (forward_update); it is done
  here, in float32, before anything reaches the scan.
* Optionally the mask is Bernoulli(p) per (batch row, chunk of b tokens),
  1 = UPDATE (PonderTTT, "Core Idea: Binary Gating via Gumbel-Softmax").
* bf16 inputs are rounded to nearest-even from the float32 draws; the float32
  copy then holds exactly the bf16 values, so every consumer sees the same
  numbers.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bits to float32 exactly."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Workload:
    name: str
    B: int
    H: int
    T: int
    d: int
    b: int
    eps: float
    minibatch: bool
    lnjac: bool
    in_bf16: bool
    out_bf16: bool
    qk_l2norm: bool = False
    random_affine: bool = False
    mask_p: Optional[float] = None
    seed: int = 0
    gate: bool = True

    @property
    def heads(self) -> int:
        return self.B * self.H

    @property
    def head_tokens(self) -> int:
        return self.B * self.H * self.T

    @property
    def n_chunks(self) -> int:
        return -(-self.T // self.b)


# The five workloads of the scan, by id. Workload 4 has two passes over the
# same inputs: mini-batch on tensor cores ("4") and per-token ("4pt").
WORKLOADS = {
    "1": Workload("1", B=1, H=1, T=64, d=16, b=16, eps=1e-5, minibatch=False,
                  lnjac=False, in_bf16=False, out_bf16=False, seed=1),
    "2s": Workload("2s", B=4, H=4, T=2048, d=64, b=16, eps=1e-6, minibatch=False,
                   lnjac=False, in_bf16=False, out_bf16=False, qk_l2norm=True, seed=2),
    "2j": Workload("2j", B=4, H=4, T=2048, d=64, b=16, eps=1e-6, minibatch=False,
                   lnjac=True, in_bf16=False, out_bf16=False, qk_l2norm=True, seed=2),
    "3": Workload("3", B=8, H=12, T=4096, d=64, b=16, eps=1e-6, minibatch=True,
                  lnjac=True, in_bf16=True, out_bf16=True, random_affine=True, seed=3),
    "4": Workload("4", B=16, H=24, T=2048, d=64, b=16, eps=1e-6, minibatch=True,
                  lnjac=True, in_bf16=True, out_bf16=True, random_affine=True, seed=4),
    "4pt": Workload("4pt", B=16, H=24, T=2048, d=64, b=16, eps=1e-6, minibatch=False,
                    lnjac=True, in_bf16=True, out_bf16=False, random_affine=True, seed=4),
    "5": Workload("5", B=2, H=32, T=32768, d=64, b=16, eps=1e-6, minibatch=True,
                  lnjac=True, in_bf16=True, out_bf16=True, random_affine=True,
                  mask_p=0.5, seed=5),
}


# Streaming decode: one token for every (batch row, head), W carried in place.
# 16384 heads of d = 64 hold 256 MB of fp32 state, twice the L2.
DECODE_WORKLOADS = {
    "dec": Workload("dec", B=512, H=32, T=1, d=64, b=1, eps=1e-6, minibatch=False,
                    lnjac=True, in_bf16=True, out_bf16=True, random_affine=True, seed=7),
}


def make_inputs(B: int, H: int, T: int, d: int, *, seed: int, b: int = 16,
                qk_l2norm: bool = False, random_affine: bool = False,
                in_bf16: bool = False, mask_p: Optional[float] = None,
                gate: bool = True, w0_std: float = 0.02, gate_channel: bool = False) -> dict:
    """Draw one seeded problem.

    Returns a dict of host arrays. q, k, v, eta_logit, gate_logit, W0, gamma,
    beta are float32 (for bf16 inputs they hold the bf16 values exactly, and
    ``*_bf16`` keys hold the uint16 bits of q, k, v, eta_logit, gate_logit);
    ``mask`` is uint8 [B, ceil(T/b)] or None. ``gate_channel`` draws one gate
    logit per feature, [B, H, T, d], instead of one per token.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    shp = (B, H, T, d)
    q = rng.standard_normal(shp, dtype=np.float32)
    k = rng.standard_normal(shp, dtype=np.float32)
    v = rng.standard_normal(shp, dtype=np.float32)
    eta = rng.standard_normal((B, H, T), dtype=np.float32)
    gshape = (B, H, T, d) if gate_channel else (B, H, T)
    gl = rng.standard_normal(gshape, dtype=np.float32) if gate else None
    W0 = (rng.standard_normal((B, H, d, d), dtype=np.float32) * np.float32(w0_std))
    if random_affine:
        gamma = (np.float32(1) + np.float32(0.1) * rng.standard_normal((H, d), dtype=np.float32))
        beta = np.float32(0.1) * rng.standard_normal((H, d), dtype=np.float32)
    else:
        gamma = np.ones((H, d), dtype=np.float32)
        beta = np.zeros((H, d), dtype=np.float32)
    mask = None
    if mask_p is not None:
        n_chunks = -(-T // b)
        mask = (rng.random((B, n_chunks)) < mask_p).astype(np.uint8)
    if qk_l2norm:
        for x in (q, k):
            nrm = np.sqrt(np.sum(x * x, axis=-1, keepdims=True, dtype=np.float32))
            x /= (nrm + np.float32(1e-6))
    out = dict(q=q, k=k, v=v, eta_logit=eta, gate_logit=gl, W0=W0.astype(np.float32),
               gamma=gamma.astype(np.float32), beta=beta.astype(np.float32), mask=mask)
    if in_bf16:
        for key in ("q", "k", "v", "eta_logit", "gate_logit"):
            if out[key] is None:
                out[key + "_bf16"] = None
                continue
            bits = f32_to_bf16_bits(out[key])
            out[key + "_bf16"] = bits
            out[key] = bf16_bits_to_f32(bits).reshape(out[key].shape)
    return out


def make_workload(w: Workload | str, **overrides) -> dict:
    """Inputs of one named workload (optionally with its sizes overridden)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    if overrides:
        w = dataclasses.replace(w, **overrides)
    return make_inputs(w.B, w.H, w.T, w.d, seed=w.seed, b=w.b, qk_l2norm=w.qk_l2norm,
                       random_affine=w.random_affine, in_bf16=w.in_bf16,
                       mask_p=w.mask_p, gate=w.gate)
