"""Shared helpers of the parity tests: move seeded inputs to torch, run both sides,
compare with the stated tolerances."""

from __future__ import annotations

import numpy as np

FP32_ATOL = 2e-4   # |gpu - ref| <= 2e-4 * (1 + |ref|), elementwise (fp32 paths)
BF16_RRMS = 2e-2   # ||gpu - ref||_2 / ||ref||_2 (bf16 tensor-core paths)


def to_torch(inp: dict, device, in_bf16: bool):
    import torch

    def t(key):
        a = inp.get(key)
        if a is None:
            return None
        if in_bf16 and key in ("q", "k", "v", "eta_logit", "gate_logit"):
            bits = inp[key + "_bf16"]
            return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    out = {key: t(key) for key in ("q", "k", "v", "eta_logit", "gate_logit", "W0", "gamma", "beta")}
    m = inp.get("mask")
    out["mask"] = None if m is None else torch.from_numpy(np.ascontiguousarray(m)).to(device)
    return out


def gpu_scan(inp: dict, *, in_bf16: bool, out_bf16: bool = False, device="cuda", **kw):
    import torch
    from test_sequence_layers_02_b200 import ttt_scan

    t = to_torch(inp, device, in_bf16)
    res = ttt_scan.scan(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"],
                        t["gamma"], t["beta"], mask=t["mask"],
                        out_dtype=torch.bfloat16 if out_bf16 else torch.float32, **kw)
    torch.cuda.synchronize()
    assert ttt_scan.check_device_status() == ttt_scan.TTT_OK
    return tuple(None if x is None else x.float().cpu().numpy().astype(np.float64) for x in res)


def oracle_scan(inp: dict, *, eps, mode, b, want_chunks=False, mask="inp",
                want_grad_norms=False):
    import oracle

    m = inp.get("mask") if isinstance(mask, str) else mask
    f = lambda a: None if a is None else np.asarray(a, dtype=np.float64)
    return oracle.forward(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["eta_logit"]),
                          f(inp["gate_logit"]), f(inp["W0"]), f(inp["gamma"]), f(inp["beta"]),
                          eps=eps, mode=mode, b=b, mask=m, want_chunks=want_chunks,
                          want_grad_norms=want_grad_norms)


def assert_fp32_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    bound = FP32_ATOL * (1.0 + np.abs(ref))
    err = np.abs(got - ref)
    bad = err > bound
    if bad.any():
        idx = np.unravel_index(np.argmax(err / bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} elements out of tolerance; worst at {idx}: "
                             f"got {got[idx]!r} ref {ref[idx]!r} (ratio {(err / bound).max():.3g})")


def rel_rms(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def assert_rrms(got, ref, what="", tol=BF16_RRMS):
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    r = rel_rms(got, ref)
    assert r <= tol, f"{what}: relative RMS {r:.3e} > {tol}"
