"""GPU parity of the scan's backward pass (``ttt_scan_backward``) against the
CPU oracle's backward (fp64, itself pinned by central finite differences of the
forward oracle): every gradient, per-token and mini-batch mode, every gradient
form, the gates, the mask, the SiLU variant, bf16 inputs and ragged tails.

The forward snapshots W_chunks the backward starts from come from the CUDA
forward (fp32 CUDA-core kernels), as in training. Tolerance: the fp32 bound
|gpu - ref| <= 2e-4 (1 + |ref|) elementwise on every gradient.
"""

import numpy as np
import pytest

import oracle
from test_sequence_layers_02_b200.workloads import make_inputs
from tests.helpers import assert_fp32_close, rel_rms, to_torch

pytestmark = pytest.mark.gpu

MINIB, LNJAC, NO_LN, GATE_CHANNEL, ABLATE, KQ_SILU = 1, 2, 4, 64, 1 << 8, 1 << 10


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from test_sequence_layers_02_b200 import build, ttt_scan
    build.build()
    ttt_scan.lib()


def _grads_draw(B, H, T, d, seed, with_dwt=True):
    rng = np.random.default_rng(seed)
    dO = rng.standard_normal((B, H, T, d)).astype(np.float32)
    dWT = (0.1 * rng.standard_normal((B, H, d, d))).astype(np.float32) if with_dwt else None
    return dO, dWT


def gpu_backward(inp, dO, dWT, *, mode, b, in_bf16=False, eps=1e-6, workspace=None):
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    t = to_torch(inp, "cuda", in_bf16)
    kw = dict(eps=eps, minibatch=bool(mode & MINIB), lnjac=bool(mode & LNJAC),
              no_ln=bool(mode & NO_LN), ablate=bool(mode & ABLATE), kq_silu=bool(mode & KQ_SILU),
              b=b, mask=t["mask"])
    _, _, Wc = ttt_scan.scan(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"],
                             t["gamma"], t["beta"], want_chunks=True, force_simt=True,
                             out_dtype=torch.float32, **kw)
    dO_t = torch.from_numpy(dO).cuda()
    dWT_t = None if dWT is None else torch.from_numpy(dWT).cuda()
    g = ttt_scan.scan_backward(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"],
                               t["gamma"], t["beta"], Wc, dO_t, dWT_t, workspace=workspace, **kw)
    torch.cuda.synchronize()
    assert ttt_scan.check_device_status() == ttt_scan.TTT_OK
    return {k_: (None if x is None else x.cpu().numpy().astype(np.float64)) for k_, x in g.items()}


def oracle_backward(inp, dO, dWT, *, mode, b, eps=1e-6):
    f = lambda a: None if a is None else np.asarray(a, dtype=np.float64)
    B, H, T, d = inp["q"].shape
    return oracle.backward(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["eta_logit"]),
                           f(inp["gate_logit"]), f(inp["W0"]), f(inp["gamma"]), f(inp["beta"]),
                           f(dO), f(dWT) if dWT is not None else np.zeros((B, H, d, d)),
                           eps=eps, mode=mode, b=b, mask=inp.get("mask"))


def compare(got, ref, what=""):
    for key in ("dq", "dk", "dv", "deta_logit", "dgate_logit", "dW0", "dgamma", "dbeta"):
        if ref[key] is None:
            assert got[key] is None, key
            continue
        assert_fp32_close(got[key], ref[key], f"{what} {key}")


CASES = [
    # (B, H, T, d, mode, b, in_bf16, gate)
    (2, 3, 53, 64, LNJAC, 16, False, "scalar"),
    (2, 3, 53, 64, 0, 16, False, "scalar"),
    (2, 2, 53, 64, NO_LN, 16, False, "scalar"),
    (2, 3, 53, 64, ABLATE, 16, False, "scalar"),
    (2, 3, 45, 16, LNJAC, 16, False, "scalar"),
    (2, 3, 45, 16, 0, 7, False, "channel"),
    (2, 3, 53, 64, LNJAC, 5, False, None),
    (2, 3, 53, 64, LNJAC, 16, True, "scalar"),
    (2, 3, 53, 64, LNJAC, 16, False, "channel"),
    (2, 3, 53, 64, LNJAC | KQ_SILU, 16, False, "scalar"),
    (2, 3, 53, 64, MINIB | LNJAC, 16, False, "scalar"),
    (2, 3, 53, 64, MINIB, 16, False, "scalar"),
    (2, 2, 53, 64, MINIB | NO_LN, 7, False, "scalar"),
    (2, 3, 53, 64, MINIB | ABLATE, 16, False, "channel"),
    (2, 3, 45, 16, MINIB | LNJAC, 5, False, "scalar"),
    (2, 3, 53, 64, MINIB | LNJAC, 16, True, "scalar"),
    (2, 3, 53, 64, MINIB | LNJAC | KQ_SILU, 16, False, None),
]


@pytest.mark.parametrize("with_mask", [False, True], ids=["nomask", "mask"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}H{c[1]}T{c[2]}d{c[3]}m{c[4]}b{c[5]}"
                         f"{'i16' if c[6] else ''}{c[7] or 'nogate'}")
def test_backward_matches_oracle(case, with_mask):
    B, H, T, d, mode, b, in_bf16, gate = case
    inp = make_inputs(B, H, T, d, seed=1000 + T + d + mode + b, random_affine=True,
                      in_bf16=in_bf16, gate=gate is not None, gate_channel=gate == "channel",
                      mask_p=0.5 if with_mask else None, b=b)
    if mode & KQ_SILU:
        inp["q"] = (0.7 * inp["q"]).astype(np.float32)   # stay in SiLU's curved range
    dO, dWT = _grads_draw(B, H, T, d, seed=2000 + T + d + mode)
    m = mode | (GATE_CHANNEL if gate == "channel" else 0)
    got = gpu_backward(inp, dO, dWT, mode=m, b=b, in_bf16=in_bf16)
    ref = oracle_backward(inp, dO, dWT, mode=m, b=b)
    compare(got, ref)
    if with_mask:
        skip = np.repeat(inp["mask"] == 0, b, axis=1)[:, :T]          # [B, T]
        assert np.all(got["deta_logit"][np.broadcast_to(skip[:, None, :], (B, H, T))] == 0.0)


def test_backward_larger_case():
    """A longer mini-batch problem (16 heads, T = 1024, bf16 inputs): relative
    RMS of every gradient within 1e-4, and the fp32 bound on dgamma, dbeta."""
    B, H, T, d, b = 2, 8, 1024, 64, 16
    inp = make_inputs(B, H, T, d, seed=3000, random_affine=True, in_bf16=True, mask_p=0.5, b=b)
    dO, dWT = _grads_draw(B, H, T, d, seed=3001)
    got = gpu_backward(inp, dO, dWT, mode=MINIB | LNJAC, b=b, in_bf16=True)
    ref = oracle_backward(inp, dO, dWT, mode=MINIB | LNJAC, b=b)
    for key in ("dq", "dk", "dv", "deta_logit", "dgate_logit", "dW0", "dgamma", "dbeta"):
        assert rel_rms(got[key], ref[key]) <= 1e-4, (key, rel_rms(got[key], ref[key]))
    assert_fp32_close(got["dgamma"], ref["dgamma"], "dgamma")
    assert_fp32_close(got["dbeta"], ref["dbeta"], "dbeta")


def test_backward_without_dWT_and_empty_cases():
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    B, H, T, d, b = 1, 2, 40, 64, 16
    inp = make_inputs(B, H, T, d, seed=3100, random_affine=True)
    dO, _ = _grads_draw(B, H, T, d, seed=3101, with_dwt=False)
    got = gpu_backward(inp, dO, None, mode=LNJAC, b=b)
    ref = oracle_backward(inp, dO, None, mode=LNJAC, b=b)
    compare(got, ref, "no dW_T")
    # T = 0: dW0 = dW_T and zero dgamma / dbeta
    inp0 = make_inputs(2, 3, 0, 64, seed=3102, random_affine=True)
    dWT = np.ones((2, 3, 64, 64), np.float32)
    got0 = gpu_backward(inp0, np.zeros((2, 3, 0, 64), np.float32), dWT, mode=LNJAC, b=16)
    assert np.array_equal(got0["dW0"], dWT.astype(np.float64))
    assert np.all(got0["dgamma"] == 0) and np.all(got0["dbeta"] == 0)
    # B = 0: zero gamma / beta gradients
    z = lambda *s: torch.zeros(*s, device="cuda")
    g = ttt_scan.scan_backward(z(0, 3, 8, 64), z(0, 3, 8, 64), z(0, 3, 8, 64), z(0, 3, 8), None,
                               torch.ones((3, 64), device="cuda"), z(3, 64),
                               z(0, 3, 2, 64, 64), z(0, 3, 8, 64), lnjac=True, b=8)
    torch.cuda.synchronize()
    assert torch.all(g["dgamma"] == 0) and g["dq"].shape == (0, 3, 8, 64)


def test_backward_is_deterministic_and_checks_its_workspace():
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    B, H, T, d, b = 4, 3, 37, 64, 16
    inp = make_inputs(B, H, T, d, seed=3200, random_affine=True, mask_p=0.5, b=b)
    dO, dWT = _grads_draw(B, H, T, d, seed=3201)
    a = gpu_backward(inp, dO, dWT, mode=LNJAC, b=b)
    c = gpu_backward(inp, dO, dWT, mode=LNJAC, b=b)
    for key in a:
        if a[key] is not None:
            assert np.array_equal(a[key], c[key]), key
    need = ttt_scan.backward_workspace_bytes(B, H, d)
    assert need == B * H * 2 * d * 4
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(ttt_scan.TTTScanError, match="INVALID"):
        gpu_backward(inp, dO, dWT, mode=LNJAC, b=b, workspace=small)
    with pytest.raises(ttt_scan.TTTScanError, match="UNSUPPORTED"):
        gpu_backward(make_inputs(1, 1, 40, 64, seed=1, b=32), np.zeros((1, 1, 40, 64), np.float32),
                     None, mode=LNJAC, b=32)
