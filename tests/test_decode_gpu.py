"""GPU parity of the streaming decode step (``ttt_decode_step``) against the
CPU oracle: single steps in every mode, the SKIP flag, chains of steps against
the per-token scan, the full-size decode workload, host buffers, edge cases."""

import numpy as np
import pytest

import oracle
from test_sequence_layers_02_b200.workloads import make_inputs
from tests.helpers import assert_fp32_close, to_torch

pytestmark = pytest.mark.gpu

LNJAC, NO_LN, GATE_CHANNEL = 2, 4, 64


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from test_sequence_layers_02_b200 import build, ttt_scan
    build.build()
    ttt_scan.lib()


def step_inputs(B, H, d, *, seed, in_bf16, gate="scalar", update_p=None):
    """One token per head: the t = 0 slice of a seeded problem."""
    inp = make_inputs(B, H, 1, d, seed=seed, random_affine=True, in_bf16=in_bf16,
                      gate=gate is not None, gate_channel=gate == "channel",
                      mask_p=update_p, b=1)
    out = {}
    for key, a in inp.items():
        if a is None or key in ("W0", "gamma", "beta", "mask"):
            out[key] = a
        else:
            out[key] = np.ascontiguousarray(a[:, :, 0])
    out["update"] = None if inp["mask"] is None else np.ascontiguousarray(inp["mask"][:, 0])
    return out


def gpu_step(inp, *, in_bf16, out_bf16, lnjac, no_ln, eps, W=None, kq_silu=False):
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    t = to_torch(inp, "cuda", in_bf16)
    W_dev = t["W0"].clone() if W is None else W
    upd = None if inp.get("update") is None else torch.from_numpy(inp["update"]).cuda()
    o = ttt_scan.decode_step(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], W_dev,
                             t["gamma"], t["beta"], eps=eps, lnjac=lnjac, no_ln=no_ln,
                             update=upd, kq_silu=kq_silu,
                             out_dtype=torch.bfloat16 if out_bf16 else torch.float32)
    torch.cuda.synchronize()
    assert ttt_scan.check_device_status() == ttt_scan.TTT_OK
    return o, W_dev


def oracle_step(inp, *, mode, eps, W=None):
    f = lambda a: None if a is None else np.asarray(a, dtype=np.float64)
    return oracle.decode_step(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["eta_logit"]),
                              f(inp["gate_logit"]), f(inp["W0"] if W is None else W),
                              f(inp["gamma"]), f(inp["beta"]), eps=eps, mode=mode,
                              update=inp.get("update"))


def np64(t):
    return t.float().cpu().numpy().astype(np.float64)


def assert_out_close(got, ref, out_bf16, what):
    """fp32 bound; a bf16 output adds its own rounding to nearest, half an ulp,
    which is at most 2^-8 of the value (bf16 keeps 8 significant bits)."""
    if not out_bf16:
        assert_fp32_close(got, ref, what)
        return
    bound = 2e-4 * (1 + np.abs(ref)) + 2.0 ** -8 * np.abs(ref)
    err = np.abs(got - ref)
    assert np.all(err <= bound), f"{what}: worst ratio {(err / bound).max():.3g}"


@pytest.mark.parametrize("d", [16, 64])
@pytest.mark.parametrize("grad", [LNJAC, 0, NO_LN], ids=["lnjac", "simple", "no_ln"])
@pytest.mark.parametrize("dtypes", [(False, False), (True, False), (True, True), (False, True)],
                         ids=["f32", "bf16in", "bf16io", "f32in_bf16out"])
@pytest.mark.parametrize("gate", ["scalar", "channel", None])
def test_decode_step_matches_oracle(d, grad, dtypes, gate):
    in_bf16, out_bf16 = dtypes
    B, H = 3, 5       # 15 heads: with d = 16 (4 heads per CTA) the last CTA is ragged
    inp = step_inputs(B, H, d, seed=500 + d + grad, in_bf16=in_bf16, gate=gate, update_p=0.7)
    mode = grad | (GATE_CHANNEL if gate == "channel" else 0)
    o, W = gpu_step(inp, in_bf16=in_bf16, out_bf16=out_bf16, lnjac=bool(grad & LNJAC),
                    no_ln=bool(grad & NO_LN), eps=1e-6)
    ro, rW = oracle_step(inp, mode=mode, eps=1e-6)
    assert_out_close(np64(o), ro, out_bf16, "o")
    assert_fp32_close(np64(W), rW, "W")


@pytest.mark.parametrize("norm_match", [False, True], ids=["ablate", "ablate_nm"])
@pytest.mark.parametrize("d", [16, 64])
def test_decode_ablation_gradient(d, norm_match):
    B, H = 3, 5
    inp = step_inputs(B, H, d, seed=540 + d, in_bf16=False, update_p=0.7)
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    t = to_torch(inp, "cuda", False)
    W = t["W0"].clone()
    o = ttt_scan.decode_step(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], W,
                             t["gamma"], t["beta"], eps=1e-6, ablate=True, norm_match=norm_match,
                             update=torch.from_numpy(inp["update"]).cuda())
    torch.cuda.synchronize()
    assert ttt_scan.check_device_status() == ttt_scan.TTT_OK
    ro, rW = oracle_step(inp, mode=(1 << 8) | ((1 << 9) if norm_match else 0), eps=1e-6)
    assert_fp32_close(np64(o), ro, "o")
    assert_fp32_close(np64(W), rW, "W")


def test_decode_skip_rows_keep_W_bit_for_bit():
    B, H, d = 6, 4, 64
    inp = step_inputs(B, H, d, seed=510, in_bf16=True, update_p=0.5)
    inp["update"] = np.array([1, 0, 1, 0, 0, 1], dtype=np.uint8)
    o, W = gpu_step(inp, in_bf16=True, out_bf16=False, lnjac=True, no_ln=False, eps=1e-6)
    W = W.cpu().numpy()
    for bi in range(B):
        same = np.array_equal(W[bi], inp["W0"][bi])
        assert same == (inp["update"][bi] == 0), bi
    ro, rW = oracle_step(inp, mode=LNJAC, eps=1e-6)
    assert_fp32_close(np64(o), ro, "o")


def test_decode_eta_zero_is_gated_readout():
    B, H, d = 2, 3, 64
    inp = step_inputs(B, H, d, seed=511, in_bf16=False)
    inp["eta_logit"] = np.full_like(inp["eta_logit"], -1e4)
    o, W = gpu_step(inp, in_bf16=False, out_bf16=False, lnjac=True, no_ln=False, eps=1e-6)
    assert np.array_equal(W.cpu().numpy(), inp["W0"])
    ref = (1 / (1 + np.exp(-inp["gate_logit"].astype(np.float64))))[..., None] * np.einsum(
        "bhrc,bhc->bhr", inp["W0"].astype(np.float64), inp["q"].astype(np.float64))
    assert_fp32_close(np64(o), ref, "o")


@pytest.mark.parametrize("grad", [LNJAC, 0])
@pytest.mark.parametrize("d", [16, 64])
def test_decode_chain_equals_per_token_scan(grad, d):
    """T single steps carrying W equal the per-token scan over the same T tokens."""
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    B, H, T = 2, 3, 40
    inp = make_inputs(B, H, T, d, seed=520 + d, random_affine=True, mask_p=0.7, b=1)
    ro, rW = oracle.forward(*(np.asarray(inp[k_], dtype=np.float64) for k_ in
                              ("q", "k", "v", "eta_logit", "gate_logit", "W0", "gamma", "beta")),
                            eps=1e-6, mode=grad, b=1, mask=inp["mask"])
    t = to_torch(inp, "cuda", False)
    W = t["W0"].clone()
    mask = torch.from_numpy(inp["mask"]).cuda()
    outs = []
    for s in range(T):
        outs.append(ttt_scan.decode_step(
            t["q"][:, :, s].contiguous(), t["k"][:, :, s].contiguous(),
            t["v"][:, :, s].contiguous(), t["eta_logit"][:, :, s].contiguous(),
            t["gate_logit"][:, :, s].contiguous(), W, t["gamma"], t["beta"], eps=1e-6,
            lnjac=bool(grad & LNJAC), update=mask[:, s].contiguous()))
    torch.cuda.synchronize()
    assert ttt_scan.check_device_status() == ttt_scan.TTT_OK
    o = torch.stack(outs, dim=2)
    assert_fp32_close(np64(o), ro, "o")
    assert_fp32_close(np64(W), rW, "W_T")
    # and against the CUDA per-token scan on the same inputs
    so, sW = ttt_scan.scan(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"],
                           t["gamma"], t["beta"], eps=1e-6, lnjac=bool(grad & LNJAC), b=1,
                           mask=mask)
    torch.cuda.synchronize()
    assert_fp32_close(np64(so), np64(o), "scan o vs decode o")


def test_decode_full_size_workload():
    """The benchmark's decode workload (B = 512, H = 32, d = 64, bf16 in/out,
    LN-Jacobian gradient), every head against the oracle."""
    B, H, d = 512, 32, 64
    inp = step_inputs(B, H, d, seed=7, in_bf16=True)
    o, W = gpu_step(inp, in_bf16=True, out_bf16=True, lnjac=True, no_ln=False, eps=1e-6)
    ro, rW = oracle_step(inp, mode=LNJAC, eps=1e-6)
    assert_out_close(np64(o), ro, True, "o")
    assert_fp32_close(np64(W), rW, "W")


def test_decode_host_buffers_end_to_end():
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    B, H, d = 4, 6, 64
    inp = step_inputs(B, H, d, seed=530, in_bf16=False, gate="channel", update_p=0.5)
    t = to_torch(inp, "cpu", False)
    W = t["W0"].clone().pin_memory()
    o = ttt_scan.decode_step(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], W,
                             t["gamma"], t["beta"], eps=1e-6, lnjac=True,
                             update=torch.from_numpy(inp["update"]))
    assert not o.is_cuda and not W.is_cuda
    ro, rW = oracle_step(inp, mode=LNJAC | GATE_CHANNEL, eps=1e-6)
    assert_fp32_close(o.numpy().astype(np.float64), ro, "o")
    assert_fp32_close(W.numpy().astype(np.float64), rW, "W")


def test_decode_empty_and_bad_arguments():
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    z = lambda *s: torch.zeros(*s, device="cuda")
    o = ttt_scan.decode_step(z(0, 3, 64), z(0, 3, 64), z(0, 3, 64), z(0, 3), None,
                             z(0, 3, 64, 64), z(3, 64), z(3, 64))
    assert o.shape == (0, 3, 64)
    with pytest.raises(ttt_scan.TTTScanError):
        ttt_scan.decode_step(z(1, 2, 32), z(1, 2, 32), z(1, 2, 32), z(1, 2), None,
                             z(1, 2, 32, 32), z(2, 32), z(2, 32))
    with pytest.raises(ValueError):
        ttt_scan.decode_step(z(1, 2, 64), z(1, 2, 64), z(1, 2, 64), z(1, 2), None,
                             z(1, 2, 64, 16), z(2, 64), z(2, 64))


@pytest.mark.parametrize("d", [16, 64])
@pytest.mark.parametrize("dtypes", [(False, False), (True, True)], ids=["f32", "bf16io"])
def test_decode_kq_silu_variant(d, dtypes):
    """The `:mlp` variant's decode step (SiLU on k and q) against the oracle."""
    in_bf16, out_bf16 = dtypes
    inp = step_inputs(3, 5, d, seed=560 + d, in_bf16=in_bf16, update_p=0.7)
    o, W = gpu_step(inp, in_bf16=in_bf16, out_bf16=out_bf16, lnjac=True, no_ln=False, eps=1e-6,
                    kq_silu=True)
    ro, rW = oracle_step(inp, mode=LNJAC | (1 << 10), eps=1e-6)
    assert_out_close(np64(o), ro, out_bf16, "o")
    assert_fp32_close(np64(W), rW, "W")
