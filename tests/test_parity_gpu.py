"""GPU parity: the CUDA path against the CPU oracle on the same seeded inputs.

Tolerances: fp32 per-token / CUDA-core paths |gpu - ref| <= 2e-4 (1 + |ref|)
elementwise on o and W_T; bf16-output tensor-core paths relative RMS <= 2e-2;
SKIP chunks bit-exact via the W_chunks snapshots.
"""

import numpy as np
import pytest

from test_sequence_layers_02_b200.workloads import WORKLOADS, make_inputs, make_workload
from tests.helpers import assert_fp32_close, assert_rrms, gpu_scan, oracle_scan, rel_rms

pytestmark = pytest.mark.gpu

LNJAC, MINIB, NO_LN = 2, 1, 4


def _mode(w):
    return (MINIB if w.minibatch else 0) | (LNJAC if w.lnjac else 0)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from test_sequence_layers_02_b200 import build, ttt_scan
    build.build()
    ttt_scan.lib()


# ---------------------------------------------------------------------------
# The named workloads at their full sizes.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("single_cta", [False, True], ids=["auto", "single_cta"])
@pytest.mark.parametrize("name", ["1", "2s", "2j"])
def test_workload_fp32_full(name, single_cta):
    from test_sequence_layers_02_b200 import ttt_scan
    w = WORKLOADS[name]
    if single_cta and w.d != 64:
        pytest.skip("d = 16 always runs one CTA per head")
    if w.d == 64:
        want = ttt_scan.KERNEL_CUDA_CORE if single_cta else ttt_scan.KERNEL_CUDA_CORE_CLUSTER
        assert ttt_scan.kernel_choice(w.B, w.H, w.T, w.d, lnjac=w.lnjac,
                                      single_cta=single_cta) == want
    inp = make_workload(w)
    o, W_T = gpu_scan(inp, in_bf16=False, eps=w.eps, lnjac=w.lnjac, b=w.b, single_cta=single_cta)
    ro, rW = oracle_scan(inp, eps=w.eps, mode=_mode(w), b=w.b)
    assert_fp32_close(o, ro, f"{name} o")
    assert_fp32_close(W_T, rW, f"{name} W_T")


def _oracle_rows(w, inp, rows, mode):
    """The oracle over batch rows [rows[0], rows[1]) of a full-size workload
    (every head of those rows; OpenMP over the heads)."""
    import oracle
    a, z = rows
    f = lambda x: None if x is None else np.asarray(x[a:z], dtype=np.float64)
    m = inp.get("mask")
    return oracle.forward(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["eta_logit"]),
                          f(inp["gate_logit"]), f(inp["W0"]), np.asarray(inp["gamma"], np.float64),
                          np.asarray(inp["beta"], np.float64), eps=w.eps, mode=mode, b=w.b,
                          mask=None if m is None else m[a:z])


def _full_compare(w, inp, o, W_T, fp32):
    """Every head of the workload against the oracle, a few batch rows per
    oracle call (about 2^20 head-tokens each, so host memory stays bounded). fp32: the elementwise bound on all of o
    and W_T. bf16: relative RMS over the WHOLE tensors (o, then W_T), and the
    same bound on every head as an extra check."""
    mode = _mode(w)
    rows_per_call = max(1, (1 << 20) // (w.H * max(1, w.T)))
    sq = {"o": [0.0, 0.0], "W_T": [0.0, 0.0]}
    for a in range(0, w.B, rows_per_call):
        z = min(w.B, a + rows_per_call)
        ro, rW = _oracle_rows(w, inp, (a, z), mode)
        go, gW = o[a:z], W_T[a:z]
        if fp32:
            assert_fp32_close(go, ro, f"{w.name} o[{a}:{z}]")
            assert_fp32_close(gW, rW, f"{w.name} W_T[{a}:{z}]")
            continue
        for nm, g, r in (("o", go, ro), ("W_T", gW, rW)):
            assert np.all(np.isfinite(g)), f"{w.name} {nm}: non-finite values"
            sq[nm][0] += float(np.sum((g - r) ** 2))
            sq[nm][1] += float(np.sum(r ** 2))
            for bi in range(z - a):
                for h in range(w.H):
                    assert_rrms(g[bi, h], r[bi, h], f"{w.name} {nm}[{a + bi},{h}]")
    if not fp32:
        for nm, (num, den) in sq.items():
            r = np.sqrt(num / den)
            assert r <= 2e-2, f"{w.name} {nm}: whole-tensor relative RMS {r:.3e} > 2e-2"


def test_workload_4pt_per_token_bf16_in_fp32_out_all_heads():
    """All 384 heads of the per-token pass of workload 4 (bf16 in, fp32 out),
    elementwise fp32 bound on o and W_T."""
    w = WORKLOADS["4pt"]
    inp = make_workload(w)
    o, W_T = gpu_scan(inp, in_bf16=True, out_bf16=False, eps=w.eps, lnjac=True, b=w.b)
    _full_compare(w, inp, o, W_T, fp32=True)


@pytest.mark.parametrize("name", ["3", "4", "5"])
def test_workload_minibatch_bf16_all_heads(name):
    """Every head of the mini-batch workloads against the oracle: relative RMS
    of the whole o and W_T (and of every head's) within 2e-2."""
    w = WORKLOADS[name]
    inp = make_workload(w)
    o, W_T = gpu_scan(inp, in_bf16=True, out_bf16=True, eps=w.eps, lnjac=True, minibatch=True, b=w.b)
    _full_compare(w, inp, o, W_T, fp32=False)


def test_workload_5_skip_chunks_bit_exact_full_size():
    """At workload 5's full size (64 heads, 2048 chunks each), the W snapshot
    after a chunk equals the one before it bit for bit exactly on the SKIP
    chunks of its batch row, and differs on every UPDATE chunk (checked on the
    device: the snapshots take 2.1 GB)."""
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    from tests.helpers import to_torch
    w = WORKLOADS["5"]
    inp = make_workload(w)
    t = to_torch(inp, "cuda", True)
    o, W_T, Wc = ttt_scan.scan(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"],
                               t["gamma"], t["beta"], eps=w.eps, minibatch=True, lnjac=True,
                               b=w.b, mask=t["mask"], out_dtype=torch.bfloat16, want_chunks=True)
    torch.cuda.synchronize()
    assert ttt_scan.check_device_status() == ttt_scan.TTT_OK
    same = torch.all((Wc[:, :, 1:] == Wc[:, :, :-1]).flatten(3), dim=3)   # [B, H, n_chunks]
    skip = (t["mask"] == 0)[:, None, :].expand_as(same)
    assert torch.equal(same, skip)
    assert torch.equal(Wc[:, :, -1], W_T)
    assert torch.equal(Wc[:, :, 0], t["W0"])


# ---------------------------------------------------------------------------
# Small cases: several chunks, ragged tails, every mode and dtype mix.
# ---------------------------------------------------------------------------

CASES = [
    # (B, H, T, d, mode, b, in_bf16, out_bf16)
    (2, 3, 53, 16, 0, 16, False, False),
    (2, 3, 53, 16, LNJAC, 16, False, False),
    (2, 3, 53, 16, NO_LN, 16, False, False),
    (2, 3, 77, 64, 0, 16, False, False),
    (2, 3, 77, 64, LNJAC, 16, False, False),
    (1, 2, 77, 64, NO_LN, 16, False, False),
    (2, 2, 70, 64, LNJAC, 24, False, False),     # internal chunk 12 (divides b) with a mask
    (1, 2, 40, 64, LNJAC, 17, False, False),     # prime b: internal chunk 1
    (2, 3, 77, 64, LNJAC, 16, True, False),
    (2, 3, 77, 64, LNJAC, 16, True, True),
    (2, 3, 77, 64, 0, 16, False, True),
    (2, 3, 53, 64, MINIB | LNJAC, 16, False, False),
    (2, 3, 53, 64, MINIB | LNJAC, 7, False, False),
    (2, 3, 53, 64, MINIB, 16, False, False),
    (2, 2, 53, 64, MINIB | NO_LN, 5, False, False),
    (2, 3, 53, 16, MINIB | LNJAC, 16, False, False),
    (2, 3, 53, 64, MINIB | LNJAC, 16, True, False),
]


@pytest.mark.parametrize("single_cta", [False, True], ids=["auto", "single_cta"])
@pytest.mark.parametrize("with_mask", [False, True])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}H{c[1]}T{c[2]}d{c[3]}m{c[4]}b{c[5]}"
                         f"{'i16' if c[6] else ''}{'o16' if c[7] else ''}")
def test_small_cases(case, with_mask, single_cta):
    """Per-token d = 64 cases run on the cluster kernel ("auto": few heads) and on
    the one-CTA-per-head kernel ("single_cta"); the rest on their only kernel."""
    B, H, T, d, mode, b, in_bf16, out_bf16 = case
    per_token64 = d == 64 and not (mode & MINIB)
    if single_cta and not per_token64:
        pytest.skip("same kernel as the auto case")
    if per_token64:
        from test_sequence_layers_02_b200 import ttt_scan
        got = ttt_scan.kernel_choice(B, H, T, d, lnjac=bool(mode & LNJAC), no_ln=bool(mode & NO_LN),
                                     in_bf16=in_bf16, out_bf16=out_bf16, b=b, single_cta=single_cta)
        assert got == (ttt_scan.KERNEL_CUDA_CORE if single_cta else ttt_scan.KERNEL_CUDA_CORE_CLUSTER)
    inp = make_inputs(B, H, T, d, seed=100 + T + d + mode + b, random_affine=True,
                      in_bf16=in_bf16, mask_p=0.5 if with_mask else None, b=b)
    eps = 1e-6
    o, W_T, Wc = gpu_scan(inp, in_bf16=in_bf16, out_bf16=out_bf16, eps=eps, b=b,
                          lnjac=bool(mode & LNJAC), minibatch=bool(mode & MINIB),
                          no_ln=bool(mode & NO_LN), force_simt=True, want_chunks=True,
                          single_cta=single_cta)
    ro, rW, rWc = oracle_scan(inp, eps=eps, mode=mode, b=b, want_chunks=True)
    if out_bf16:
        assert_rrms(o, ro, "o", tol=1e-2)
        assert_fp32_close(W_T, rW, "W_T")
    else:
        assert_fp32_close(o, ro, "o")
        assert_fp32_close(W_T, rW, "W_T")
    assert_fp32_close(Wc, rWc, "W_chunks")
    if with_mask:
        m = inp["mask"]
        for bi in range(B):
            for c in range(m.shape[1]):
                same = np.array_equal(Wc[bi, :, c + 1], Wc[bi, :, c])
                assert same == (m[bi, c] == 0), (bi, c, m[bi, c])


def test_minibatch_b1_equals_per_token_on_gpu():
    inp = make_inputs(2, 2, 45, 64, seed=7, random_affine=True)
    o1, W1 = gpu_scan(inp, in_bf16=False, eps=1e-6, lnjac=True, b=1)
    o2, W2 = gpu_scan(inp, in_bf16=False, eps=1e-6, lnjac=True, b=1, minibatch=True)
    assert_fp32_close(o2, o1, "o")
    assert_fp32_close(W2, W1, "W_T")


def test_eta_zero_and_no_gate():
    inp = make_inputs(2, 2, 37, 64, seed=8, random_affine=True)
    inp["eta_logit"] = np.full_like(inp["eta_logit"], -1e4)
    inp["gate_logit"] = None
    for mb in (False, True):
        o, W_T = gpu_scan(inp, in_bf16=False, eps=1e-6, lnjac=True, minibatch=mb, force_simt=True)
        assert np.array_equal(W_T, inp["W0"].astype(np.float64))
        ref = np.einsum("bhrc,bhtc->bhtr", inp["W0"].astype(np.float64), inp["q"].astype(np.float64))
        assert_fp32_close(o, ref, "o")


def test_empty_and_single_token():
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    # T = 0: W_T = W0, no outputs
    inp = make_inputs(2, 2, 0, 64, seed=9)
    o, W_T = gpu_scan(inp, in_bf16=False, eps=1e-6)
    assert o.shape == (2, 2, 0, 64)
    assert np.array_equal(W_T, inp["W0"].astype(np.float64))
    # T = 1
    inp = make_inputs(1, 3, 1, 64, seed=10, random_affine=True)
    for mode in (0, LNJAC, MINIB | LNJAC):
        o, W_T = gpu_scan(inp, in_bf16=False, eps=1e-6, lnjac=bool(mode & LNJAC),
                          minibatch=bool(mode & MINIB), force_simt=True)
        ro, rW = oracle_scan(inp, eps=1e-6, mode=mode, b=16)
        assert_fp32_close(o, ro, "o")
        assert_fp32_close(W_T, rW, "W_T")
    # B*H = 0
    q = torch.empty((0, 4, 8, 64), device="cuda")
    z = torch.empty((0, 4, 8), device="cuda")
    o, W_T = ttt_scan.scan(q, q, q, z, z, torch.empty((0, 4, 64, 64), device="cuda"),
                           torch.ones((4, 64), device="cuda"), torch.zeros((4, 64), device="cuda"))
    assert o.shape == (0, 4, 8, 64)


def test_in_place_W_T_and_chaining():
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    from tests.helpers import to_torch
    B, H, T1, T2, d, b = 2, 2, 48, 29, 64, 16
    inp = make_inputs(B, H, T1 + T2, d, seed=11, random_affine=True, mask_p=0.5, b=b)
    t = to_torch(inp, "cuda", False)
    for mb in (False, True):
        kw = dict(eps=1e-6, lnjac=True, minibatch=mb, b=b, force_simt=True)
        o, W_T = ttt_scan.scan(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"],
                               t["gamma"], t["beta"], mask=t["mask"], **kw)
        n1 = T1 // b
        W = t["W0"].clone()
        sl = lambda x, a, z: x[:, :, a:z].contiguous()
        oa, _ = ttt_scan.scan(sl(t["q"], 0, T1), sl(t["k"], 0, T1), sl(t["v"], 0, T1),
                              sl(t["eta_logit"], 0, T1), sl(t["gate_logit"], 0, T1), W,
                              t["gamma"], t["beta"], mask=t["mask"][:, :n1].contiguous(),
                              W_T=W, **kw)                           # in place
        ob, Wb = ttt_scan.scan(sl(t["q"], T1, None), sl(t["k"], T1, None), sl(t["v"], T1, None),
                               sl(t["eta_logit"], T1, None), sl(t["gate_logit"], T1, None), W,
                               t["gamma"], t["beta"], mask=t["mask"][:, n1:].contiguous(), **kw)
        torch.cuda.synchronize()
        # the look-ahead form rounds differently at a resume point, so the two
        # runs agree to the fp32 tolerance rather than bit for bit
        assert_fp32_close(torch.cat([oa, ob], dim=2).cpu().numpy(), o.cpu().numpy(), "o")
        assert_fp32_close(Wb.cpu().numpy(), W_T.cpu().numpy(), "W_T")


def test_host_buffers_match_device_path():
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    inp = make_inputs(2, 3, 64, 64, seed=12, random_affine=True)
    cpu = {k: (None if v is None else torch.from_numpy(np.ascontiguousarray(v)))
           for k, v in inp.items() if not k.endswith("_bf16")}
    o_h, W_h = ttt_scan.scan(cpu["q"], cpu["k"], cpu["v"], cpu["eta_logit"], cpu["gate_logit"],
                             cpu["W0"], cpu["gamma"], cpu["beta"], eps=1e-6, lnjac=True)
    assert not o_h.is_cuda
    o_d, W_d = gpu_scan(inp, in_bf16=False, eps=1e-6, lnjac=True)
    assert np.array_equal(o_h.numpy().astype(np.float64), o_d)
    assert np.array_equal(W_h.numpy().astype(np.float64), W_d)


def test_binding_rejects_bad_shapes():
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    q = torch.zeros((1, 1, 8, 64), device="cuda")
    with pytest.raises(ValueError):
        ttt_scan.scan(q, q, q, torch.zeros((1, 1, 7), device="cuda"), None,
                      torch.zeros((1, 1, 64, 64), device="cuda"), None, None, no_ln=True)
    with pytest.raises(ttt_scan.TTTScanError) as e:
        ttt_scan.scan(q, q, q, torch.zeros((1, 1, 8), device="cuda"), None,
                      torch.zeros((1, 1, 64, 64), device="cuda"), None, None)   # LN needs gamma
    assert e.value.status == ttt_scan.TTT_ERR_INVALID_ARG


def test_cluster_wait_timeout_reports_and_recovers():
    """With a wait limit of 0 the cluster kernel's bounded waits for its peers'
    P give up at once: the call must report TTT_ERR_DEVICE_TIMEOUT (no hang, no
    trap) and the context must stay usable for a normal call afterwards."""
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    from tests.helpers import to_torch
    inp = make_inputs(1, 2, 80, 64, seed=13, random_affine=True)
    assert ttt_scan.kernel_choice(1, 2, 80, 64, lnjac=True) == ttt_scan.KERNEL_CUDA_CORE_CLUSTER
    t = to_torch(inp, "cuda", False)
    args = (t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"], t["gamma"], t["beta"])
    ttt_scan.set_wait_limit(0)
    try:
        ttt_scan.scan(*args, eps=1e-6, lnjac=True)
        assert ttt_scan.check_device_status() == ttt_scan.TTT_ERR_DEVICE_TIMEOUT
    finally:
        ttt_scan.set_wait_limit(1 << 20)
    assert ttt_scan.check_device_status() == ttt_scan.TTT_OK
    o, W_T = ttt_scan.scan(*args, eps=1e-6, lnjac=True)
    torch.cuda.synchronize()
    assert ttt_scan.check_device_status() == ttt_scan.TTT_OK
    ro, rW = oracle_scan(inp, eps=1e-6, mode=LNJAC, b=16)
    assert_fp32_close(o.cpu().numpy(), ro, "o")
    assert_fp32_close(W_T.cpu().numpy(), rW, "W_T")


# ---------------------------------------------------------------------------
# Ablation gradient ("Error Correction in Trained TTT Layers", Abstract): the
# prediction's contribution removed, the LayerNorm Jacobian kept, optionally
# rescaled per token to the full gradient's norm. Per-token mode.
# ---------------------------------------------------------------------------

ABLATE, NORM_MATCH = 1 << 8, 1 << 9


@pytest.mark.parametrize("single_cta", [False, True], ids=["auto", "single_cta"])
@pytest.mark.parametrize("norm_match", [False, True], ids=["ablate", "ablate_nm"])
@pytest.mark.parametrize("case", [(2, 3, 53, 16, 16, False), (2, 3, 77, 64, 16, False),
                                  (2, 2, 70, 64, 24, False), (2, 3, 77, 64, 16, True)],
                         ids=lambda c: f"B{c[0]}H{c[1]}T{c[2]}d{c[3]}b{c[4]}{'i16' if c[5] else ''}")
@pytest.mark.parametrize("with_mask", [False, True])
def test_ablation_gradient_small_cases(case, norm_match, with_mask, single_cta):
    """Per-token ablation on the cluster kernel (d = 64, few heads) and on one
    CTA per head."""
    from test_sequence_layers_02_b200 import ttt_scan
    B, H, T, d, b, in_bf16 = case
    if single_cta and d != 64:
        pytest.skip("d = 16 always runs one CTA per head")
    want = (ttt_scan.KERNEL_CUDA_CORE if (single_cta or d != 64)
            else ttt_scan.KERNEL_CUDA_CORE_CLUSTER)
    assert ttt_scan.kernel_choice(B, H, T, d, ablate=True, norm_match=norm_match,
                                  in_bf16=in_bf16, single_cta=single_cta) == want
    inp = make_inputs(B, H, T, d, seed=600 + T + d + b, random_affine=True, in_bf16=in_bf16,
                      mask_p=0.5 if with_mask else None, b=b)
    mode = ABLATE | (NORM_MATCH if norm_match else 0)
    o, W_T, Wc = gpu_scan(inp, in_bf16=in_bf16, eps=1e-6, b=b, ablate=True,
                          norm_match=norm_match, want_chunks=True, single_cta=single_cta)
    ro, rW, rWc = oracle_scan(inp, eps=1e-6, mode=mode, b=b, want_chunks=True)
    assert_fp32_close(o, ro, "o")
    assert_fp32_close(W_T, rW, "W_T")
    assert_fp32_close(Wc, rWc, "W_chunks")


@pytest.mark.parametrize("norm_match", [False, True], ids=["ablate", "ablate_nm"])
def test_ablation_gradient_headline_shape(norm_match):
    w = WORKLOADS["2j"]
    inp = make_workload(w)
    mode = ABLATE | (NORM_MATCH if norm_match else 0)
    o, W_T = gpu_scan(inp, in_bf16=False, eps=w.eps, b=w.b, ablate=True, norm_match=norm_match)
    ro, rW = oracle_scan(inp, eps=w.eps, mode=mode, b=w.b)
    assert_fp32_close(o, ro, "o")
    assert_fp32_close(W_T, rW, "W_T")


@pytest.mark.parametrize("case", [
    # (B, H, T, d, b, in_bf16)
    (2, 3, 77, 64, 16, False),
    (2, 3, 53, 16, 16, False),
    (2, 2, 70, 64, 24, True),     # internal chunk 12, bf16 inputs
], ids=["d64", "d16", "d64_b24_bf16"])
@pytest.mark.parametrize("norm_match", [False, True], ids=["ablate", "ablate_nm"])
@pytest.mark.parametrize("with_mask", [False, True], ids=["nomask", "mask"])
def test_ablation_grad_norms(case, norm_match, with_mask):
    """Per-token (||G_full||, ||G_ablation||) against the oracle (fp32 bound),
    exact zeros on SKIP chunks, and the scan's outputs unchanged by asking."""
    B, H, T, d, b, in_bf16 = case
    inp = make_inputs(B, H, T, d, seed=650 + T + d + b, random_affine=True, in_bf16=in_bf16,
                      mask_p=0.5 if with_mask else None, b=b)
    mode = ABLATE | (NORM_MATCH if norm_match else 0)
    o, W_T, gn = gpu_scan(inp, in_bf16=in_bf16, eps=1e-6, b=b, ablate=True, norm_match=norm_match,
                          want_grad_norms=True)
    ro, rW, rgn = oracle_scan(inp, eps=1e-6, mode=mode, b=b, want_grad_norms=True)
    assert_fp32_close(o, ro, "o")
    assert_fp32_close(W_T, rW, "W_T")
    assert_fp32_close(gn, rgn, "grad_norms")
    if with_mask:
        skip = np.repeat(inp["mask"] == 0, b, axis=1)[:, :T]          # [B, T]
        assert skip.any()
        assert np.all(gn[skip[:, None, :, None].repeat(H, 1).repeat(2, 3)] == 0.0)


def test_ablation_grad_norm_ratio_headline_shape():
    """The mean gradient norm ratio over the headline workload's tokens, GPU
    against the oracle."""
    w = WORKLOADS["2j"]
    inp = make_workload(w)
    o, W_T, gn = gpu_scan(inp, in_bf16=False, eps=w.eps, b=w.b, ablate=True, want_grad_norms=True)
    ro, rW, rgn = oracle_scan(inp, eps=w.eps, mode=ABLATE, b=w.b, want_grad_norms=True)
    assert_fp32_close(gn, rgn, "grad_norms")
    ratio, rratio = (gn[..., 1] / gn[..., 0]).mean(), (rgn[..., 1] / rgn[..., 0]).mean()
    assert abs(ratio - rratio) <= 2e-4 * rratio, (ratio, rratio)


def test_ablation_rejected_where_not_defined():
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    inp = make_inputs(1, 2, 32, 64, seed=14, random_affine=True)
    from tests.helpers import to_torch
    t = to_torch(inp, "cuda", False)
    args = (t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"], t["gamma"], t["beta"])
    with pytest.raises(ttt_scan.TTTScanError, match="INVALID"):
        ttt_scan.scan(*args, ablate=True, no_ln=True)
    with pytest.raises(ttt_scan.TTTScanError, match="INVALID"):
        ttt_scan.scan(*args, norm_match=True)
    with pytest.raises(ttt_scan.TTTScanError, match="INVALID"):
        ttt_scan.scan(*args, lnjac=True, want_grad_norms=True)


# ---------------------------------------------------------------------------
# Per-feature output gate [B, H, T, d] (the elementwise reading of the sigmoid
# output gate), in every scan kernel that takes it.
# ---------------------------------------------------------------------------

GATE_CHANNEL = 1 << 6


@pytest.mark.parametrize("case", [
    # (B, H, T, d, mode, b, in_bf16, single_cta)
    (2, 3, 77, 64, LNJAC, 16, False, False),     # per-token, 4-CTA clusters
    (2, 3, 77, 64, LNJAC, 16, False, True),      # per-token, one CTA per head
    (2, 3, 53, 16, 0, 16, False, False),          # d = 16
    (2, 3, 53, 64, MINIB | LNJAC, 16, False, False),
    (2, 3, 77, 64, MINIB | LNJAC, 16, True, False),   # bf16 mini-batch: tensor-core kernel
], ids=["cluster", "single_cta", "d16", "minibatch_f32", "minibatch_bf16"])
@pytest.mark.parametrize("with_mask", [False, True])
def test_per_feature_gate(case, with_mask):
    from test_sequence_layers_02_b200 import ttt_scan
    B, H, T, d, mode, b, in_bf16, single_cta = case
    tc = bool(mode & MINIB) and in_bf16
    want = (ttt_scan.KERNEL_TENSOR_CORE if tc else
            ttt_scan.KERNEL_CUDA_CORE if (single_cta or d != 64 or mode & MINIB)
            else ttt_scan.KERNEL_CUDA_CORE_CLUSTER)
    got = ttt_scan.kernel_choice(B, H, T, d, minibatch=bool(mode & MINIB), lnjac=bool(mode & LNJAC),
                                 in_bf16=in_bf16, b=b, single_cta=single_cta, gate_channel=True)
    assert got == want or (want == ttt_scan.KERNEL_CUDA_CORE_CLUSTER and
                           got == ttt_scan.KERNEL_CUDA_CORE)
    inp = make_inputs(B, H, T, d, seed=700 + T + d + mode, random_affine=True, in_bf16=in_bf16,
                      gate_channel=True, mask_p=0.5 if with_mask else None, b=b)
    o, W_T = gpu_scan(inp, in_bf16=in_bf16, eps=1e-6, b=b, lnjac=bool(mode & LNJAC),
                      minibatch=bool(mode & MINIB), single_cta=single_cta)
    ro, rW = oracle_scan(inp, eps=1e-6, mode=mode | GATE_CHANNEL, b=b)
    check = assert_rrms if tc else assert_fp32_close   # bf16 operands on the tensor cores
    check(o, ro, "o")
    check(W_T, rW, "W_T")


# ---------------------------------------------------------------------------
# Ablation gradient in mini-batch mode ("Error Correction in Trained TTT
# Layers", Abstract: the intervention was run on mini-batch TTT-Linear models):
# every gradient of a chunk at W_s, on the CUDA-core and tensor-core kernels.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("variant", ["ablate", "ablate_nm", "norms"])
@pytest.mark.parametrize("case", [
    # (B, H, T, d, b, in_bf16, force_simt)
    (2, 3, 53, 64, 16, False, True),     # CUDA cores, fp32
    (2, 3, 53, 16, 7, False, True),      # d = 16, b = 7
    (2, 3, 77, 64, 16, True, False),     # tensor cores
], ids=["simt_d64", "simt_d16", "tc"])
@pytest.mark.parametrize("with_mask", [False, True], ids=["nomask", "mask"])
def test_ablation_minibatch(case, variant, with_mask):
    from test_sequence_layers_02_b200 import ttt_scan
    B, H, T, d, b, in_bf16, simt = case
    nm, norms = variant == "ablate_nm", variant == "norms"
    want = ttt_scan.KERNEL_CUDA_CORE if simt else ttt_scan.KERNEL_TENSOR_CORE
    assert ttt_scan.kernel_choice(B, H, T, d, minibatch=True, ablate=True, norm_match=nm,
                                  in_bf16=in_bf16, out_bf16=in_bf16, b=b, force_simt=simt) == want
    inp = make_inputs(B, H, T, d, seed=800 + T + d + b, random_affine=True, in_bf16=in_bf16,
                      mask_p=0.5 if with_mask else None, b=b)
    mode = MINIB | ABLATE | (NORM_MATCH if nm else 0)
    res = gpu_scan(inp, in_bf16=in_bf16, out_bf16=in_bf16, eps=1e-6, b=b, minibatch=True,
                   ablate=True, norm_match=nm, force_simt=simt, want_grad_norms=norms)
    ref = oracle_scan(inp, eps=1e-6, mode=mode, b=b, want_grad_norms=norms)
    names = ["o", "W_T"] + (["grad_norms"] if norms else [])
    for got, r, nm_ in zip(res, ref, names):
        if simt:
            assert_fp32_close(got, r, nm_)
        else:
            assert_rrms(got, r, nm_)
    if norms and with_mask:
        skip = np.repeat(inp["mask"] == 0, b, axis=1)[:, :T]
        assert np.all(res[2][skip[:, None, :, None].repeat(H, 1).repeat(2, 3)] == 0.0)


# ---------------------------------------------------------------------------
# The `:mlp` variant ("Edifice.Recurrent.TTT", `build` options, `:variant`):
# SiLU on keys and queries as they are loaded, in every kernel.
# ---------------------------------------------------------------------------

KQ_SILU = 1 << 10


@pytest.mark.parametrize("case", [
    # (B, H, T, d, mode, b, in_bf16, single_cta, force_simt)
    (2, 3, 77, 64, LNJAC, 16, False, False, False),          # per-token, 4-CTA clusters
    (2, 3, 77, 64, LNJAC, 16, False, True, False),           # per-token, one CTA per head
    (2, 3, 53, 16, 0, 16, False, False, False),              # d = 16
    (2, 2, 53, 64, NO_LN, 16, False, True, False),
    (2, 3, 53, 64, MINIB | LNJAC, 16, False, False, True),   # mini-batch, CUDA cores
    (2, 3, 77, 64, MINIB | LNJAC, 16, True, False, False),   # mini-batch, tensor cores
    (2, 3, 77, 64, MINIB, 16, True, False, False),
], ids=["cluster", "single_cta", "d16", "no_ln", "minibatch_simt", "tc_lnjac", "tc_simple"])
@pytest.mark.parametrize("with_mask", [False, True])
def test_kq_silu_variant(case, with_mask):
    from test_sequence_layers_02_b200 import ttt_scan
    B, H, T, d, mode, b, in_bf16, single_cta, simt = case
    tc = bool(mode & MINIB) and in_bf16 and not simt
    if not tc and not (mode & MINIB) and d == 64:
        want = ttt_scan.KERNEL_CUDA_CORE if single_cta else ttt_scan.KERNEL_CUDA_CORE_CLUSTER
    else:
        want = ttt_scan.KERNEL_TENSOR_CORE if tc else ttt_scan.KERNEL_CUDA_CORE
    assert ttt_scan.kernel_choice(B, H, T, d, minibatch=bool(mode & MINIB), lnjac=bool(mode & LNJAC),
                                  no_ln=bool(mode & NO_LN), in_bf16=in_bf16, out_bf16=in_bf16, b=b,
                                  single_cta=single_cta, force_simt=simt, kq_silu=True) == want
    inp = make_inputs(B, H, T, d, seed=900 + T + d + mode, random_affine=True, in_bf16=in_bf16,
                      mask_p=0.5 if with_mask else None, b=b)
    o, W_T = gpu_scan(inp, in_bf16=in_bf16, out_bf16=in_bf16, eps=1e-6, b=b,
                      lnjac=bool(mode & LNJAC), no_ln=bool(mode & NO_LN),
                      minibatch=bool(mode & MINIB), single_cta=single_cta, force_simt=simt,
                      kq_silu=True)
    ro, rW = oracle_scan(inp, eps=1e-6, mode=mode | KQ_SILU, b=b)
    if tc:
        assert_rrms(o, ro, "o")
        assert_rrms(W_T, rW, "W_T")
        # and the variant is not the plain scan
        po, _ = oracle_scan(inp, eps=1e-6, mode=mode, b=b)
        assert rel_rms(o, po) > 0.1
    else:
        assert_fp32_close(o, ro, "o")
        assert_fp32_close(W_T, rW, "W_T")


def test_kq_silu_rejected_on_bf16_cuda_core_tiles():
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    from tests.helpers import to_torch
    inp = make_inputs(1, 2, 32, 64, seed=15, random_affine=True, in_bf16=True)
    t = to_torch(inp, "cuda", True)
    args = (t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"], t["gamma"], t["beta"])
    with pytest.raises(ttt_scan.TTTScanError, match="UNSUPPORTED"):
        ttt_scan.scan(*args, kq_silu=True, lnjac=True)
    with pytest.raises(ttt_scan.TTTScanError, match="UNSUPPORTED"):
        ttt_scan.scan(*args, kq_silu=True, minibatch=True, force_simt=True)
    torch.cuda.synchronize()
