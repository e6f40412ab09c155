"""GPU parity of the tcgen05 mini-batch kernel (d = 64, b = 16, bf16 inputs)
against the CPU oracle, plus its bounded-wait failure path."""

import numpy as np
import pytest

from test_sequence_layers_02_b200.workloads import make_inputs
from tests.helpers import assert_fp32_close, assert_rrms, gpu_scan, oracle_scan, rel_rms

pytestmark = pytest.mark.gpu

LNJAC, MINIB, NO_LN = 2, 1, 4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from test_sequence_layers_02_b200 import build, ttt_scan
    build.build()
    ttt_scan.lib()


@pytest.mark.parametrize("grad", [LNJAC, 0, NO_LN], ids=["lnjac", "simple", "no_ln"])
@pytest.mark.parametrize("out_bf16", [True, False], ids=["o16", "o32"])
@pytest.mark.parametrize("T", [16, 77, 160])
def test_tc_matches_oracle(grad, out_bf16, T):
    B, H = 2, 3
    inp = make_inputs(B, H, T, 64, seed=200 + T + grad, random_affine=True, in_bf16=True)
    o, W_T = gpu_scan(inp, in_bf16=True, out_bf16=out_bf16, eps=1e-6, b=16, minibatch=True,
                      lnjac=bool(grad & LNJAC), no_ln=bool(grad & NO_LN))
    ro, rW = oracle_scan(inp, eps=1e-6, mode=MINIB | grad, b=16)
    assert_rrms(o, ro, "o")
    assert_rrms(W_T, rW, "W_T")


@pytest.mark.parametrize("grad", [LNJAC, 0, NO_LN], ids=["lnjac", "simple", "no_ln"])
@pytest.mark.parametrize("BH", [(4, 37), (10, 15), (10, 30), (10, 45)],
                         ids=["148heads", "150heads", "300heads", "450heads"])
def test_tc_all_occupancy_builds(grad, BH):
    """On B200's 148 SMs: up to 148 heads run the one-CTA-per-SM build, 150
    the two-per-SM build, 300 the three-per-SM kernel (one wave instead of
    two), 450 the two-per-SM build again (two waves either way); each against
    the oracle, with a ragged tail and a SKIP/UPDATE mask."""
    B, H = BH
    inp = make_inputs(B, H, 40, 64, seed=250 + grad + B, random_affine=True, in_bf16=True,
                      mask_p=0.7, b=16)
    o, W_T = gpu_scan(inp, in_bf16=True, out_bf16=True, eps=1e-6, b=16, minibatch=True,
                      lnjac=bool(grad & LNJAC), no_ln=bool(grad & NO_LN))
    ro, rW = oracle_scan(inp, eps=1e-6, mode=MINIB | grad, b=16)
    assert_rrms(o, ro, "o")
    assert_rrms(W_T, rW, "W_T")


@pytest.mark.parametrize("BH,T", [((2, 3), 161), ((2, 3), 176), ((2, 3), 177), ((2, 3), 330),
                                  ((10, 15), 97), ((10, 15), 112), ((10, 15), 113),
                                  ((10, 15), 330), ((10, 30), 80), ((10, 30), 81),
                                  ((10, 30), 97), ((10, 30), 330)],
                         ids=["1perSM-11chunks", "1perSM-11full", "1perSM-12chunks",
                              "1perSM-21chunks", "2perSM-7chunks", "2perSM-7full",
                              "2perSM-8chunks", "2perSM-21chunks", "3perSM-5chunks",
                              "3perSM-6chunks", "3perSM-7chunks", "3perSM-21chunks"])
def test_tc_stage_ring_boundaries(BH, T):
    """The TMA stage ring refills stage x % NST with chunk x once chunk x - NST
    has finished: ten stages with one CTA per SM (6 heads), six with two (150
    heads on 148 SMs), five in the three-per-SM kernel (300 heads). Lengths at
    and just past the ring (the first refills, a full last chunk or a
    one-token one) and several times around it, with a SKIP/UPDATE mask,
    against the oracle."""
    B, H = BH
    inp = make_inputs(B, H, T, 64, seed=270 + T + B, random_affine=True, in_bf16=True,
                      mask_p=0.6, b=16)
    o, W_T = gpu_scan(inp, in_bf16=True, out_bf16=True, eps=1e-6, b=16, minibatch=True,
                      lnjac=True)
    ro, rW = oracle_scan(inp, eps=1e-6, mode=MINIB | LNJAC, b=16)
    assert_rrms(o, ro, "o")
    assert_rrms(W_T, rW, "W_T")


@pytest.mark.parametrize("T", [64, 77])
def test_tc_mask_is_bit_exact_on_skipped_chunks(T):
    B, H, b = 2, 3, 16
    inp = make_inputs(B, H, T, 64, seed=300 + T, random_affine=True, in_bf16=True, mask_p=0.5, b=b)
    o, W_T, Wc = gpu_scan(inp, in_bf16=True, out_bf16=True, eps=1e-6, b=b, minibatch=True,
                          lnjac=True, want_chunks=True)
    ro, rW, rWc = oracle_scan(inp, eps=1e-6, mode=MINIB | LNJAC, b=b, want_chunks=True)
    assert_rrms(o, ro, "o")
    assert_rrms(W_T, rW, "W_T")
    m = inp["mask"]
    for bi in range(B):
        for c in range(m.shape[1]):
            same = np.array_equal(Wc[bi, :, c + 1], Wc[bi, :, c])
            assert same == (m[bi, c] == 0), (bi, c)
    np.testing.assert_array_equal(Wc[:, :, 0], inp["W0"])
    np.testing.assert_array_equal(Wc[:, :, -1], W_T)


def test_tc_agrees_with_cuda_core_kernel():
    inp = make_inputs(2, 4, 200, 64, seed=400, random_affine=True, in_bf16=True)
    kw = dict(in_bf16=True, out_bf16=False, eps=1e-6, b=16, minibatch=True, lnjac=True)
    o_tc, W_tc = gpu_scan(inp, **kw)
    o_s, W_s = gpu_scan(inp, force_simt=True, **kw)
    assert rel_rms(o_tc, o_s) <= 2e-2
    assert rel_rms(W_tc, W_s) <= 2e-2


def test_tc_eta_zero_and_no_gate():
    inp = make_inputs(1, 2, 50, 64, seed=401, random_affine=True, in_bf16=True)
    inp["eta_logit_bf16"] = np.full_like(inp["eta_logit_bf16"], 0xC61C)   # bf16(-9984)
    inp["eta_logit"] = np.full_like(inp["eta_logit"], -9984.0)
    inp["gate_logit"] = None
    inp["gate_logit_bf16"] = None
    o, W_T = gpu_scan(inp, in_bf16=True, out_bf16=False, eps=1e-6, b=16, minibatch=True, lnjac=True)
    assert np.array_equal(W_T, inp["W0"].astype(np.float64))
    ref = np.einsum("bhrc,bhtc->bhtr", inp["W0"].astype(np.float64), inp["q"].astype(np.float64))
    assert_rrms(o, ref, "o", tol=5e-3)


@pytest.mark.parametrize("BH", [(1, 2), (10, 30)], ids=["2heads", "300heads"])
def test_tc_wait_timeout_reports_and_recovers(BH):
    """With a wait limit of 0 every bounded wait gives up at once: the kernel
    (either tensor-core kernel: 300 heads take the three-per-SM one) must
    report TTT_ERR_DEVICE_TIMEOUT (no hang, no trap), and the context must
    stay usable for a normal call afterwards."""
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    from tests.helpers import to_torch
    inp = make_inputs(*BH, 48, 64, seed=402, random_affine=True, in_bf16=True)
    t = to_torch(inp, "cuda", True)
    args = (t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"], t["W0"], t["gamma"], t["beta"])
    ttt_scan.set_wait_limit(0)
    try:
        ttt_scan.scan(*args, eps=1e-6, b=16, minibatch=True, lnjac=True)
        assert ttt_scan.check_device_status() == ttt_scan.TTT_ERR_DEVICE_TIMEOUT
    finally:
        ttt_scan.set_wait_limit(1 << 20)
    assert ttt_scan.check_device_status() == ttt_scan.TTT_OK   # cleared by the read
    o, W_T = ttt_scan.scan(*args, eps=1e-6, b=16, minibatch=True, lnjac=True)
    torch.cuda.synchronize()
    assert ttt_scan.check_device_status() == ttt_scan.TTT_OK
    ro, rW = oracle_scan(inp, eps=1e-6, mode=MINIB | LNJAC, b=16)
    assert_rrms(o.float().cpu().numpy(), ro, "o")


@pytest.mark.parametrize("BH,T,out_bf16", [((2, 3), 77, True), ((2, 3), 160, False),
                                            ((10, 30), 40, True)],
                         ids=["6heads_ragged", "6heads_o32", "300heads"])
def test_tc_per_feature_gate(BH, T, out_bf16):
    """A per-feature gate [B, H, T, d] on the tensor-core kernel (its bulk warps
    stage each chunk's gate logits in shared memory), with a mask and a ragged
    tail; 300 heads keep to the two-per-SM build (the three-per-SM kernel has
    no per-feature gate)."""
    from test_sequence_layers_02_b200 import ttt_scan
    B, H = BH
    inp = make_inputs(B, H, T, 64, seed=600 + T + B, random_affine=True, in_bf16=True,
                      gate_channel=True, mask_p=0.6, b=16)
    assert ttt_scan.kernel_choice(B, H, T, 64, minibatch=True, lnjac=True, in_bf16=True,
                                  out_bf16=out_bf16, b=16, gate_channel=True) == \
        ttt_scan.KERNEL_TENSOR_CORE
    o, W_T = gpu_scan(inp, in_bf16=True, out_bf16=out_bf16, eps=1e-6, b=16, minibatch=True,
                      lnjac=True)
    ro, rW = oracle_scan(inp, eps=1e-6, mode=MINIB | LNJAC | (1 << 6), b=16)
    assert_rrms(o, ro, "o")
    assert_rrms(W_T, rW, "W_T")
