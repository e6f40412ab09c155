"""The end-to-end entry point ttt_scan_forward_host (host buffers, the sequence
in segments whose copies overlap the scans) against the oracle, at the same
tolerances as the device path, and against the device path itself: equal bit
for bit when one segment covers the sequence; otherwise equal up to rounding,
because the state W passes between segments exactly but the kernels' look-ahead
products restart at a segment boundary (z of the first chunk comes straight
from the state, not from an older state plus corrections)."""

import numpy as np
import pytest
import torch

from test_sequence_layers_02_b200.workloads import make_inputs
from tests.helpers import assert_fp32_close, assert_rrms, oracle_scan, rel_rms, to_torch

pytestmark = pytest.mark.gpu

MINIB, LNJAC = 1, 2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from test_sequence_layers_02_b200 import build, ttt_scan
    build.build()
    ttt_scan.lib()


def _both(inp, in_bf16, seg_tokens, pinned=True, **kw):
    from test_sequence_layers_02_b200 import ttt_scan
    dev = to_torch(inp, "cuda", in_bf16)
    host = {k: (None if v is None else v.cpu()) for k, v in dev.items()}
    if pinned:
        host = {k: (None if v is None else v.pin_memory()) for k, v in host.items()}
    args = ("q", "k", "v", "eta_logit", "gate_logit", "W0", "gamma", "beta")
    o_d, w_d = ttt_scan.scan(*(dev[a] for a in args), mask=dev["mask"], **kw)
    torch.cuda.synchronize()
    assert ttt_scan.check_device_status() == ttt_scan.TTT_OK
    full = dict(minibatch=False, lnjac=False, no_ln=False, b=16, out_dtype=None, force_simt=False,
                single_cta=False, ablate=False, norm_match=False, kq_silu=False, o=None,
                W_T=None, stream=None, eps=1e-6)
    full.update(kw)
    o_h, w_h = ttt_scan._scan_host(*(host[a] for a in args), mask=host["mask"],
                                   seg_tokens=seg_tokens, **full)
    f = lambda t: t.float().cpu().numpy().astype(np.float64)
    return (f(o_d), f(w_d)), (f(o_h), f(w_h))


@pytest.mark.parametrize("seg", [0, 64, 256, 1024])
def test_minibatch_tensor_cores_with_mask(seg):
    # T = 1000: the last segment (and chunk) is ragged; 1024 covers it in one segment
    inp = make_inputs(2, 3, 1000, 64, seed=500, random_affine=True, in_bf16=True, mask_p=0.5, b=16)
    dev, host = _both(inp, True, seg, minibatch=True, lnjac=True, b=16,
                      out_dtype=torch.bfloat16, eps=1e-6)
    ro, rw = oracle_scan(inp, eps=1e-6, mode=MINIB | LNJAC, b=16)
    assert_rrms(host[0], ro, "o")
    assert_rrms(host[1], rw, "W_T")
    if seg == 1024:
        assert np.array_equal(host[0], dev[0]) and np.array_equal(host[1], dev[1])
    else:
        assert rel_rms(host[0], dev[0]) <= 1e-2 and rel_rms(host[1], dev[1]) <= 1e-2


@pytest.mark.parametrize("seg", [0, 48, 160])
def test_per_token_fp32(seg):
    inp = make_inputs(1, 4, 700, 64, seed=501, qk_l2norm=True)
    dev, host = _both(inp, False, seg, lnjac=True, b=16, eps=1e-6)
    ro, rw = oracle_scan(inp, eps=1e-6, mode=LNJAC, b=16)
    assert_fp32_close(host[0], ro, "o")
    assert_fp32_close(host[1], rw, "W_T")
    assert rel_rms(host[0], dev[0]) <= 1e-5 and rel_rms(host[1], dev[1]) <= 1e-5


def test_cuda_core_minibatch_channel_gate_small_b():
    inp = make_inputs(2, 2, 300, 64, seed=502, random_affine=True, gate_channel=True,
                      mask_p=0.6, b=8)
    dev, host = _both(inp, False, 32, minibatch=True, lnjac=True, b=8, eps=1e-6)
    ro, rw = oracle_scan(inp, eps=1e-6, mode=MINIB | LNJAC | (1 << 6), b=8)  # per-feature gate
    assert_fp32_close(host[0], ro, "o")
    assert_fp32_close(host[1], rw, "W_T")


def test_d16_one_segment_and_pageable_memory():
    inp = make_inputs(3, 2, 50, 16, seed=503)
    dev, host = _both(inp, False, 0, pinned=False, b=16, eps=1e-5)
    assert np.array_equal(host[0], dev[0]) and np.array_equal(host[1], dev[1])


def test_in_place_state_and_empty_sequence():
    from test_sequence_layers_02_b200 import ttt_scan
    inp = make_inputs(1, 2, 200, 64, seed=504, random_affine=True, in_bf16=True)
    dev = to_torch(inp, "cuda", True)
    args = ("q", "k", "v", "eta_logit", "gate_logit", "W0", "gamma", "beta")
    o_d, w_d = ttt_scan.scan(*(dev[a] for a in args), minibatch=True, lnjac=True, b=16)
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in dev.items()}
    W = host["W0"].clone()
    o_h, w_h = ttt_scan.scan(host["q"], host["k"], host["v"], host["eta_logit"],
                             host["gate_logit"], W, host["gamma"], host["beta"], minibatch=True,
                             lnjac=True, b=16, W_T=W)
    assert w_h.data_ptr() == W.data_ptr()
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(W, w_d.cpu())   # one segment: exact
    # T = 0: W_T = W0 and nothing else
    e = {k: (None if v is None else v[:, :, :0].contiguous()) for k, v in host.items()
         if k in ("q", "k", "v", "eta_logit", "gate_logit")}
    o0, w0 = ttt_scan.scan(e["q"], e["k"], e["v"], e["eta_logit"], e["gate_logit"],
                           host["W0"], host["gamma"], host["beta"], minibatch=True, lnjac=True,
                           b=16)
    assert o0.shape[2] == 0 and torch.equal(w0, host["W0"])
