"""The no-allocation entry point of the backward pass, ttt_scan_backward_noalloc.

Some callers cannot call cudaMalloc: code running inside a framework whose
allocator owns the whole device memory pool, or a latency-critical loop where
cudaMalloc's implicit device synchronisation is not acceptable. For them the
backward pass has a variant whose scratch (the per-head gamma / beta partial
sums) lives in a fixed array in device memory that the library itself holds.
This test calls it through the C ABI and checks it against
ttt_scan_backward (the caller-workspace entry point) on two calls in a row:
the second call must not be disturbed by what the first left in the shared
array. It sits in a file of its own that pytest collects last.
"""

import ctypes

import numpy as np
import pytest

from test_sequence_layers_02_b200.workloads import make_inputs
from tests.helpers import assert_fp32_close, to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from test_sequence_layers_02_b200 import build, ttt_scan
    build.build()
    L = ttt_scan.lib()
    vp, i = ctypes.c_void_p, ctypes.c_int
    L.ttt_scan_backward_noalloc.argtypes = [vp] * 7 + [i] * 4 + [ctypes.c_float, ctypes.c_uint,
                                                                 i] + [vp] * 13
    L.ttt_scan_backward_noalloc.restype = i
    return L


def _problem(B, H, T, d, b, seed):
    """Inputs, the forward's snapshots and dO, dW_T on the device."""
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    inp = make_inputs(B, H, T, d, seed=seed, random_affine=True, mask_p=0.5, b=b)
    t = to_torch(inp, "cuda", False)
    _, _, t["W_chunks"] = ttt_scan.scan(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"],
                                        t["W0"], t["gamma"], t["beta"], eps=1e-6, lnjac=True,
                                        b=b, mask=t["mask"], want_chunks=True)
    rng = np.random.default_rng(seed + 1)
    t["dO"] = torch.from_numpy(rng.standard_normal((B, H, T, d), dtype=np.float32)).cuda()
    t["dW_T"] = torch.from_numpy(
        (0.1 * rng.standard_normal((B, H, d, d))).astype(np.float32)).cuda()
    return t


def _noalloc(lib, t, eps, b):
    import torch
    B, H, T, d = t["q"].shape
    f32 = dict(dtype=torch.float32, device="cuda")
    out = dict(dq=torch.empty((B, H, T, d), **f32), dk=torch.empty((B, H, T, d), **f32),
               dv=torch.empty((B, H, T, d), **f32), deta_logit=torch.empty((B, H, T), **f32),
               dgate_logit=torch.empty((B, H, T), **f32), dW0=torch.empty((B, H, d, d), **f32),
               dgamma=torch.empty((H, d), **f32), dbeta=torch.empty((H, d), **f32))
    p = lambda x: ctypes.c_void_p(x.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.ttt_scan_backward_noalloc(
        p(t["q"]), p(t["k"]), p(t["v"]), p(t["eta_logit"]), p(t["gate_logit"]), p(t["gamma"]),
        p(t["beta"]), B, H, T, d, eps, 2, b, p(t["mask"]), p(t["W_chunks"]), p(t["dO"]),
        p(t["dW_T"]), p(out["dq"]), p(out["dk"]), p(out["dv"]), p(out["deta_logit"]),
        p(out["dgate_logit"]), p(out["dW0"]), p(out["dgamma"]), p(out["dbeta"]), stream)
    assert rc == 0, rc
    return out


def test_noalloc_backward_matches_the_workspace_entry_point_twice(lib):
    import torch
    from test_sequence_layers_02_b200 import ttt_scan
    # two different problems in a row: the second must not see the first's
    # partial sums in the shared array
    for (B, H, T, d, b, seed) in ((3, 4, 45, 64, 16, 4100), (2, 5, 37, 16, 8, 4200)):
        t = _problem(B, H, T, d, b, seed)
        got = _noalloc(lib, t, 1e-6, b)
        ref = ttt_scan.scan_backward(t["q"], t["k"], t["v"], t["eta_logit"], t["gate_logit"],
                                     t["gamma"], t["beta"], t["W_chunks"], t["dO"], t["dW_T"],
                                     eps=1e-6, lnjac=True, b=b, mask=t["mask"])
        torch.cuda.synchronize()
        assert ttt_scan.check_device_status() == ttt_scan.TTT_OK
        for key, r in ref.items():
            assert_fp32_close(got[key].cpu().numpy(), r.cpu().numpy(), f"noalloc {key}")


def test_noalloc_backward_rejects_more_heads_than_its_scratch_holds(lib):
    # 2^20 floats of scratch hold 2 d floats per head: 8192 heads at d = 64
    z = ctypes.c_void_p(1 << 40)  # never dereferenced: the size check comes first
    rc = lib.ttt_scan_backward_noalloc(z, z, z, z, None, z, z, 8193, 1, 16, 64, 1e-6, 2, 16,
                                       None, z, z, None, z, z, z, z, None, z, z, z, None)
    assert rc == -2   # TTT_ERR_UNSUPPORTED
