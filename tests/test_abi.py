"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments before touching the GPU (these run without a GPU)."""

import ctypes
import re
from pathlib import Path

import pytest

from test_sequence_layers_02_b200 import build as pkg_build

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def lib():
    pkg_build.build()
    from test_sequence_layers_02_b200 import ttt_scan
    return ttt_scan.lib()


def declared_functions():
    names = []
    for h in sorted((ROOT / "include").glob("*.h")):
        text = re.sub(r"/\*.*?\*/", "", h.read_text(), flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(ttt_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_headers_declare_the_boundary():
    names = declared_functions()
    for must in ("ttt_scan_forward", "ttt_scan_forward_grad_norms", "ttt_decode_step",
                 "ttt_scan_kernel_choice",
                 "ttt_check_device_status",
                 "ttt_status_string", "ttt_set_wait_limit", "ttt_probe_ffma"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_status_strings(lib):
    from test_sequence_layers_02_b200 import ttt_scan as ts
    assert ts.status_string(0) == "TTT_OK"
    assert ts.status_string(-1) == "TTT_ERR_INVALID_ARG"
    assert ts.status_string(-2) == "TTT_ERR_UNSUPPORTED"
    assert ts.status_string(-3) == "TTT_ERR_CUDA"
    assert ts.status_string(-4) == "TTT_ERR_DEVICE_TIMEOUT"
    assert ts.status_string(12345) == "TTT_UNKNOWN_STATUS"


# Fake, 16-byte-aligned, non-overlapping "device" addresses: argument checks
# reject the calls below before any CUDA call, so nothing is dereferenced.
BASE = 1 << 40
STRIDE = 1 << 32


def addr(i, off=0):
    return ctypes.c_void_p(BASE + i * STRIDE + off)


def call(lib, **over):
    a = dict(q=addr(0), k=addr(1), v=addr(2), eta=addr(3), gate=addr(4), W0=addr(5),
             gamma=addr(6), beta=addr(7), B=2, H=3, T=40, d=64, eps=1e-6, mode=0, b=16,
             mask=None, o=addr(8), W_T=addr(9), W_chunks=None)
    a.update(over)
    return lib.ttt_scan_forward(a["q"], a["k"], a["v"], a["eta"], a["gate"], a["W0"], a["gamma"],
                                a["beta"], a["B"], a["H"], a["T"], a["d"], a["eps"], a["mode"],
                                a["b"], a["mask"], a["o"], a["W_T"], a["W_chunks"], None)


INVALID, UNSUPPORTED = -1, -2


@pytest.mark.parametrize("over", [
    dict(q=None), dict(k=None), dict(v=None), dict(eta=None), dict(W0=None), dict(o=None),
    dict(W_T=None), dict(gamma=None), dict(beta=None),
    dict(q=addr(0, 4)), dict(o=addr(8, 8)), dict(mask=addr(10, 1)), dict(W_chunks=addr(11, 2)),
    dict(B=-1), dict(H=-1), dict(T=-1), dict(b=0), dict(b=-3), dict(d=0), dict(d=-64),
    dict(eps=-1e-6), dict(eps=float("nan")), dict(eps=float("inf")),
    dict(mode=1 << 11), dict(mode=1 << 31),
    dict(mode=(1 << 8) | 4),              # ablation without a LayerNorm
    dict(mode=1 << 9),                    # norm matching without the ablation
    dict(o=addr(0)),                      # output over an input
    dict(o=addr(2, 1 << 12)),             # output inside v
    dict(W_T=addr(5, 256)),               # W_T partially overlapping W0
    dict(W_T=addr(8)),                    # W_T over o
    dict(W_chunks=addr(9)),               # W_chunks over W_T
], ids=lambda o: ",".join(f"{k}" for k in o))
def test_invalid_arguments_rejected(lib, over):
    assert call(lib, **over) == INVALID


@pytest.mark.parametrize("over", [dict(d=32), dict(d=128), dict(d=17),
                                  dict(mode=1, b=17), dict(mode=1 | 32, b=32),
                                  dict(mode=(1 << 10) | 8),            # SiLU, bf16, per-token
                                  dict(mode=(1 << 10) | 8 | 1 | 32)])  # SiLU, bf16, CUDA-core mini-batch
def test_unsupported_shapes(lib, over):
    assert call(lib, **over) == UNSUPPORTED


def call_gn(lib, **over):
    """ttt_scan_forward_grad_norms with the same fake arguments as call()."""
    a = dict(q=addr(0), k=addr(1), v=addr(2), eta=addr(3), gate=addr(4), W0=addr(5),
             gamma=addr(6), beta=addr(7), B=2, H=3, T=40, d=64, eps=1e-6, mode=(1 << 8) | 2,
             b=16, mask=None, o=addr(8), W_T=addr(9), W_chunks=None, gn=addr(12))
    a.update(over)
    fn = lib.ttt_scan_forward_grad_norms
    fn.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int] * 4 + [ctypes.c_float, ctypes.c_uint,
                                                                 ctypes.c_int] + [ctypes.c_void_p] * 6
    return fn(a["q"], a["k"], a["v"], a["eta"], a["gate"], a["W0"], a["gamma"], a["beta"],
              a["B"], a["H"], a["T"], a["d"], a["eps"], a["mode"], a["b"], a["mask"], a["o"],
              a["W_T"], a["W_chunks"], a["gn"], None)


@pytest.mark.parametrize("over,want", [
    (dict(mode=2), INVALID),                       # norms need the ablation gradient
    (dict(mode=0), INVALID),
    (dict(gn=None), INVALID),                      # no output for a non-empty problem
    (dict(gn=addr(12, 4)), INVALID),               # misaligned
    (dict(gn=addr(8)), INVALID),                   # over o
    (dict(gn=addr(9)), INVALID),                   # over W_T
    (dict(gn=addr(2, 1 << 10)), INVALID),          # inside v
    (dict(mode=(1 << 8) | 8 | (1 << 10)), UNSUPPORTED),   # SiLU on bf16 CUDA-core tiles
    (dict(d=32), UNSUPPORTED),
    (dict(B=0), 0), (dict(B=0, gn=None), 0), (dict(T=0, B=0), 0),   # empty: nothing launched
], ids=lambda x: ",".join(x) if isinstance(x, dict) else str(x))
def test_grad_norms_entry_checks(lib, over, want):
    assert call_gn(lib, **over) == want


def test_no_ln_needs_no_affine_and_empty_batch_is_noop(lib):
    # no heads: valid, nothing launched
    assert call(lib, B=0) == 0
    assert call(lib, H=0) == 0
    assert call(lib, B=0, gamma=None, beta=None, mode=4) == 0


def test_in_place_W_T_is_accepted_by_the_checks(lib):
    assert call(lib, B=0, W_T=addr(5)) == 0


def dcall(lib, **over):
    a = dict(q=addr(0), k=addr(1), v=addr(2), eta=addr(3), gate=addr(4), W=addr(5),
             gamma=addr(6), beta=addr(7), B=2, H=3, d=64, eps=1e-6, mode=0, update=None,
             o=addr(8))
    a.update(over)
    return lib.ttt_decode_step(a["q"], a["k"], a["v"], a["eta"], a["gate"], a["W"], a["gamma"],
                               a["beta"], a["B"], a["H"], a["d"], a["eps"], a["mode"],
                               a["update"], a["o"], None)


@pytest.mark.parametrize("over", [
    dict(q=None), dict(k=None), dict(v=None), dict(eta=None), dict(W=None), dict(o=None),
    dict(gamma=None), dict(beta=None),
    dict(q=addr(0, 4)), dict(W=addr(5, 8)), dict(update=addr(10, 1)), dict(o=addr(8, 2)),
    dict(B=-1), dict(H=-1), dict(d=0), dict(eps=-1.0), dict(eps=float("nan")),
    dict(mode=1 << 11), dict(mode=(1 << 8) | 4), dict(mode=1 << 9),
    dict(o=addr(1)),                      # output over an input
    dict(W=addr(8)),                      # state over the output
    dict(W=addr(2, 64)),                  # state inside v
    dict(gate=addr(8, 64), mode=64),      # per-feature gate inside the output
], ids=lambda o: ",".join(f"{k}" for k in o))
def test_decode_invalid_arguments_rejected(lib, over):
    assert dcall(lib, **over) == INVALID


@pytest.mark.parametrize("over", [dict(d=32), dict(d=17), dict(mode=1), dict(mode=1 | 2)])
def test_decode_unsupported(lib, over):
    assert dcall(lib, **over) == UNSUPPORTED


def test_decode_empty_and_no_ln(lib):
    assert dcall(lib, B=0) == 0
    assert dcall(lib, H=0, gamma=None, beta=None, mode=4) == 0
    assert dcall(lib, B=0, q=None, k=None, v=None, eta=None, W=None, o=None) == 0


def test_kernel_choice_without_launching(lib):
    f = lib.ttt_scan_kernel_choice
    MINIB, LNJAC, BF16 = 1, 2, 8
    assert f(2, 3, 40, 64, MINIB | LNJAC | BF16, 16) == 3            # tensor cores
    assert f(2, 3, 40, 64, MINIB | LNJAC | BF16 | 32, 16) == 1       # forced CUDA cores
    assert f(2, 3, 40, 16, 0, 16) == 1                               # d = 16: one CTA per head
    assert f(2, 3, 40, 64, 1 << 7, 16) == 1                          # single CTA asked for
    assert f(0, 3, 40, 64, 0, 16) == 0                               # nothing to launch
    assert f(2, 3, 40, 64, 1 << 11, 16) == INVALID
    assert f(2, 3, 40, 64, 1 << 9, 16) == INVALID                     # norm match alone
    assert f(2, 3, 40, 64, (1 << 8) | 4, 16) == INVALID               # ablation without LN
    assert f(2, 3, 40, 64, 1 | (1 << 8), 16) == 1                     # mini-batch ablation, fp32
    assert f(2, 3, 40, 64, MINIB | BF16 | (1 << 8), 16) == 3          # ... bf16: tensor cores
    assert f(2, 3, 40, 64, MINIB | BF16 | (1 << 8) | (1 << 9), 16) == 3
    assert f(2, 3, 40, 64, 1 << 8, 16) in (1, 2)                      # per-token ablation
    assert f(2, 3, 40, 64, (1 << 10) | BF16, 16) == UNSUPPORTED       # SiLU on bf16 CUDA-core tiles
    assert f(2, 3, 40, 64, (1 << 10) | BF16 | MINIB, 16) == 3         # ... on the tensor cores
    assert f(2, 3, 40, 64, 1 << 10, 16) in (1, 2)                     # SiLU, fp32, per-token
    assert f(2, 3, 40, 16, (1 << 10) | MINIB, 16) == 1
    assert f(2, 3, 40, 64, 0, 0) == INVALID
    assert f(2, 3, 40, 32, 0, 16) == UNSUPPORTED
    assert f(2, 3, 40, 64, MINIB, 17) == UNSUPPORTED
    assert f(2, 3, 40, 64, MINIB | LNJAC | BF16 | (1 << 6), 16) == 3 # per-feature gate: tensor cores
    # per-token d = 64 picks the cluster kernel only where clusters fit on a device
    assert f(2, 3, 40, 64, LNJAC, 16) in (1, 2)


def test_wait_limit(lib):
    assert lib.ttt_set_wait_limit(-1) == INVALID
    assert lib.ttt_set_wait_limit(1 << 20) == 0


def test_probe_rejects_bad_arguments(lib):
    flops = ctypes.c_double()
    assert lib.ttt_probe_ffma(0, 256, 10, addr(0), ctypes.byref(flops), None) == -1
    assert lib.ttt_probe_ffma(4, 100, 10, addr(0), ctypes.byref(flops), None) == -1
    assert lib.ttt_probe_ffma(4, 256, 10, None, ctypes.byref(flops), None) == -1


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    from test_sequence_layers_02_b200 import ttt_scan as ts
    monkeypatch.setattr(ts, "_lib", None)
    monkeypatch.setattr(ts, "_LIB_PATH", tmp_path / "missing.so")
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        ts.lib()


def bcall(lib, **over):
    """ttt_scan_backward with fake, non-overlapping device addresses."""
    a = dict(q=addr(0), k=addr(1), v=addr(2), eta=addr(3), gate=addr(4), gamma=addr(6),
             beta=addr(7), B=2, H=3, T=40, d=64, eps=1e-6, mode=2, b=16, mask=None,
             Wc=addr(13), dO=addr(14), dWT=None, dq=addr(15), dk=addr(16), dv=addr(17),
             deta=addr(18), dgate=addr(19), dW0=addr(20), dgamma=addr(21), dbeta=addr(22),
             ws=addr(23), ws_bytes=1 << 20)
    a.update(over)
    return lib.ttt_scan_backward(a["q"], a["k"], a["v"], a["eta"], a["gate"], a["gamma"],
                                 a["beta"], a["B"], a["H"], a["T"], a["d"], a["eps"], a["mode"],
                                 a["b"], a["mask"], a["Wc"], a["dO"], a["dWT"], a["dq"], a["dk"],
                                 a["dv"], a["deta"], a["dgate"], a["dW0"], a["dgamma"],
                                 a["dbeta"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("over", [
    dict(q=None), dict(dO=None), dict(Wc=None), dict(dq=None), dict(dW0=None),
    dict(dgate=None),                     # a gate needs its gradient
    dict(dgamma=None), dict(ws=None),     # LayerNorm: gamma / beta gradients and workspace
    dict(ws_bytes=2 * 3 * 2 * 64 * 4 - 4),
    dict(dq=addr(15, 4)), dict(B=-1), dict(b=0), dict(eps=-1.0), dict(mode=1 << 11),
    dict(mode=(1 << 8) | 4), dict(mode=1 << 9),
    dict(dq=addr(0)),                     # output over an input
    dict(dk=addr(15)),                    # two outputs on one buffer
    dict(ws=addr(21)),                    # workspace over dgamma
], ids=lambda o: ",".join(f"{k}" for k in o))
def test_backward_invalid_arguments_rejected(lib, over):
    assert bcall(lib, **over) == INVALID


@pytest.mark.parametrize("over", [dict(d=32), dict(b=17), dict(mode=(1 << 8) | (1 << 9) | 2)])
def test_backward_unsupported(lib, over):
    assert bcall(lib, **over) == UNSUPPORTED


def test_backward_workspace_bytes_and_no_ln(lib):
    f = lib.ttt_scan_backward_workspace_bytes
    assert f(2, 3, 64, 2) == 2 * 3 * 2 * 64 * 4
    assert f(2, 3, 64, 4) == 0                       # no LayerNorm: no gamma / beta
    assert f(0, 3, 64, 2) == 0
    # no LayerNorm: gamma, beta, their gradients and the workspace may be absent
    assert bcall(lib, B=0, mode=4, gamma=None, beta=None, dgamma=None, dbeta=None, ws=None) == 0


# ---- ttt_scan_forward_host: the end-to-end entry point (host buffers) ----
def call_host(lib, **over):
    """ttt_scan_forward_host with fake host addresses; every call below is
    rejected (or is empty) before any copy is enqueued."""
    a = dict(q=addr(0), k=addr(1), v=addr(2), eta=addr(3), gate=addr(4), W0=addr(5),
             gamma=addr(6), beta=addr(7), B=2, H=3, T=40, d=64, eps=1e-6, mode=1 | 2 | 8 | 16,
             b=16, mask=None, o=addr(8), W_T=addr(9), seg=0, ws=addr(12), ws_bytes=None)
    a.update(over)
    if a["ws_bytes"] is None:
        a["ws_bytes"] = lib.ttt_scan_forward_host_workspace_bytes(
            a["B"], a["H"], a["T"], a["d"], a["mode"], a["b"], max(a["seg"], 0))
    return lib.ttt_scan_forward_host(a["q"], a["k"], a["v"], a["eta"], a["gate"], a["W0"],
                                     a["gamma"], a["beta"], a["B"], a["H"], a["T"], a["d"],
                                     a["eps"], a["mode"], a["b"], a["mask"], a["o"], a["W_T"],
                                     a["seg"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("over,want", [
    (dict(seg=5), INVALID),                    # not a multiple of b
    (dict(seg=-16), INVALID),
    (dict(B=-1), INVALID), (dict(T=-1), INVALID), (dict(b=0), INVALID),
    (dict(eps=float("nan")), INVALID), (dict(mode=1 << 11), INVALID),
    (dict(q=None), INVALID), (dict(W0=None), INVALID), (dict(o=None), INVALID),
    (dict(gamma=None), INVALID),
    (dict(ws=None), INVALID), (dict(ws=addr(12, 8)), INVALID),   # missing / misaligned workspace
    (dict(ws_bytes=1024), INVALID),            # workspace too small
    (dict(o=addr(0)), INVALID),                # output over an input
    (dict(W_T=addr(8)), INVALID),              # W_T over o
    (dict(W_T=addr(5, 256)), INVALID),         # W_T partially over W0
    (dict(d=32), UNSUPPORTED),
    (dict(B=0), 0),                            # no heads: nothing to do
], ids=lambda x: ",".join(x) if isinstance(x, dict) else str(x))
def test_host_entry_checks(lib, over, want):
    assert call_host(lib, **over) == want


def test_host_workspace_bytes(lib):
    f = lib.ttt_scan_forward_host_workspace_bytes
    MB = 1 | 2 | 8 | 16
    assert f(2, 32, 32768, 64, MB, 16, 5) == 0           # not a multiple of b
    assert f(2, 32, 32768, 64, MB, 16, -16) == 0
    assert f(-1, 32, 32768, 64, MB, 16, 0) == 0
    default = f(2, 32, 32768, 64, MB, 16, 0)
    assert default == f(2, 32, 32768, 64, MB, 16, 4096)  # the default: an eighth of T
    # two segments' worth of inputs and outputs, plus the state
    per_seg = 2 * 32 * 4096 * (3 * 64 * 2 + 2 * 2 + 64 * 2)
    assert 2 * per_seg < default < 2 * per_seg + 2 * 32 * 64 * 64 * 4 + (1 << 20)
    assert f(2, 32, 32768, 64, MB, 16, 1024) < default < f(2, 32, 32768, 64, MB, 16, 32768)
    # a segment never exceeds the sequence
    assert f(1, 1, 40, 64, MB, 16, 0) == f(1, 1, 40, 64, MB, 16, 1024)
