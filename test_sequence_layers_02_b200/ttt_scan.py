"""Thin Python binding of ``libttt_scan.so`` (argument marshalling only).

Every step of the scan runs in the library's CUDA kernels; this module checks
shapes and dtypes, allocates outputs with torch, and passes raw device pointers
and the current CUDA stream to ``ttt_scan_forward``, ``ttt_scan_backward`` and
``ttt_decode_step`` (include/ttt_scan.h). There
is no CPU fallback: if the library cannot be loaded, the first call raises.
"""

from __future__ import annotations

import ctypes
from pathlib import Path
from typing import Optional

import torch

_LIB_PATH = Path(__file__).resolve().parent / "libttt_scan.so"

# Mode bits of include/ttt_scan.h.
MODE_MINIBATCH = 1 << 0
GRAD_LNJAC = 1 << 1
NO_LN = 1 << 2
IN_BF16 = 1 << 3
OUT_BF16 = 1 << 4
KERNEL_SIMT = 1 << 5
GATE_CHANNEL = 1 << 6
KERNEL_SINGLE_CTA = 1 << 7
GRAD_ABLATE = 1 << 8
GRAD_NORM_MATCH = 1 << 9
KQ_SILU = 1 << 10

# Kernel identifiers of ttt_scan_kernel_choice.
KERNEL_NONE, KERNEL_CUDA_CORE, KERNEL_CUDA_CORE_CLUSTER, KERNEL_TENSOR_CORE = 0, 1, 2, 3

TTT_OK = 0
TTT_ERR_INVALID_ARG = -1
TTT_ERR_UNSUPPORTED = -2
TTT_ERR_CUDA = -3
TTT_ERR_DEVICE_TIMEOUT = -4


class TTTScanError(RuntimeError):
    def __init__(self, status: int, what: str = "ttt_scan_forward"):
        self.status = status
        super().__init__(f"{what} failed: {status_string(status)} ({status})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not _LIB_PATH.exists():
            raise RuntimeError(
                f"{_LIB_PATH.name} is missing: build it with "
                "`python -m test_sequence_layers_02_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(str(_LIB_PATH))
        vp, i, u = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
        L.ttt_scan_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i,
                                       ctypes.c_float, u, i, vp, vp, vp, vp, vp]
        L.ttt_scan_forward.restype = i
        L.ttt_scan_forward_grad_norms.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i,
                                                  ctypes.c_float, u, i, vp, vp, vp, vp, vp, vp]
        L.ttt_scan_forward_grad_norms.restype = i
        L.ttt_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i,
                                      ctypes.c_float, u, vp, vp, vp]
        L.ttt_decode_step.restype = i
        L.ttt_scan_kernel_choice.argtypes = [i, i, i, i, u, i]
        L.ttt_scan_kernel_choice.restype = i
        L.ttt_check_device_status.argtypes = [vp]
        L.ttt_check_device_status.restype = i
        L.ttt_status_string.argtypes = [i]
        L.ttt_status_string.restype = ctypes.c_char_p
        L.ttt_set_wait_limit.argtypes = [ctypes.c_longlong]
        L.ttt_set_wait_limit.restype = i
        L.ttt_scan_forward_host_workspace_bytes.argtypes = [i, i, i, i, u, i, i]
        L.ttt_scan_forward_host_workspace_bytes.restype = ctypes.c_size_t
        L.ttt_scan_forward_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i,
                                            ctypes.c_float, u, i, vp, vp, vp, i, vp,
                                            ctypes.c_size_t, vp]
        L.ttt_scan_forward_host.restype = i
        L.ttt_scan_backward_workspace_bytes.argtypes = [i, i, i, u]
        L.ttt_scan_backward_workspace_bytes.restype = ctypes.c_size_t
        L.ttt_scan_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, ctypes.c_float,
                                        u, i, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                        vp, ctypes.c_size_t, vp]
        L.ttt_scan_backward.restype = i
        L.ttt_probe_ffma.argtypes = [i, i, i, vp, ctypes.POINTER(ctypes.c_double), vp]
        L.ttt_probe_ffma.restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().ttt_status_string(int(status)).decode()


def check_device_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronise the stream and return the device status (TTT_OK when clean)."""
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(lib().ttt_check_device_status(ctypes.c_void_p(s.cuda_stream)))


def set_wait_limit(polls: int) -> None:
    rc = lib().ttt_set_wait_limit(int(polls))
    if rc != TTT_OK:
        raise TTTScanError(rc, "ttt_set_wait_limit")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_inputs(q, k, v, eta_logit, gate_logit, W0, gamma, beta, b, mask):
    """Shapes, dtypes and contiguity of a scan's inputs; returns the sizes."""
    if q.dim() != 4:
        raise ValueError("q must be [B, H, T, d]")
    B, H, T, d = q.shape
    in_dtype = q.dtype
    if in_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("inputs must be float32 or bfloat16")
    channel = gate_logit is not None and gate_logit.dim() == 4
    for name, t, shp in (("k", k, (B, H, T, d)), ("v", v, (B, H, T, d)),
                         ("eta_logit", eta_logit, (B, H, T)),
                         ("gate_logit", gate_logit, (B, H, T, d) if channel else (B, H, T))):
        if t is None and name == "gate_logit":
            continue
        if tuple(t.shape) != shp or t.dtype != in_dtype or not t.is_contiguous():
            raise ValueError(f"{name}: expected contiguous {shp} {in_dtype}")
    if tuple(W0.shape) != (B, H, d, d) or W0.dtype != torch.float32 or not W0.is_contiguous():
        raise ValueError("W0: expected contiguous [B, H, d, d] float32")
    for name, t in (("gamma", gamma), ("beta", beta)):
        if t is None:
            continue
        if tuple(t.shape) != (H, d) or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{name}: expected contiguous [H, d] float32")
    n_chunks = -(-T // b) if b > 0 else 0
    if mask is not None:
        if tuple(mask.shape) != (B, n_chunks) or mask.dtype != torch.uint8 or not mask.is_contiguous():
            raise ValueError(f"mask: expected contiguous [B, {n_chunks}] uint8")
    return B, H, T, d, in_dtype, channel, n_chunks


def _mode_bits(minibatch, lnjac, no_ln, in_dtype, out_dtype, force_simt, single_cta, ablate,
               norm_match, channel, kq_silu) -> int:
    return ((MODE_MINIBATCH if minibatch else 0) | (GRAD_LNJAC if lnjac else 0) |
            (NO_LN if no_ln else 0) | (IN_BF16 if in_dtype == torch.bfloat16 else 0) |
            (OUT_BF16 if out_dtype == torch.bfloat16 else 0) | (KERNEL_SIMT if force_simt else 0) |
            (KERNEL_SINGLE_CTA if single_cta else 0) | (GRAD_ABLATE if ablate else 0) |
            (GRAD_NORM_MATCH if norm_match else 0) | (GATE_CHANNEL if channel else 0) |
            (KQ_SILU if kq_silu else 0))


def host_workspace_bytes(B: int, H: int, T: int, d: int, mode: int, b: int,
                         seg_tokens: int = 0) -> int:
    """Device workspace of ``ttt_scan_forward_host`` (0 for invalid sizes)."""
    return int(lib().ttt_scan_forward_host_workspace_bytes(B, H, T, d, mode, b, seg_tokens))


def _scan_host(q, k, v, eta_logit, gate_logit, W0, gamma, beta, *, eps, minibatch, lnjac, no_ln,
               b, mask, out_dtype, force_simt, single_cta, ablate, norm_match, kq_silu, o, W_T,
               stream, seg_tokens: int = 0):
    """The end-to-end scan of host tensors through ``ttt_scan_forward_host``."""
    for name, t in (("q", q), ("k", k), ("v", v), ("eta_logit", eta_logit),
                    ("gate_logit", gate_logit), ("W0", W0), ("gamma", gamma), ("beta", beta),
                    ("mask", mask), ("o", o), ("W_T", W_T)):
        if t is not None and t.is_cuda:
            raise ValueError(f"{name}: with host inputs every tensor must be in host memory")
    B, H, T, d, in_dtype, channel, n_chunks = _check_inputs(q, k, v, eta_logit, gate_logit, W0,
                                                            gamma, beta, b, mask)
    out_dtype = out_dtype or in_dtype
    mode = _mode_bits(minibatch, lnjac, no_ln, in_dtype, out_dtype, force_simt, single_cta,
                      ablate, norm_match, channel, kq_silu)
    if o is None:
        o = torch.empty((B, H, T, d), dtype=out_dtype, pin_memory=True)
    if W_T is None:
        W_T = torch.empty((B, H, d, d), dtype=torch.float32, pin_memory=True)
    if (tuple(o.shape) != (B, H, T, d) or o.dtype != out_dtype or not o.is_contiguous() or
            tuple(W_T.shape) != (B, H, d, d) or W_T.dtype != torch.float32 or
            not W_T.is_contiguous()):
        raise ValueError("o / W_T: expected contiguous [B, H, T, d] out_dtype / [B, H, d, d] float32")
    dev = torch.device("cuda", torch.cuda.current_device())
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    nbytes = host_workspace_bytes(B, H, T, d, mode, b, seg_tokens)
    with torch.cuda.stream(s):
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    rc = lib().ttt_scan_forward_host(
        _ptr(q), _ptr(k), _ptr(v), _ptr(eta_logit), _ptr(gate_logit), _ptr(W0), _ptr(gamma),
        _ptr(beta), B, H, T, d, float(eps), mode, int(b), _ptr(mask), _ptr(o), _ptr(W_T),
        int(seg_tokens), _ptr(ws), ctypes.c_size_t(ws.numel()), ctypes.c_void_p(s.cuda_stream))
    if rc != TTT_OK:
        raise TTTScanError(rc)
    rc = check_device_status(s)  # synchronises the stream: o and W_T are in host memory
    if rc != TTT_OK:
        raise TTTScanError(rc, "device")
    return o, W_T


def scan(q, k, v, eta_logit, gate_logit, W0, gamma, beta, *, eps: float = 1e-6,
         minibatch: bool = False, lnjac: bool = False, no_ln: bool = False,
         b: int = 16, mask=None, out_dtype: Optional[torch.dtype] = None,
         force_simt: bool = False, single_cta: bool = False, ablate: bool = False,
         norm_match: bool = False, kq_silu: bool = False, want_chunks: bool = False,
         want_grad_norms: bool = False, o: Optional[torch.Tensor] = None,
         W_T: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None):
    """TTT-Linear scan ``(o, W_T) = scan(q, k, v, eta_logit, gate_logit, W0, gamma, beta)``.

    q, k, v: [B, H, T, d] fp32 or bf16; eta_logit: [B, H, T] with the same
    dtype; gate_logit: [B, H, T], or [B, H, T, d] for a per-feature gate, or
    None; W0: [B, H, d, d] fp32 (z = W k);
    gamma, beta: [H, d] fp32 (may be None with ``no_ln``); mask: [B, ceil(T/b)]
    uint8 or None. ``out_dtype`` defaults to the input dtype. ``force_simt``
    keeps mini-batch mode on the CUDA-core kernel; ``single_cta`` keeps
    per-token mode on one CTA per head (see ``kernel_choice``). ``ablate``
    selects the ablation gradient (the LayerNorm Jacobian applied to
    -gamma * v), ``norm_match`` rescales it per token to the full gradient's norm.
    ``kq_silu`` runs the `:mlp` variant (SiLU on every key and query).
    ``want_grad_norms`` (with ``ablate``) also returns [B, H, T, 2]
    fp32: per token the norms of the full and of the ablated gradient (zeros
    on SKIP chunks), after W_T (and the chunk snapshots, if asked for).

    CUDA tensors run on ``stream`` (default: the current stream) and return
    without synchronising. CPU tensors take the end-to-end path, the library's
    ``ttt_scan_forward_host``: the sequence is copied to the current CUDA device
    in segments that overlap the scan of the previous segment and the copy-back
    of the one before, and the call returns once o / W_T are in host memory
    (page-locked host tensors make the copies asynchronous). With
    ``want_chunks`` or ``want_grad_norms``, CPU tensors are copied in whole,
    scanned and copied back on ``stream``.
    """
    host = not q.is_cuda
    if host and not want_chunks and not want_grad_norms:
        return _scan_host(q, k, v, eta_logit, gate_logit, W0, gamma, beta, eps=eps,
                          minibatch=minibatch, lnjac=lnjac, no_ln=no_ln, b=b, mask=mask,
                          out_dtype=out_dtype, force_simt=force_simt, single_cta=single_cta,
                          ablate=ablate, norm_match=norm_match, kq_silu=kq_silu, o=o, W_T=W_T,
                          stream=stream)
    if host:
        dev = torch.device("cuda", torch.cuda.current_device())
        s = stream if stream is not None else torch.cuda.current_stream(dev)
        with torch.cuda.stream(s):
            mv = lambda t: None if t is None else t.to(dev, non_blocking=True)
            q, k, v, eta_logit, gate_logit, W0, gamma, beta, mask = map(
                mv, (q, k, v, eta_logit, gate_logit, W0, gamma, beta, mask))
        o_dev, wt_dev = None, None
    else:
        o_dev, wt_dev = o, W_T
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
    B, H, T, d, in_dtype, channel, n_chunks = _check_inputs(q, k, v, eta_logit, gate_logit, W0,
                                                            gamma, beta, b, mask)
    out_dtype = out_dtype or in_dtype
    mode = _mode_bits(minibatch, lnjac, no_ln, in_dtype, out_dtype, force_simt, single_cta,
                      ablate, norm_match, channel, kq_silu)
    with torch.cuda.stream(s):
        if o_dev is None:
            o_dev = torch.empty((B, H, T, d), dtype=out_dtype, device=q.device)
        if wt_dev is None:
            wt_dev = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
        wc = (torch.empty((B, H, n_chunks + 1, d, d), dtype=torch.float32, device=q.device)
              if want_chunks else None)
        gn = (torch.empty((B, H, T, 2), dtype=torch.float32, device=q.device)
              if want_grad_norms else None)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(eta_logit), _ptr(gate_logit), _ptr(W0), _ptr(gamma),
            _ptr(beta), B, H, T, d, float(eps), mode, int(b), _ptr(mask), _ptr(o_dev),
            _ptr(wt_dev), _ptr(wc))
    if want_grad_norms:
        rc = lib().ttt_scan_forward_grad_norms(*args, _ptr(gn), ctypes.c_void_p(s.cuda_stream))
    else:
        rc = lib().ttt_scan_forward(*args, ctypes.c_void_p(s.cuda_stream))
    if rc != TTT_OK:
        raise TTTScanError(rc)
    if host:
        o_h = o if o is not None else torch.empty(o_dev.shape, dtype=o_dev.dtype, pin_memory=True)
        wt_h = W_T if W_T is not None else torch.empty(wt_dev.shape, dtype=torch.float32,
                                                       pin_memory=True)
        with torch.cuda.stream(s):
            o_h.copy_(o_dev, non_blocking=True)
            wt_h.copy_(wt_dev, non_blocking=True)
            extra = tuple(x.to("cpu") for x in (wc, gn) if x is not None)
        rc = check_device_status(s)
        if rc != TTT_OK:
            raise TTTScanError(rc, "device")
        return (o_h, wt_h) + extra
    extra = ((wc,) if want_chunks else ()) + ((gn,) if want_grad_norms else ())
    return (o_dev, wt_dev) + extra


def scan_backward(q, k, v, eta_logit, gate_logit, gamma, beta, W_chunks, dO, dW_T=None, *,
                  eps: float = 1e-6, minibatch: bool = False, lnjac: bool = False,
                  no_ln: bool = False, ablate: bool = False, kq_silu: bool = False, b: int = 16,
                  mask=None, workspace: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> dict:
    """Gradients of ``<dO, o> + <dW_T, W_T>`` for a ``scan`` with the same arguments.

    Inputs as for ``scan`` (CUDA tensors), plus ``W_chunks`` [B, H, ceil(T/b) + 1,
    d, d] (the snapshots ``scan(..., want_chunks=True)`` returns), ``dO`` [B, H, T,
    d] fp32 and ``dW_T`` [B, H, d, d] fp32 or None (zero). ``workspace`` (optional)
    is a device tensor of at least ``backward_workspace_bytes`` bytes; by default
    one is allocated here. Returns a dict of fp32 tensors dq, dk, dv, deta_logit,
    dgate_logit (None without a gate), dW0, dgamma, dbeta (None with ``no_ln``).
    Runs on ``stream`` (default: the current stream) without synchronising.
    """
    if q.dim() != 4 or not q.is_cuda:
        raise ValueError("q must be a CUDA tensor [B, H, T, d]")
    B, H, T, d = q.shape
    in_dtype = q.dtype
    channel = gate_logit is not None and gate_logit.dim() == 4
    n_chunks = -(-T // b) if b > 0 else 0
    for name, t, shp, dt in (("k", k, (B, H, T, d), in_dtype), ("v", v, (B, H, T, d), in_dtype),
                             ("eta_logit", eta_logit, (B, H, T), in_dtype),
                             ("gate_logit", gate_logit, (B, H, T, d) if channel else (B, H, T),
                              in_dtype),
                             ("W_chunks", W_chunks, (B, H, n_chunks + 1, d, d), torch.float32),
                             ("dO", dO, (B, H, T, d), torch.float32),
                             ("dW_T", dW_T, (B, H, d, d), torch.float32),
                             ("mask", mask, (B, n_chunks), torch.uint8)):
        if t is None and name in ("gate_logit", "dW_T", "mask"):
            continue
        if tuple(t.shape) != shp or t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"{name}: expected contiguous {shp} {dt}")
    mode = ((MODE_MINIBATCH if minibatch else 0) | (GRAD_LNJAC if lnjac else 0) |
            (NO_LN if no_ln else 0) | (IN_BF16 if in_dtype == torch.bfloat16 else 0) |
            (GRAD_ABLATE if ablate else 0) | (GATE_CHANNEL if channel else 0) |
            (KQ_SILU if kq_silu else 0))
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    need = int(lib().ttt_scan_backward_workspace_bytes(B, H, d, mode))
    f32 = dict(dtype=torch.float32, device=q.device)
    with torch.cuda.stream(s):
        out = dict(dq=torch.empty((B, H, T, d), **f32), dk=torch.empty((B, H, T, d), **f32),
                   dv=torch.empty((B, H, T, d), **f32), deta_logit=torch.empty((B, H, T), **f32),
                   dgate_logit=None if gate_logit is None else torch.empty(gate_logit.shape, **f32),
                   dW0=torch.empty((B, H, d, d), **f32),
                   dgamma=None if no_ln else torch.empty((H, d), **f32),
                   dbeta=None if no_ln else torch.empty((H, d), **f32))
        if workspace is None and need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().ttt_scan_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(eta_logit), _ptr(gate_logit), _ptr(gamma), _ptr(beta),
        B, H, T, d, float(eps), mode, int(b), _ptr(mask), _ptr(W_chunks), _ptr(dO), _ptr(dW_T),
        _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["deta_logit"]),
        _ptr(out["dgate_logit"]), _ptr(out["dW0"]), _ptr(out["dgamma"]), _ptr(out["dbeta"]),
        _ptr(workspace), ws_bytes, ctypes.c_void_p(s.cuda_stream))
    if rc != TTT_OK:
        raise TTTScanError(rc, "ttt_scan_backward")
    return out


def backward_workspace_bytes(B: int, H: int, d: int, *, no_ln: bool = False) -> int:
    """Bytes of device workspace ``ttt_scan_backward`` needs for these sizes."""
    return int(lib().ttt_scan_backward_workspace_bytes(B, H, d, NO_LN if no_ln else 0))


def kernel_choice(B: int, H: int, T: int, d: int, *, minibatch: bool = False,
                  lnjac: bool = False, no_ln: bool = False, in_bf16: bool = False,
                  out_bf16: bool = False, b: int = 16, force_simt: bool = False,
                  single_cta: bool = False, ablate: bool = False, norm_match: bool = False,
                  kq_silu: bool = False, gate_channel: bool = False) -> int:
    """The KERNEL_* identifier ``scan`` would run for these sizes (launches nothing)."""
    mode = ((MODE_MINIBATCH if minibatch else 0) | (GRAD_LNJAC if lnjac else 0) |
            (NO_LN if no_ln else 0) | (IN_BF16 if in_bf16 else 0) | (OUT_BF16 if out_bf16 else 0) |
            (KERNEL_SIMT if force_simt else 0) | (KERNEL_SINGLE_CTA if single_cta else 0) |
            (GRAD_ABLATE if ablate else 0) | (GRAD_NORM_MATCH if norm_match else 0) |
            (KQ_SILU if kq_silu else 0) | (GATE_CHANNEL if gate_channel else 0))
    rc = lib().ttt_scan_kernel_choice(B, H, T, d, mode, b)
    if rc < 0:
        raise TTTScanError(rc, "ttt_scan_kernel_choice")
    return rc


def decode_step(q, k, v, eta_logit, gate_logit, W, gamma, beta, *, eps: float = 1e-6,
                lnjac: bool = False, no_ln: bool = False, ablate: bool = False,
                norm_match: bool = False, kq_silu: bool = False, update=None,
                out_dtype: Optional[torch.dtype] = None, o: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None):
    """One streaming step ``o = decode_step(q, k, v, eta_logit, gate_logit, W, gamma, beta)``.

    q, k, v: [B, H, d] fp32 or bf16; eta_logit: [B, H] (same dtype); gate_logit:
    [B, H], or [B, H, d] for a per-feature gate, or None; W: [B, H, d, d] fp32,
    UPDATED IN PLACE; gamma, beta: [H, d] fp32 (may be None with ``no_ln``);
    update: [B] uint8 (0 = SKIP) or None. Returns o [B, H, d] (``out_dtype``,
    default the input dtype).

    CUDA tensors run on ``stream`` without synchronising. CPU tensors take the
    end-to-end path: inputs and W go to the current CUDA device, the step runs
    there, and o and the new W come back (W is overwritten in host memory); the
    copies and the step are all issued on ``stream``, so they are ordered.
    ``kq_silu`` runs the `:mlp` variant (SiLU on k and q).
    """
    host = not q.is_cuda
    W_host = None
    if host:
        dev = torch.device("cuda", torch.cuda.current_device())
        s = stream if stream is not None else torch.cuda.current_stream(dev)
        W_host = W
        with torch.cuda.stream(s):
            mv = lambda t: None if t is None else t.to(dev, non_blocking=True)
            q, k, v, eta_logit, gate_logit, W, gamma, beta, update = map(
                mv, (q, k, v, eta_logit, gate_logit, W, gamma, beta, update))
        o_dev = None
    else:
        o_dev = o
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
    if q.dim() != 3:
        raise ValueError("q must be [B, H, d]")
    B, H, d = q.shape
    in_dtype = q.dtype
    if in_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("inputs must be float32 or bfloat16")
    channel = gate_logit is not None and gate_logit.dim() == 3
    for name, t, shp in (("k", k, (B, H, d)), ("v", v, (B, H, d)), ("eta_logit", eta_logit, (B, H)),
                         ("gate_logit", gate_logit, (B, H, d) if channel else (B, H))):
        if t is None and name == "gate_logit":
            continue
        if tuple(t.shape) != shp or t.dtype != in_dtype or not t.is_contiguous():
            raise ValueError(f"{name}: expected contiguous {shp} {in_dtype}")
    if tuple(W.shape) != (B, H, d, d) or W.dtype != torch.float32 or not W.is_contiguous():
        raise ValueError("W: expected contiguous [B, H, d, d] float32")
    for name, t in (("gamma", gamma), ("beta", beta)):
        if t is not None and (tuple(t.shape) != (H, d) or t.dtype != torch.float32
                              or not t.is_contiguous()):
            raise ValueError(f"{name}: expected contiguous [H, d] float32")
    if update is not None and (tuple(update.shape) != (B,) or update.dtype != torch.uint8):
        raise ValueError("update: expected [B] uint8")
    out_dtype = out_dtype or in_dtype
    mode = ((GRAD_LNJAC if lnjac else 0) | (NO_LN if no_ln else 0) |
            (IN_BF16 if in_dtype == torch.bfloat16 else 0) |
            (OUT_BF16 if out_dtype == torch.bfloat16 else 0) | (GATE_CHANNEL if channel else 0) |
            (GRAD_ABLATE if ablate else 0) | (GRAD_NORM_MATCH if norm_match else 0) |
            (KQ_SILU if kq_silu else 0))
    if o_dev is None:
        with torch.cuda.stream(s):
            o_dev = torch.empty((B, H, d), dtype=out_dtype, device=q.device)
    rc = lib().ttt_decode_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(eta_logit), _ptr(gate_logit), _ptr(W), _ptr(gamma),
        _ptr(beta), B, H, d, float(eps), mode, _ptr(update), _ptr(o_dev),
        ctypes.c_void_p(s.cuda_stream))
    if rc != TTT_OK:
        raise TTTScanError(rc, "ttt_decode_step")
    if host:
        o_h = o if o is not None else torch.empty(o_dev.shape, dtype=o_dev.dtype, pin_memory=True)
        with torch.cuda.stream(s):
            o_h.copy_(o_dev, non_blocking=True)
            W_host.copy_(W, non_blocking=True)
        rc = check_device_status(s)
        if rc != TTT_OK:
            raise TTTScanError(rc, "device")
        return o_h
    return o_dev


def probe_ffma(blocks: int, threads: int, iters: int, sink: torch.Tensor,
               stream: Optional[torch.cuda.Stream] = None) -> float:
    """Enqueue the FFMA throughput probe; returns the flop count of the launch."""
    flops = ctypes.c_double(0.0)
    s = stream if stream is not None else torch.cuda.current_stream()
    rc = lib().ttt_probe_ffma(blocks, threads, iters, _ptr(sink), ctypes.byref(flops),
                              ctypes.c_void_p(s.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"ttt_probe_ffma failed ({rc})")
    return flops.value
