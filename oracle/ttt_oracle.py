"""ctypes wrapper around the plain CPU oracle of the TTT-Linear scan.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg use this module; the product path never imports it. It shares
no code with the CUDA package.

The oracle follows "Edifice.Recurrent.TTT", section "Equations (TTT-Linear)"
for the per-token recurrence, "Error Correction in Trained TTT Layers"
(Abstract) for the gradient through the LayerNorm Jacobian, PonderTTT
("Technical Architecture": dual-form updates; "Core Idea": SKIP/UPDATE
decisions per chunk) for the mini-batch mode and the mask. The arithmetic lives
in ``ttt_oracle.cpp``; this file only marshals numpy arrays.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "ttt_oracle.cpp"
_LIB = _HERE / "libttt_oracle.so"

# Mode bits (same integers as the public scan interface).
MINIBATCH = 1 << 0
GRAD_LNJAC = 1 << 1
NO_LN = 1 << 2
GATE_CHANNEL = 1 << 6
GRAD_ABLATE = 1 << 8
GRAD_NORM_MATCH = 1 << 9
# The `:mlp` variant: SiLU on keys and queries before the inner model (oracle
# only for now; the bit is reserved for the scan's interface).
KQ_SILU = 1 << 10

_lib = None


def build(force: bool = False) -> Path:
    """Compile the oracle into ``libttt_oracle.so`` next to its source."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.tmp{os.getpid()}")
        cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared",
               "-fno-fast-math", "-ffp-contract=off", str(_SRC), "-o", str(tmp)]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # A pre-built copy may be named explicitly (used by the mutation check
        # of the pins, which loads deliberately broken builds of this oracle).
        override = os.environ.get("TTT_ORACLE_LIB")
        if override:
            lib = ctypes.CDLL(override)
        else:
            build()
            lib = ctypes.CDLL(str(_LIB))
        dp = ctypes.POINTER(ctypes.c_double)
        fp = ctypes.POINTER(ctypes.c_float)
        u8p = ctypes.POINTER(ctypes.c_ubyte)
        i = ctypes.c_int
        lib.ttt_oracle_forward_f64.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, i, i, i, i,
                                               ctypes.c_double, ctypes.c_uint, i, u8p,
                                               dp, dp, dp, dp, i]
        lib.ttt_oracle_forward_f64.restype = i
        lib.ttt_oracle_forward_f32.argtypes = [fp, fp, fp, fp, fp, fp, fp, fp, i, i, i, i,
                                               ctypes.c_float, ctypes.c_uint, i, u8p,
                                               fp, fp, fp, fp, i]
        lib.ttt_oracle_forward_f32.restype = i
        lib.ttt_oracle_lngrad_f64.argtypes = [dp, dp, dp, dp, i, ctypes.c_double,
                                              ctypes.c_uint, dp, dp, dp, dp]
        lib.ttt_oracle_lngrad_f64.restype = i
        lib.ttt_oracle_backward_f64.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, i, i, i, i,
                                                ctypes.c_double, ctypes.c_uint, i, u8p, dp, dp,
                                                dp, dp, dp, dp, dp, dp, dp, dp]
        lib.ttt_oracle_backward_f64.restype = i
        lib.ttt_oracle_max_threads.argtypes = []
        lib.ttt_oracle_max_threads.restype = i
        _lib = lib
    return _lib


def _ptr(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def max_threads() -> int:
    return int(_load().ttt_oracle_max_threads())


def forward(q, k, v, eta_logit, gate_logit, W0, gamma, beta, *, eps: float,
            mode: int, b: int = 16, mask=None, want_chunks: bool = False,
            want_grad_norms: bool = False, nthreads: int = 0, dtype=np.float64):
    """Run the oracle scan.

    Shapes: q, k, v [B, H, T, d]; eta_logit [B, H, T]; gate_logit [B, H, T], or
    [B, H, T, d] with GATE_CHANNEL in ``mode``, or None; W0 [B, H, d, d] with
    z = W k; gamma, beta [H, d] (ignored with NO_LN);
    mask [B, ceil(T/b)] uint8 (1 = UPDATE) or None.

    Returns ``(o, W_T)`` or ``(o, W_T, W_chunks)`` when ``want_chunks``; W_chunks
    has shape [B, H, ceil(T/b) + 1, d, d] and holds W before every chunk and
    after the last one. ``want_grad_norms`` (GRAD_ABLATE only) appends
    ``grad_norms`` [B, H, T, 2]: per token the L2 norm of the full
    Jacobian-form gradient and of the ablated gradient before any norm
    matching (zeros on SKIP chunks, which take no gradient).
    ``dtype=np.float32`` runs the float twin.
    """
    lib = _load()
    f64 = np.dtype(dtype) == np.float64
    ct = ctypes.c_double if f64 else ctypes.c_float
    cvt = (lambda a: None if a is None else np.ascontiguousarray(a, dtype=dtype))
    q, k, v, eta_logit, gate_logit, W0 = map(cvt, (q, k, v, eta_logit, gate_logit, W0))
    B, H, T, d = q.shape
    if gamma is None:
        gamma = np.ones((H, d))
    if beta is None:
        beta = np.zeros((H, d))
    gamma, beta = cvt(gamma), cvt(beta)
    if b <= 0:
        raise ValueError(f"chunk size b must be positive, got {b}")
    if gate_logit is not None:
        gshape = (B, H, T, d) if mode & GATE_CHANNEL else (B, H, T)
        if gate_logit.shape != gshape:
            raise ValueError(f"gate_logit: expected shape {gshape}, got {gate_logit.shape}")
    n_chunks = -(-T // b)
    if mask is not None:
        mask = np.ascontiguousarray(mask, dtype=np.uint8)
        assert mask.shape == (B, n_chunks), mask.shape
    o = np.empty((B, H, T, d), dtype=dtype)
    W_T = np.empty((B, H, d, d), dtype=dtype)
    W_chunks = np.empty((B, H, n_chunks + 1, d, d), dtype=dtype) if want_chunks else None
    gnorms = np.empty((B, H, T, 2), dtype=dtype) if want_grad_norms else None
    fn = lib.ttt_oracle_forward_f64 if f64 else lib.ttt_oracle_forward_f32
    rc = fn(_ptr(q, ct), _ptr(k, ct), _ptr(v, ct), _ptr(eta_logit, ct),
            _ptr(gate_logit, ct), _ptr(W0, ct), _ptr(gamma, ct), _ptr(beta, ct),
            B, H, T, d, eps, mode, b, _ptr(mask, ctypes.c_ubyte),
            _ptr(o, ct), _ptr(W_T, ct), _ptr(W_chunks, ct), _ptr(gnorms, ct), nthreads)
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (rc={rc})")
    out = (o, W_T) + ((W_chunks,) if want_chunks else ()) + ((gnorms,) if want_grad_norms else ())
    return out


def backward(q, k, v, eta_logit, gate_logit, W0, gamma, beta, dO, dW_T, *, eps: float,
             mode: int, b: int = 16, mask=None):
    """Backward of the per-token scan: the gradients of L = <dO, o> + <dW_T, W_T>
    with respect to every input, by reverse mode through the tokens.

    Shapes as for ``forward``; dO [B, H, T, d], dW_T [B, H, d, d]. Returns a dict
    with dq, dk, dv, deta_logit, dgate_logit (None without a gate), dW0, dgamma,
    dbeta (summed over the batch rows; None with NO_LN). Per-token or
    mini-batch mode; the SIMPLE, LN-Jacobian, no-LayerNorm or ablation gradient
    (not norm matching); the SiLU variant (KQ_SILU).
    """
    lib = _load()
    dp = ctypes.c_double
    cvt = (lambda a: None if a is None else np.ascontiguousarray(a, dtype=np.float64))
    q, k, v, eta_logit, gate_logit, W0, dO, dW_T = map(
        cvt, (q, k, v, eta_logit, gate_logit, W0, dO, dW_T))
    B, H, T, d = q.shape
    no_ln = bool(mode & NO_LN)
    gamma = np.ones((H, d)) if gamma is None else cvt(gamma)
    beta = np.zeros((H, d)) if beta is None else cvt(beta)
    if mask is not None:
        mask = np.ascontiguousarray(mask, dtype=np.uint8)
    out = dict(dq=np.empty_like(q), dk=np.empty_like(k), dv=np.empty_like(v),
               deta_logit=np.empty_like(eta_logit),
               dgate_logit=None if gate_logit is None else np.empty_like(gate_logit),
               dW0=np.empty_like(W0), dgamma=np.zeros((H, d)), dbeta=np.zeros((H, d)))
    rc = lib.ttt_oracle_backward_f64(
        _ptr(q, dp), _ptr(k, dp), _ptr(v, dp), _ptr(eta_logit, dp), _ptr(gate_logit, dp),
        _ptr(W0, dp), _ptr(gamma, dp), _ptr(beta, dp), B, H, T, d, eps, mode, b,
        _ptr(mask, ctypes.c_ubyte), _ptr(dO, dp), _ptr(dW_T, dp), _ptr(out["dq"], dp),
        _ptr(out["dk"], dp), _ptr(out["dv"], dp), _ptr(out["deta_logit"], dp),
        _ptr(out["dgate_logit"], dp), _ptr(out["dW0"], dp), _ptr(out["dgamma"], dp),
        _ptr(out["dbeta"], dp))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (rc={rc})")
    if no_ln:
        out["dgamma"] = out["dbeta"] = None
    return out


def decode_step(q, k, v, eta_logit, gate_logit, W, gamma, beta, *, eps: float,
                mode: int, update=None, dtype=np.float64):
    """One streaming step: the per-token recurrence for a single token.

    q, k, v [B, H, d]; eta_logit [B, H]; gate_logit [B, H] (or [B, H, d] with
    GATE_CHANNEL, or None); W [B, H, d, d]; update [B] uint8 (0 = SKIP) or None.
    Returns ``(o [B, H, d], W_new [B, H, d, d])``. This is ``forward`` with
    T = 1 and a one-token mask chunk; it adds no arithmetic of its own.
    """
    if mode & MINIBATCH:
        raise ValueError("a single-token step has no mini-batch form")
    ex = lambda a: None if a is None else np.asarray(a)[:, :, None]
    m = None if update is None else np.asarray(update, dtype=np.uint8).reshape(-1, 1)
    o, W_new = forward(ex(q), ex(k), ex(v), ex(eta_logit), ex(gate_logit), W, gamma, beta,
                       eps=eps, mode=mode, b=1, mask=m, dtype=dtype)
    return o[:, :, 0], W_new


def lngrad(z, v, gamma, beta, *, eps: float, mode: int, want_norms: bool = False):
    """One inner LayerNorm + gradient on a single d-vector.

    Returns ``(pred, G, xhat)``; with NO_LN, pred = xhat = z and G = z - v.
    GRAD_ABLATE gives the ablation gradient (prediction removed, LayerNorm
    Jacobian kept), GRAD_NORM_MATCH additionally rescales it to the norm of the
    full Jacobian-form gradient. ``want_norms`` (GRAD_ABLATE only) appends the
    pair (norm of the full gradient, norm of the ablated one before matching).
    """
    lib = _load()
    z = np.ascontiguousarray(z, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    d = z.shape[0]
    gamma = np.ones(d) if gamma is None else np.ascontiguousarray(gamma, dtype=np.float64)
    beta = np.zeros(d) if beta is None else np.ascontiguousarray(beta, dtype=np.float64)
    pred, G, xhat = np.empty(d), np.empty(d), np.empty(d)
    norms = np.empty(2) if want_norms else None
    dp = ctypes.c_double
    rc = lib.ttt_oracle_lngrad_f64(_ptr(z, dp), _ptr(v, dp), _ptr(gamma, dp), _ptr(beta, dp),
                                   d, eps, mode, _ptr(pred, dp), _ptr(G, dp), _ptr(xhat, dp),
                                   _ptr(norms, dp))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (rc={rc})")
    return (pred, G, xhat, norms) if want_norms else (pred, G, xhat)


def forward_heads(inputs: dict, heads, *, eps: float, mode: int, b: int,
                  nthreads: int = 0):
    """Oracle on a sample of (batch row, head) pairs of a larger problem.

    ``inputs`` holds full-size host arrays (keys q, k, v, eta_logit, gate_logit,
    W0, gamma, beta, mask). Heads are independent recurrences, so each sampled
    head is run alone with its own batch row's mask and its own gamma/beta.
    Returns a list of ``(o [T, d], W_T [d, d])`` in the order of ``heads``.
    """
    out = []
    for bi, h in heads:
        g = inputs.get("gate_logit")
        m = inputs.get("mask")
        gam = inputs.get("gamma")
        bet = inputs.get("beta")
        o, W_T = forward(
            inputs["q"][bi:bi + 1, h:h + 1], inputs["k"][bi:bi + 1, h:h + 1],
            inputs["v"][bi:bi + 1, h:h + 1], inputs["eta_logit"][bi:bi + 1, h:h + 1],
            None if g is None else g[bi:bi + 1, h:h + 1],
            inputs["W0"][bi:bi + 1, h:h + 1],
            None if gam is None else gam[h:h + 1], None if bet is None else bet[h:h + 1],
            eps=eps, mode=mode, b=b, mask=None if m is None else m[bi:bi + 1],
            nthreads=nthreads)
        out.append((o[0, 0], W_T[0, 0]))
    return out
