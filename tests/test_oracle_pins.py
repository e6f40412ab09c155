"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each test names the passage it rests on. Together they are chosen so that a
plausible slip in the oracle (a dropped term, a wrong sign or index, a
transposed operand, a pre-/post-update mix-up, a wrong chunk boundary) fails
at least one of them:

* hand-evaluated single-token example at d = 2 (golden file);
* LayerNorm invariants and the d = 2 closed form;
* central finite differences of the squared-error loss (LNJAC, NO_LN);
* eta == 0 and all-SKIP freeze W exactly;
* NO_LN equals the brute-force delta rule, and causal linear attention for
  orthogonal keys from W0 = 0;
* exact overwrite at eta ||k||^2 = 1;
* column sums of W conserved under the LNJAC gradient;
* cancellation of the prediction-derived gradient term as eps -> 0;
* mini-batch with b = 1, or with keys orthogonal inside each chunk, equals the
  per-token recurrence; mini-batch with b = T as one vectorised expression;
* chaining (resume from W_T), mask == eta forced to 0 on the same chunks;
* the per-channel output gate is elementwise: it leaves W alone, scales each
  feature of the ungated output by its own sigmoid, and a gate that is the same
  on every feature reproduces the scalar gate;
* a chain of single-token steps is the per-token scan with a one-token mask;
* the ablation gradient is the full Jacobian-form gradient minus its
  prediction-derived part (the P8 closed form at gamma = 1, beta = 0), is
  linear in v and vanishes at v = 0; norm matching gives the full gradient's
  norm in the ablation's direction.
"""

import numpy as np
import pytest

import oracle
from oracle import (GATE_CHANNEL, GRAD_ABLATE, GRAD_LNJAC, GRAD_NORM_MATCH, KQ_SILU, MINIBATCH,
                    NO_LN)
from test_sequence_layers_02_b200.workloads import make_inputs
from tests.conftest import load_golden


def sig(x):
    return 1.0 / (1.0 + np.exp(-np.asarray(x, dtype=np.float64)))


def f64(inp):
    return {k: (None if v is None else np.asarray(v, dtype=np.float64)) if k != "mask" else v
            for k, v in inp.items()}


def run(inp, *, mode, b=16, eps=1e-5, mask="inp", want_chunks=False):
    m = inp.get("mask") if isinstance(mask, str) else mask
    return oracle.forward(inp["q"], inp["k"], inp["v"], inp["eta_logit"], inp["gate_logit"],
                          inp["W0"], inp["gamma"], inp["beta"], eps=eps, mode=mode, b=b,
                          mask=m, want_chunks=want_chunks)


# ----------------------------------------------------------------------------
# Hand-evaluated example ("Edifice.Recurrent.TTT", Equations (TTT-Linear)).
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("name,mode", [("SIMPLE", 0), ("LNJAC", GRAD_LNJAC), ("NO_LN", NO_LN)])
def test_p2_hand_example_d2(name, mode):
    g = load_golden("p2_d2_single_token.txt")
    d = 2
    W0 = np.array(g["W0"]).reshape(1, 1, d, d)
    k = np.array(g["k"]).reshape(1, 1, 1, d)
    q = np.array(g["q"]).reshape(1, 1, 1, d)
    v = np.array(g["v"]).reshape(1, 1, 1, d)
    gam = np.array(g["gamma"]).reshape(1, d)
    bet = np.array(g["beta"]).reshape(1, d)
    el = np.full((1, 1, 1), g["eta_logit"])
    gl = np.full((1, 1, 1), g["gate_logit"])
    for minib in (0, MINIBATCH):
        o, W1 = oracle.forward(q, k, v, el, gl, W0, gam, bet, eps=g["eps"], mode=mode | minib, b=1)
        np.testing.assert_allclose(W1.ravel(), g[f"{name}.W1"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(o.ravel(), g[f"{name}.o"], rtol=0, atol=1e-14)
    pred, G, xhat = oracle.lngrad(np.array(g["z"]), np.array(g["v"]), gam[0], bet[0],
                                  eps=g["eps"], mode=mode)
    np.testing.assert_allclose(G, g[f"{name}.G"], rtol=0, atol=1e-14)
    if name != "NO_LN":
        np.testing.assert_allclose(xhat, g["xhat"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(pred, g["pred"], rtol=0, atol=1e-14)


def test_ln_closed_form_d2():
    """At d = 2, xhat = +-(delta/2)/sqrt(delta^2/4 + eps), delta = z1 - z2."""
    rng = np.random.default_rng(11)
    for _ in range(20):
        z = rng.normal(size=2) * rng.uniform(0.01, 3)
        eps = 10 ** rng.uniform(-8, 0)
        delta = z[0] - z[1]
        x1 = (delta / 2) / np.sqrt(delta * delta / 4 + eps)
        _, _, xhat = oracle.lngrad(z, np.zeros(2), None, None, eps=eps, mode=0)
        np.testing.assert_allclose(xhat, [x1, -x1], rtol=1e-13, atol=1e-15)


def test_ln_invariants():
    """mean(xhat) = 0 and mean(xhat^2) = var / (var + eps); pred = gamma xhat + beta."""
    rng = np.random.default_rng(12)
    for d in (3, 16, 64):
        for _ in range(5):
            z = rng.normal(size=d) * 0.3 + rng.normal()
            gam, bet = rng.normal(1, 0.1, d), rng.normal(0, 0.1, d)
            eps = 1e-3
            pred, G, xhat = oracle.lngrad(z, rng.normal(size=d), gam, bet, eps=eps, mode=0)
            var = np.var(z)
            assert abs(xhat.mean()) < 1e-14
            np.testing.assert_allclose((xhat ** 2).mean(), var / (var + eps), rtol=1e-12)
            np.testing.assert_allclose(pred, gam * xhat + bet, rtol=1e-13, atol=1e-14)
            # xhat is an increasing affine image of z
            assert np.all(np.argsort(xhat) == np.argsort(z))


# ----------------------------------------------------------------------------
# Finite differences of 1/2 ||gamma * LN(W k) + beta - v||^2
# ("Error Correction in Trained TTT Layers", Abstract: the inner gradient of
# the LayerNorm-based squared-error objective).
# ----------------------------------------------------------------------------

def _loss_np(W, k, v, gam, bet, eps, no_ln):
    z = W @ k
    if no_ln:
        pred = z
    else:
        pred = gam * (z - np.mean(z)) / np.sqrt(np.var(z) + eps) + bet
    r = pred - v
    return 0.5 * float(r @ r)


@pytest.mark.parametrize("no_ln", [False, True])
def test_p3_gradient_matches_finite_differences(no_ln):
    rng = np.random.default_rng(13)
    mode = NO_LN if no_ln else GRAD_LNJAC
    for d in (2, 3, 5, 8):
        W = rng.normal(size=(d, d)) * 0.3
        k, v, q = rng.normal(size=d), rng.normal(size=d), rng.normal(size=d)
        gam, bet = rng.normal(1, 0.2, d), rng.normal(0, 0.2, d)
        eps = 1e-3
        h = 1e-6
        fd = np.zeros((d, d))
        for r in range(d):
            for c in range(d):
                Wp, Wm = W.copy(), W.copy()
                Wp[r, c] += h
                Wm[r, c] -= h
                fd[r, c] = (_loss_np(Wp, k, v, gam, bet, eps, no_ln)
                            - _loss_np(Wm, k, v, gam, bet, eps, no_ln)) / (2 * h)
        # the oracle's update over one token: W1 = W0 - eta * grad_W
        el = np.zeros((1, 1, 1))
        eta = 0.5 / d
        _, W1 = oracle.forward(q.reshape(1, 1, 1, d), k.reshape(1, 1, 1, d), v.reshape(1, 1, 1, d),
                               el, None, W.reshape(1, 1, d, d), gam.reshape(1, d),
                               bet.reshape(1, d), eps=eps, mode=mode, b=1)
        grad = (W - W1[0, 0]) / eta
        scale = np.abs(fd).max()
        assert np.abs(grad - fd).max() <= 1e-7 * scale, (d, np.abs(grad - fd).max(), scale)


# ----------------------------------------------------------------------------
# eta == 0 and the SKIP mask (Abstract of "Error Correction in Trained TTT
# Layers": freezing all fast-weight updates; PonderTTT "Core Idea").
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [0, GRAD_LNJAC, MINIBATCH | GRAD_LNJAC, MINIBATCH])
def test_p1_eta_zero_freezes_W(mode):
    inp = f64(make_inputs(2, 2, 37, 16, seed=21, random_affine=True))
    inp["eta_logit"] = np.full_like(inp["eta_logit"], -1e4)
    o, W_T = run(inp, mode=mode, b=8)
    assert np.array_equal(W_T, inp["W0"])
    expect = sig(inp["gate_logit"])[..., None] * np.einsum("bhrc,bhtc->bhtr", inp["W0"], inp["q"])
    np.testing.assert_allclose(o, expect, rtol=1e-13, atol=1e-15)
    # an all-SKIP mask gives the same thing with ordinary logits
    inp2 = f64(make_inputs(2, 2, 37, 16, seed=21, random_affine=True))
    mask = np.zeros((2, 5), np.uint8)
    o2, W_T2 = run(inp2, mode=mode, b=8, mask=mask)
    assert np.array_equal(W_T2, inp2["W0"])
    np.testing.assert_allclose(o2, expect, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("mode", [0, GRAD_LNJAC, MINIBATCH | GRAD_LNJAC])
def test_mask_equals_eta_zero_on_skipped_chunks(mode):
    B, H, T, d, b = 2, 3, 45, 16, 8
    inp = f64(make_inputs(B, H, T, d, seed=22, random_affine=True, mask_p=0.5, b=b))
    mask = inp["mask"]
    assert mask.min() == 0 and mask.max() == 1
    o, W_T, Wc = run(inp, mode=mode, b=b, want_chunks=True)
    # same result when the SKIP chunks get eta_logit = -1e4 and no mask is given
    el = inp["eta_logit"].copy()
    for bi in range(B):
        for c in range(mask.shape[1]):
            if mask[bi, c] == 0:
                el[bi, :, c * b:(c + 1) * b] = -1e4
    inp2 = dict(inp, eta_logit=el)
    o2, W_T2 = run(inp2, mode=mode, b=b, mask=None)
    np.testing.assert_array_equal(W_T, W_T2)
    np.testing.assert_allclose(o, o2, rtol=1e-14, atol=1e-16)
    # W_chunks: bit-exact freeze on SKIP chunks, change on UPDATE chunks
    for bi in range(B):
        for c in range(mask.shape[1]):
            same = np.array_equal(Wc[bi, :, c + 1], Wc[bi, :, c])
            assert same == (mask[bi, c] == 0)
    np.testing.assert_array_equal(Wc[:, :, 0], inp["W0"])
    np.testing.assert_array_equal(Wc[:, :, -1], W_T)


# ----------------------------------------------------------------------------
# Delta rule / linear attention ("Edifice.Recurrent.TTT", Key Innovations:
# without the LayerNorm, TTT-Linear is linear attention with the delta rule).
# ----------------------------------------------------------------------------

def _delta_rule_product_form(W0, K, V, eta):
    """W_t = W0 prod_{s<=t}(I - eta_s k_s k_s^T) + sum_s eta_s v_s k_s^T prod_{r>s}(I - eta_r k_r k_r^T)."""
    T, d = K.shape
    I = np.eye(d)
    P = [I - eta[s] * np.outer(K[s], K[s]) for s in range(T)]
    Ws = []
    for t in range(T):
        acc = W0.copy()
        for s in range(t + 1):
            acc = acc @ P[s]
        for s in range(t + 1):
            term = eta[s] * np.outer(V[s], K[s])
            for r in range(s + 1, t + 1):
                term = term @ P[r]
            acc = acc + term
        Ws.append(acc)
    return Ws


def test_p5_no_ln_equals_brute_force_delta_rule():
    d, T = 6, 9
    inp = f64(make_inputs(1, 1, T, d, seed=23))
    K, V, Q = inp["k"][0, 0], inp["v"][0, 0], inp["q"][0, 0]
    eta = sig(inp["eta_logit"][0, 0]) / d
    gate = sig(inp["gate_logit"][0, 0])
    Ws = _delta_rule_product_form(inp["W0"][0, 0], K, V, eta)
    o, W_T = run(inp, mode=NO_LN, b=4)
    for t in range(T):
        np.testing.assert_allclose(o[0, 0, t], gate[t] * (Ws[t] @ Q[t]), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(W_T[0, 0], Ws[-1], rtol=1e-11, atol=1e-13)


def test_p5_orthogonal_keys_from_zero_is_causal_linear_attention():
    d, T = 16, 12
    rng = np.random.default_rng(24)
    basis, _ = np.linalg.qr(rng.normal(size=(d, d)))
    K = basis[:T] * rng.uniform(0.5, 2.0, size=(T, 1))   # mutually orthogonal keys
    Q, V = rng.normal(size=(T, d)), rng.normal(size=(T, d))
    el, gl = rng.normal(size=T), rng.normal(size=T)
    eta, gate = sig(el) / d, sig(gl)
    attn = np.tril(Q @ K.T) * eta[None, :]                # causal, inclusive of s = t
    expect = gate[:, None] * (attn @ V)
    for mode in (NO_LN, NO_LN | MINIBATCH):
        o, W_T = oracle.forward(Q[None, None], K[None, None], V[None, None], el[None, None],
                                gl[None, None], np.zeros((1, 1, d, d)), None, None,
                                eps=1e-5, mode=mode, b=5)
        np.testing.assert_allclose(o[0, 0], expect, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(W_T[0, 0], (V * eta[:, None]).T @ K, rtol=1e-12, atol=1e-13)


def test_p7_exact_overwrite():
    """No LN, k in {+-1}^d, eta = 1/d: eta ||k||^2 = 1, so W_t k_t = v_t and o_t = sig(g_t) v_t
    ("Edifice.Recurrent.TTT", Paper-Faithful Implementation item 2: the 1/d scaling)."""
    d, T = 16, 20
    rng = np.random.default_rng(25)
    K = rng.choice([-1.0, 1.0], size=(T, d))
    V = rng.normal(size=(T, d))
    el = np.full(T, 40.0)             # sigmoid(40) == 1 in double
    gl = rng.normal(size=T)
    assert sig(40.0) == 1.0
    o, _, Wc = oracle.forward(K[None, None], K[None, None], V[None, None], el[None, None],
                              gl[None, None], rng.normal(size=(1, 1, d, d)) * 0.02, None, None,
                              eps=1e-5, mode=NO_LN, b=1, want_chunks=True)
    np.testing.assert_allclose(o[0, 0], sig(gl)[:, None] * V, rtol=1e-12, atol=1e-12)
    for t in range(T):
        np.testing.assert_allclose(Wc[0, 0, t + 1] @ K[t], V[t], rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------
# Structure of the LayerNorm-Jacobian gradient ("Error Correction in Trained
# TTT Layers", Abstract).
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [GRAD_LNJAC, GRAD_LNJAC | MINIBATCH])
def test_p6_lnjac_conserves_column_sums(mode):
    inp = f64(make_inputs(2, 2, 64, 16, seed=26, random_affine=True))
    o, W_T = run(inp, mode=mode, b=16)
    # 1^T G = 0, so sum over the output index of W never changes
    np.testing.assert_allclose(W_T.sum(axis=2), inp["W0"].sum(axis=2), rtol=0, atol=1e-13)
    # and W does move
    assert np.abs(W_T - inp["W0"]).max() > 1e-2
    # the simplified gradient does not have this property
    o2, W_T2 = run(inp, mode=mode & ~GRAD_LNJAC, b=16)
    assert np.abs(W_T2.sum(axis=2) - inp["W0"].sum(axis=2)).max() > 1e-3


def test_p8_prediction_term_cancels_as_eps_to_zero():
    """gamma = 1, beta = 0: the gradient of the prediction part alone (v = 0) is
    xhat * eps / (s (var + eps)), which vanishes as eps -> 0."""
    rng = np.random.default_rng(27)
    d = 16
    z = rng.normal(size=d) * 0.05 + 0.01
    var = np.var(z)
    for eps in (1e-2, 1e-4, 1e-6, 1e-9):
        _, G0, xhat = oracle.lngrad(z, np.zeros(d), None, None, eps=eps, mode=GRAD_LNJAC)
        s = np.sqrt(var + eps)
        np.testing.assert_allclose(G0, xhat * eps / (s * (var + eps)), rtol=1e-9, atol=1e-15)
    # and with v != 0 the gradient is linear in v (the v part is J^T applied to -v)
    v1, v2 = rng.normal(size=d), rng.normal(size=d)
    G = lambda v: oracle.lngrad(z, v, None, None, eps=1e-6, mode=GRAD_LNJAC)[1]
    np.testing.assert_allclose(G(v1 + v2) - G(np.zeros(d)), (G(v1) - G(np.zeros(d))) + (G(v2) - G(np.zeros(d))),
                               rtol=1e-9, atol=1e-9)


# ----------------------------------------------------------------------------
# Ablation gradient ("Error Correction in Trained TTT Layers", Abstract: the
# prediction's contribution removed, the LayerNorm Jacobian retained).
# ----------------------------------------------------------------------------

def test_ablation_differs_from_full_by_the_prediction_term():
    """gamma = 1, beta = 0: G_full - G_ablation is the prediction part alone,
    xhat * eps / (s (var + eps)) (the same closed form as P8)."""
    rng = np.random.default_rng(28)
    d = 16
    z = rng.normal(size=d) * 0.05 + 0.01
    v = rng.normal(size=d)
    var = np.var(z)
    for eps in (1e-2, 1e-4, 1e-6):
        _, Gf, xhat = oracle.lngrad(z, v, None, None, eps=eps, mode=GRAD_LNJAC)
        _, Ga, _ = oracle.lngrad(z, v, None, None, eps=eps, mode=GRAD_ABLATE)
        s = np.sqrt(var + eps)
        np.testing.assert_allclose(Gf - Ga, xhat * eps / (s * (var + eps)), rtol=1e-9, atol=1e-13)


def test_ablation_with_affine_is_the_v_part_of_the_full_gradient():
    """Any gamma, beta: G_ablation(z, v) = G_full(z, v) - G_full(z, 0), is linear
    in v and is 0 at v = 0 (the prediction, beta included, no longer enters)."""
    rng = np.random.default_rng(29)
    d = 24
    z = rng.normal(size=d) * 0.3
    gam = 1.0 + 0.2 * rng.normal(size=d)
    bet = 0.3 * rng.normal(size=d)
    v1, v2 = rng.normal(size=d), rng.normal(size=d)
    full = lambda v: oracle.lngrad(z, v, gam, bet, eps=1e-6, mode=GRAD_LNJAC)[1]
    abl = lambda v: oracle.lngrad(z, v, gam, bet, eps=1e-6, mode=GRAD_ABLATE)[1]
    np.testing.assert_allclose(abl(v1), full(v1) - full(np.zeros(d)), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(abl(v1 + 2.5 * v2), abl(v1) + 2.5 * abl(v2), rtol=1e-9, atol=1e-12)
    np.testing.assert_array_equal(abl(np.zeros(d)), np.zeros(d))


def test_norm_matching_keeps_direction_and_takes_the_full_norm():
    rng = np.random.default_rng(30)
    d = 32
    z = rng.normal(size=d) * 0.2
    gam = 1.0 + 0.1 * rng.normal(size=d)
    bet = 0.1 * rng.normal(size=d)
    v = rng.normal(size=d)
    Gf = oracle.lngrad(z, v, gam, bet, eps=1e-6, mode=GRAD_LNJAC)[1]
    Ga = oracle.lngrad(z, v, gam, bet, eps=1e-6, mode=GRAD_ABLATE)[1]
    Gn = oracle.lngrad(z, v, gam, bet, eps=1e-6, mode=GRAD_ABLATE | GRAD_NORM_MATCH)[1]
    np.testing.assert_allclose(np.linalg.norm(Gn), np.linalg.norm(Gf), rtol=1e-12)
    lam = np.dot(Gn, Ga) / np.dot(Ga, Ga)
    assert lam > 0
    np.testing.assert_allclose(Gn, lam * Ga, rtol=1e-12, atol=1e-15)
    # zero ablation gradient (v = 0) stays zero
    G0 = oracle.lngrad(z, np.zeros(d), gam, bet, eps=1e-6, mode=GRAD_ABLATE | GRAD_NORM_MATCH)[1]
    np.testing.assert_array_equal(G0, np.zeros(d))


def test_grad_norms_are_the_norms_of_the_two_gradients():
    """The norms output is (||G_full||, ||G_ablation||), the latter before any
    norm matching; each gradient comes from its own (separately pinned) mode."""
    rng = np.random.default_rng(31)
    d = 32
    z = rng.normal(size=d) * 0.2
    gam = 1.0 + 0.1 * rng.normal(size=d)
    bet = 0.1 * rng.normal(size=d)
    v = rng.normal(size=d)
    Gf = oracle.lngrad(z, v, gam, bet, eps=1e-6, mode=GRAD_LNJAC)[1]
    Ga = oracle.lngrad(z, v, gam, bet, eps=1e-6, mode=GRAD_ABLATE)[1]
    for nm in (0, GRAD_NORM_MATCH):
        n = oracle.lngrad(z, v, gam, bet, eps=1e-6, mode=GRAD_ABLATE | nm, want_norms=True)[3]
        np.testing.assert_allclose(n, [np.linalg.norm(Gf), np.linalg.norm(Ga)], rtol=1e-12)
    with pytest.raises(ValueError):
        oracle.lngrad(z, v, gam, bet, eps=1e-6, mode=GRAD_LNJAC, want_norms=True)


def test_grad_norm_ratio_is_one_at_released_init_in_the_zero_eps_limit():
    """gamma = 1, beta = 0: the prediction-derived part cancels as eps -> 0
    ("Error Correction in Trained TTT Layers", Abstract), so the ratio
    ||G_ablation|| / ||G_full|| is 1 at eps = 0; for eps > 0 it differs from 1
    by at most ||xhat eps / (s (var + eps))|| / ||G_full|| (triangle inequality
    on the closed-form difference)."""
    rng = np.random.default_rng(32)
    d = 64
    z = rng.normal(size=d) * 0.1 + 0.02
    v = rng.normal(size=d)
    n0 = oracle.lngrad(z, v, None, None, eps=0.0, mode=GRAD_ABLATE, want_norms=True)[3]
    np.testing.assert_allclose(n0[1] / n0[0], 1.0, rtol=1e-12)
    var = np.var(z)
    for eps in (1e-2, 1e-4):
        n = oracle.lngrad(z, v, None, None, eps=eps, mode=GRAD_ABLATE, want_norms=True)[3]
        xhat = (z - z.mean()) / np.sqrt(var + eps)
        gap = np.linalg.norm(xhat) * eps / (np.sqrt(var + eps) * (var + eps))
        assert abs(n[1] - n[0]) <= gap * (1 + 1e-9) + 1e-15
        assert abs(n[1] / n[0] - 1.0) > 1e-6   # the bound is not vacuous here


@pytest.mark.parametrize("nm", [0, GRAD_NORM_MATCH], ids=["ablate", "ablate_nm"])
def test_scan_grad_norms_follow_the_state_trajectory(nm):
    """Per-token norms of the scan equal the single-vector norms at
    z_t = W_{t-1} k_t, with W_{t-1} read from the per-token state snapshots
    (b = 1) and the matvec done here in numpy; SKIP tokens take no gradient
    and report zeros."""
    inp = f64(make_inputs(1, 2, 20, 16, seed=33, random_affine=True, mask_p=0.7, b=1))
    mode = GRAD_ABLATE | nm
    o, W_T, Wc, gn = oracle.forward(inp["q"], inp["k"], inp["v"], inp["eta_logit"],
                                    inp["gate_logit"], inp["W0"], inp["gamma"], inp["beta"],
                                    eps=1e-6, mode=mode, b=1, mask=inp["mask"], want_chunks=True,
                                    want_grad_norms=True)
    assert gn.shape == (1, 2, 20, 2)
    m = inp["mask"][0]
    assert 0 < m.sum() < 20
    for h in range(2):
        for t in range(20):
            if not m[t]:
                np.testing.assert_array_equal(gn[0, h, t], [0.0, 0.0])
                continue
            z = Wc[0, h, t] @ inp["k"][0, h, t]
            n = oracle.lngrad(z, inp["v"][0, h, t], inp["gamma"][h], inp["beta"][h], eps=1e-6,
                              mode=mode, want_norms=True)[3]
            np.testing.assert_allclose(gn[0, h, t], n, rtol=1e-12)
    with pytest.raises(ValueError):
        oracle.forward(inp["q"], inp["k"], inp["v"], inp["eta_logit"], inp["gate_logit"],
                       inp["W0"], inp["gamma"], inp["beta"], eps=1e-6, mode=GRAD_LNJAC, b=1,
                       want_grad_norms=True)


def test_ablation_mode_combinations():
    inp = f64(make_inputs(1, 1, 8, 16, seed=39))
    with pytest.raises(ValueError):
        run(inp, mode=GRAD_ABLATE | NO_LN)
    with pytest.raises(ValueError):
        run(inp, mode=GRAD_NORM_MATCH)
    o, W = run(inp, mode=GRAD_ABLATE | GRAD_NORM_MATCH)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(W))


# ----------------------------------------------------------------------------
# The `:mlp` variant ("Edifice.Recurrent.TTT", `build` options, `:variant`):
# SiLU on the keys and the queries before the inner model.
# ----------------------------------------------------------------------------

def test_kq_silu_known_values():
    """W0 = I, eta = 0, no gate: o_t = SiLU(q_t) exactly; SiLU(1) = e / (1 + e),
    SiLU(-1) = 1 / (1 + e) - 1 ... written from the constants, not the oracle."""
    d, T = 4, 3
    q = np.array([[0.0, 1.0, -1.0, 2.0], [20.0, -20.0, 0.5, -0.5], [3.0, -3.0, 1e-3, -1e-3]])
    k = np.ones((T, d))
    e = np.e
    want = np.array([
        [0.0, e / (1 + e), -1.0 / (1 + e), 2.0 * e * e / (1 + e * e)],
        [20.0 / (1 + np.exp(-20.0)), -20.0 * np.exp(-20.0) / (1 + np.exp(-20.0)),
         0.5 / (1 + np.exp(-0.5)), -0.5 / (1 + np.exp(0.5))],
        [3.0 / (1 + np.exp(-3.0)), -3.0 / (1 + np.exp(3.0)),
         1e-3 / (1 + np.exp(-1e-3)), -1e-3 / (1 + np.exp(1e-3))]])
    sh = lambda a: a.reshape(1, 1, *a.shape)
    o, W_T = oracle.forward(sh(q), sh(k), sh(np.zeros((T, d))), np.full((1, 1, T), -1e4), None,
                            np.eye(d).reshape(1, 1, d, d), np.ones((1, d)), np.zeros((1, d)),
                            eps=1e-6, mode=KQ_SILU | GRAD_LNJAC, b=1)
    np.testing.assert_allclose(o[0, 0], want, rtol=1e-14, atol=1e-300)
    np.testing.assert_array_equal(W_T[0, 0], np.eye(d))


@pytest.mark.parametrize("grad", [0, GRAD_LNJAC, NO_LN], ids=["simple", "lnjac", "no_ln"])
@pytest.mark.parametrize("minib", [0, MINIBATCH], ids=["per_token", "minibatch"])
def test_kq_silu_is_the_linear_scan_on_silu_features(grad, minib):
    """The variant equals the linear scan run on SiLU(k), SiLU(q) computed here
    in numpy (v, the logits and the state untouched), with a mask and a ragged
    tail."""
    inp = f64(make_inputs(2, 3, 37, 16, seed=41, random_affine=True, mask_p=0.6, b=8))
    silu = lambda x: x / (1.0 + np.exp(-x))
    lin = dict(inp, q=silu(inp["q"]), k=silu(inp["k"]))
    o1, W1 = run(inp, mode=grad | minib | KQ_SILU, b=8, eps=1e-6)
    o2, W2 = run(lin, mode=grad | minib, b=8, eps=1e-6)
    np.testing.assert_allclose(o1, o2, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(W1, W2, rtol=1e-11, atol=1e-13)
    o3, _ = run(inp, mode=grad | minib, b=8, eps=1e-6)
    assert not np.allclose(o1, o3)      # the variant does change the result


# ----------------------------------------------------------------------------
# Backward of the per-token scan (no page gives it: reverse mode through the
# forward steps), pinned by central finite differences of the forward oracle.
# ----------------------------------------------------------------------------

def _fd_check_backward(inp, mode, b, eps, seed, tol=1e-7):
    rng = np.random.default_rng(seed)
    keys = ("q", "k", "v", "eta_logit", "gate_logit", "W0", "gamma", "beta")
    x = {k_: (None if inp[k_] is None else np.asarray(inp[k_], np.float64)) for k_ in keys}
    dO = rng.normal(size=x["q"].shape)
    dWT = rng.normal(size=x["W0"].shape)
    m = inp.get("mask")
    g = oracle.backward(**x, dO=dO, dW_T=dWT, eps=eps, mode=mode, b=b, mask=m)

    def loss(xx):
        o, W = oracle.forward(**xx, eps=eps, mode=mode, b=b, mask=m)
        return float((dO * o).sum() + (dWT * W).sum())

    names = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("eta_logit", "deta_logit"),
             ("gate_logit", "dgate_logit"), ("W0", "dW0")]
    if not mode & NO_LN:
        names += [("gamma", "dgamma"), ("beta", "dbeta")]
    for key, gk in names:
        if x[key] is None:
            assert g[gk] is None
            continue
        a = x[key]
        fd = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            h = 1e-6 * max(1.0, abs(a[idx]))
            ap, am = a.copy(), a.copy()
            ap[idx] += h
            am[idx] -= h
            fd[idx] = (loss(dict(x, **{key: ap})) - loss(dict(x, **{key: am}))) / (2 * h)
        scale = np.abs(fd).max() + 1e-12
        assert np.abs(fd - g[gk]).max() <= tol * scale, (key, np.abs(fd - g[gk]).max() / scale)


@pytest.mark.parametrize("grad", [0, GRAD_LNJAC, NO_LN], ids=["simple", "lnjac", "no_ln"])
def test_backward_matches_finite_differences(grad):
    inp = make_inputs(1, 2, 7, 4, seed=45 + grad, random_affine=True, mask_p=0.6, b=2)
    _fd_check_backward(inp, grad, b=2, eps=1e-5, seed=46)


@pytest.mark.parametrize("grad", [0, GRAD_LNJAC, NO_LN], ids=["simple", "lnjac", "no_ln"])
def test_backward_minibatch_matches_finite_differences(grad):
    """Mini-batch mode, b = 3 over T = 8 (ragged tail), with a mask."""
    inp = make_inputs(1, 2, 8, 4, seed=52 + grad, random_affine=True, mask_p=0.6, b=3)
    _fd_check_backward(inp, MINIBATCH | grad, b=3, eps=1e-5, seed=53)


def test_backward_per_feature_gate_and_no_gate():
    inp = make_inputs(1, 1, 5, 4, seed=47, random_affine=True, gate_channel=True)
    _fd_check_backward(inp, GRAD_LNJAC | GATE_CHANNEL, b=16, eps=1e-5, seed=48)
    inp = make_inputs(1, 1, 5, 4, seed=49, random_affine=True, gate=False)
    _fd_check_backward(inp, GRAD_LNJAC, b=16, eps=1e-5, seed=50)


@pytest.mark.parametrize("mode", [GRAD_ABLATE, MINIBATCH | GRAD_ABLATE, KQ_SILU | GRAD_LNJAC,
                                  MINIBATCH | KQ_SILU],
                         ids=["ablate", "ablate_minibatch", "silu_lnjac", "silu_minibatch"])
def test_backward_ablation_and_silu_match_finite_differences(mode):
    inp = make_inputs(1, 2, 6, 4, seed=54 + mode % 97, random_affine=True, mask_p=0.7, b=2)
    _fd_check_backward(inp, mode, b=2, eps=1e-5, seed=55)


def test_backward_rejects_what_it_does_not_take():
    inp = f64(make_inputs(1, 1, 4, 4, seed=51))
    z = np.zeros_like(inp["q"])
    for mode in (GRAD_ABLATE | GRAD_NORM_MATCH, GRAD_ABLATE | NO_LN):
        with pytest.raises(ValueError):
            oracle.backward(inp["q"], inp["k"], inp["v"], inp["eta_logit"], inp["gate_logit"],
                            inp["W0"], inp["gamma"], inp["beta"], z, np.zeros_like(inp["W0"]),
                            eps=1e-5, mode=mode)


# ----------------------------------------------------------------------------
# Mini-batch (dual form; PonderTTT "Technical Architecture").
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("grad", [0, GRAD_LNJAC, NO_LN])
def test_p4_minibatch_b1_equals_per_token(grad):
    inp = f64(make_inputs(2, 2, 33, 16, seed=28, random_affine=True))
    o1, W1 = run(inp, mode=grad, b=1)
    o2, W2 = run(inp, mode=grad | MINIBATCH, b=1)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(W2, W1, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("grad", [0, GRAD_LNJAC])
@pytest.mark.parametrize("b", [4, 7, 16])
def test_minibatch_equals_per_token_for_chunk_orthogonal_keys(grad, b):
    """If the keys of each chunk are mutually orthogonal, W_s k_i = W_{i-1} k_i inside the
    chunk, so the dual form and the per-token recurrence coincide (any b, ragged tail)."""
    d, T = 16, 3 * b + (b // 2 + 1)
    rng = np.random.default_rng(29 + b)
    K = np.empty((T, d))
    for c0 in range(0, T, b):
        n = min(b, T - c0)
        basis, _ = np.linalg.qr(rng.normal(size=(d, d)))
        K[c0:c0 + n] = basis[:n] * rng.uniform(2.0, 6.0, size=(n, 1))
    inp = f64(make_inputs(1, 1, T, d, seed=30, random_affine=True))
    inp["k"] = K[None, None]
    o1, W1 = run(inp, mode=grad, b=b)
    o2, W2 = run(inp, mode=grad | MINIBATCH, b=b)
    np.testing.assert_allclose(o2, o1, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(W2, W1, rtol=1e-11, atol=1e-12)
    # generic keys do differ between the two modes
    inp3 = f64(make_inputs(1, 1, T, d, seed=30, random_affine=True))
    o3, _ = run(inp3, mode=grad, b=b)
    o4, _ = run(inp3, mode=grad | MINIBATCH, b=b)
    assert np.abs(o3 - o4).max() > 1e-6


def test_p10_minibatch_single_chunk_vectorised():
    """b = T: every z_i uses W0; O = sig(g) (Q W0^T - (tril(Q K^T) eta) G); W_T = W0 - G^T diag(eta) K."""
    d, T = 16, 24
    inp = f64(make_inputs(1, 1, T, d, seed=31, random_affine=True))
    Q, K, V = inp["q"][0, 0], inp["k"][0, 0], inp["v"][0, 0]
    W0, gam, bet = inp["W0"][0, 0], inp["gamma"][0], inp["beta"][0]
    eta = sig(inp["eta_logit"][0, 0]) / d
    gate = sig(inp["gate_logit"][0, 0])
    Z = K @ W0.T
    G = np.stack([oracle.lngrad(Z[i], V[i], gam, bet, eps=1e-5, mode=GRAD_LNJAC)[1] for i in range(T)])
    O = gate[:, None] * (Q @ W0.T - (np.tril(Q @ K.T) * eta[None, :]) @ G)
    WT = W0 - G.T @ (eta[:, None] * K)
    o, W_T = run(inp, mode=MINIBATCH | GRAD_LNJAC, b=T)
    np.testing.assert_allclose(o[0, 0], O, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(W_T[0, 0], WT, rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------
# Chaining: W_T is the resumable state.
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [0, GRAD_LNJAC, MINIBATCH | GRAD_LNJAC])
def test_p9_chaining(mode):
    B, H, d, b = 2, 2, 16, 8
    T1, T2 = 24, 21
    inp = f64(make_inputs(B, H, T1 + T2, d, seed=32, random_affine=True, mask_p=0.6, b=b))
    o, W_T = run(inp, mode=mode, b=b)
    sl = lambda a, s: None if a is None else a[:, :, s]
    n1 = T1 // b
    first = dict(inp, q=sl(inp["q"], slice(0, T1)), k=sl(inp["k"], slice(0, T1)),
                 v=sl(inp["v"], slice(0, T1)), eta_logit=sl(inp["eta_logit"], slice(0, T1)),
                 gate_logit=sl(inp["gate_logit"], slice(0, T1)), mask=inp["mask"][:, :n1])
    oa, Wa = run(first, mode=mode, b=b)
    second = dict(inp, q=sl(inp["q"], slice(T1, None)), k=sl(inp["k"], slice(T1, None)),
                  v=sl(inp["v"], slice(T1, None)), eta_logit=sl(inp["eta_logit"], slice(T1, None)),
                  gate_logit=sl(inp["gate_logit"], slice(T1, None)), W0=Wa,
                  mask=inp["mask"][:, n1:])
    ob, Wb = run(second, mode=mode, b=b)
    np.testing.assert_array_equal(np.concatenate([oa, ob], axis=2), o)
    np.testing.assert_array_equal(Wb, W_T)


def test_no_gate_means_unit_gate():
    inp = f64(make_inputs(1, 2, 10, 16, seed=33))
    o1, W1 = run(inp, mode=GRAD_LNJAC)
    inp2 = dict(inp, gate_logit=None)
    o2, W2 = run(inp2, mode=GRAD_LNJAC)
    np.testing.assert_array_equal(W1, W2)
    np.testing.assert_allclose(o1, sig(inp["gate_logit"])[..., None] * o2, rtol=1e-14)


# ----------------------------------------------------------------------------
# Per-channel output gate: the elementwise reading of the sigmoid output gate
# ("Edifice.Recurrent.TTT", "Paper-Faithful Implementation", item 4).
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [GRAD_LNJAC, MINIBATCH | GRAD_LNJAC, 0])
def test_gate_channel_is_elementwise_and_leaves_W_alone(mode):
    B, H, T, d = 2, 3, 21, 16
    inp = f64(make_inputs(B, H, T, d, seed=35, random_affine=True, gate_channel=True))
    assert inp["gate_logit"].shape == (B, H, T, d)
    o_g, W_g = run(inp, mode=mode | GATE_CHANNEL, b=8)
    o_n, W_n = run(dict(inp, gate_logit=None), mode=mode | GATE_CHANNEL, b=8)
    np.testing.assert_array_equal(W_g, W_n)
    np.testing.assert_allclose(o_g, sig(inp["gate_logit"]) * o_n, rtol=1e-14, atol=1e-300)


@pytest.mark.parametrize("mode", [GRAD_LNJAC, MINIBATCH])
def test_gate_channel_constant_over_features_equals_scalar_gate(mode):
    B, H, T, d = 2, 2, 13, 16
    inp = f64(make_inputs(B, H, T, d, seed=36, random_affine=True))
    o_s, W_s = run(inp, mode=mode, b=4)
    wide = np.repeat(inp["gate_logit"][..., None], d, axis=-1)
    o_c, W_c = run(dict(inp, gate_logit=wide), mode=mode | GATE_CHANNEL, b=4)
    np.testing.assert_array_equal(o_c, o_s)
    np.testing.assert_array_equal(W_c, W_s)


def test_gate_shape_must_match_mode():
    inp = f64(make_inputs(1, 1, 4, 16, seed=37))
    with pytest.raises(ValueError):
        run(inp, mode=GATE_CHANNEL)


# ----------------------------------------------------------------------------
# Streaming decode: one token at a time, W carried between calls.
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [0, GRAD_LNJAC, NO_LN, GRAD_LNJAC | GATE_CHANNEL])
def test_decode_steps_chain_to_the_per_token_scan(mode):
    B, H, T, d = 2, 3, 9, 16
    inp = f64(make_inputs(B, H, T, d, seed=38, random_affine=True, mask_p=0.6, b=1,
                          gate_channel=bool(mode & GATE_CHANNEL)))
    o_ref, W_ref = run(inp, mode=mode, b=1)
    W = inp["W0"]
    for t in range(T):
        o_t, W = oracle.decode_step(inp["q"][:, :, t], inp["k"][:, :, t], inp["v"][:, :, t],
                                    inp["eta_logit"][:, :, t], inp["gate_logit"][:, :, t],
                                    W, inp["gamma"], inp["beta"], eps=1e-5, mode=mode,
                                    update=inp["mask"][:, t])
        np.testing.assert_array_equal(o_t, o_ref[:, :, t])
    np.testing.assert_array_equal(W, W_ref)
    with pytest.raises(ValueError):
        oracle.decode_step(inp["q"][:, :, 0], inp["k"][:, :, 0], inp["v"][:, :, 0],
                           inp["eta_logit"][:, :, 0], None, W, inp["gamma"], inp["beta"],
                           eps=1e-5, mode=MINIBATCH)


def test_float_twin_close_to_double():
    inp = make_inputs(1, 1, 64, 16, seed=1)
    o64, W64 = run(f64(inp), mode=0)
    o32, W32 = oracle.forward(inp["q"], inp["k"], inp["v"], inp["eta_logit"], inp["gate_logit"],
                              inp["W0"], inp["gamma"], inp["beta"], eps=1e-5, mode=0, b=16,
                              dtype=np.float32)
    assert o32.dtype == np.float32
    assert np.abs(o32 - o64).max() <= 1e-4 * (1 + np.abs(o64).max())


def test_oracle_rejects_bad_arguments():
    inp = f64(make_inputs(1, 1, 8, 16, seed=34))
    with pytest.raises(ValueError):
        run(inp, mode=0, b=0)
