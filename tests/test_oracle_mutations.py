"""The oracle's pins must catch plausible slips.

Each case below plants one mistake in a temporary copy of the oracle source
(on the CPU, never in the CUDA path), builds it, and runs the pin suite
against that build in a child process. Every mutant must make at least one pin
fail; the unmodified source must pass.
"""

import os
import subprocess
import sys
import tempfile
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
SRC = ROOT / "oracle" / "ttt_oracle.cpp"

# (name, text in the oracle source, replacement)
MUTATIONS = [
    ("update_sign", "W[r * d + cc] -= eta * G[r] * kt[cc];", "W[r * d + cc] += eta * G[r] * kt[cc];"),
    ("update_transposed", "W[r * d + cc] -= eta * G[r] * kt[cc];", "W[r * d + cc] -= eta * G[cc] * kt[r];"),
    ("eta_without_1_over_d", "const S eta = update ? sigmoid(eta_logit[t]) / S(d) : S(0);",
     "const S eta = update ? sigmoid(eta_logit[t]) : S(0);"),
    ("output_before_update",
     "for (int r = 0; r < d; ++r)\n          for (int cc = 0; cc < d; ++cc) W[r * d + cc] -= eta * G[r] * kt[cc];\n"
     "        matvec(W.data(), qt, d, Wq.data());",
     "matvec(W.data(), qt, d, Wq.data());\n        for (int r = 0; r < d; ++r)\n"
     "          for (int cc = 0; cc < d; ++cc) W[r * d + cc] -= eta * G[r] * kt[cc];"),
    ("lnjac_drop_mean_g", "out[f] = (g[f] - mean_g - xhat[f] * mean_gx) / s;", "out[f] = (g[f] - xhat[f] * mean_gx) / s;"),
    ("lnjac_drop_xhat_term", "out[f] = (g[f] - mean_g - xhat[f] * mean_gx) / s;", "out[f] = (g[f] - mean_g) / s;"),
    ("lnjac_drop_gamma", "g[f] = gamma[f] * (pred[f] - v[f]);", "g[f] = (pred[f] - v[f]);"),
    ("lnjac_no_1_over_s", "out[f] = (g[f] - mean_g - xhat[f] * mean_gx) / s;", "out[f] = (g[f] - mean_g - xhat[f] * mean_gx);"),
    ("eps_outside_sqrt", "const S s = std::sqrt(var + eps);", "const S s = std::sqrt(var) + eps;"),
    ("unbiased_variance", "var /= S(d);", "var /= S(d - 1);"),
    ("drop_beta", "pred[f] = gamma[f] * xhat[f] + beta[f];", "pred[f] = gamma[f] * xhat[f];"),
    ("ablation_keeps_beta", "for (int f = 0; f < d; ++f) g[f] = gamma[f] * (-v[f]);",
     "for (int f = 0; f < d; ++f) g[f] = gamma[f] * (beta[f] - v[f]);"),
    ("ablation_without_jacobian", "        jacobian_t(g, G);\n        S n_full = 0, n_abl = 0;",
     "        for (int f = 0; f < d; ++f) G[f] = g[f];\n        S n_full = 0, n_abl = 0;"),
    ("norm_match_without_sqrt", "std::sqrt(n_full / n_abl)", "(n_full / n_abl)"),
    ("grad_norms_both_full", "norms[1] = std::sqrt(n_abl);", "norms[1] = std::sqrt(n_full);"),
    ("grad_norms_squared", "norms[0] = std::sqrt(n_full);", "norms[0] = n_full;"),
    ("kq_silu_keys_only", "      qs[i] = silu(q[i]);", "      qs[i] = q[i];"),
    ("kq_silu_as_sigmoid", "  return x * sigmoid(x);", "  return sigmoid(x);"),
    ("backward_drops_explicit_1_over_s", "      ds -= dG[f] * G[f] / s;", "      ds -= 0 * G[f];"),
    ("backward_dk_without_update_term", "      dk[(size_t)t * d + c] = -eta * acc;",
     "      dk[(size_t)t * d + c] = 0;"),
    ("backward_minibatch_without_readout_terms", "const S dyG = dot(dy.data(), Gj, d);",
     "const S dyG = 0;"),
    ("scalar_gate_ignored", "  return sigmoid(gate_logit[t]);", "  return S(1);"),
    ("gate_channel_wrong_feature", "sigmoid(gate_logit[(size_t)t * d + r])",
     "sigmoid(gate_logit[(size_t)t * d + (d - 1 - r)])"),
    ("gate_channel_read_as_scalar", "if (mode & kGateChannel) return sigmoid(gate_logit[(size_t)t * d + r]);",
     "if (mode & kGateChannel) return sigmoid(gate_logit[t]);"),
    ("gate_channel_wrong_head_offset", "gate_logit + ((mode & kGateChannel) ? tok * d : tok)",
     "gate_logit + tok"),
    ("minibatch_exclusive_prefix", "for (int j = 0; j <= i; ++j) {", "for (int j = 0; j < i; ++j) {"),
    ("minibatch_wrong_key_index", "const S a = etas[j] * dot(k + (size_t)(t0 + j) * d, qt, d);",
     "const S a = etas[j] * dot(k + (size_t)(t0 + i) * d, qt, d);"),
    ("mask_ignored", "(mask_row == nullptr) || (mask_row[c] != 0)", "true"),
    ("tail_chunk_dropped", "const int n_chunks = (T + b - 1) / b;\n  std::vector<S> W(",
     "const int n_chunks = T / b;\n  std::vector<S> W("),
    ("minibatch_update_uses_q", "const S* kj = k + (size_t)(t0 + j) * d;", "const S* kj = q + (size_t)(t0 + j) * d;"),
]


def _build(src_text, out):
    with tempfile.NamedTemporaryFile("w", suffix=".cpp", delete=False) as f:
        f.write(src_text)
        path = f.name
    try:
        subprocess.run(["g++", "-O1", "-std=c++17", "-fopenmp", "-fPIC", "-shared",
                        "-ffp-contract=off", path, "-o", out], check=True)
    finally:
        os.unlink(path)


def _run_pins(lib):
    env = dict(os.environ, TTT_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        str(ROOT / "tests" / "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_mutation(name, old, new, tmp_path):
    text = SRC.read_text()
    assert text.count(old) >= 1, f"mutation {name}: anchor text not found in the oracle"
    mutated = text.replace(old, new, 1)
    lib = str(tmp_path / f"lib_{name}.so")
    _build(mutated, lib)
    assert _run_pins(lib) != 0, f"no pin failed for the planted slip '{name}'"


def test_unmutated_oracle_passes_pins(tmp_path):
    lib = str(tmp_path / "lib_clean.so")
    _build(SRC.read_text(), lib)
    assert _run_pins(lib) == 0
