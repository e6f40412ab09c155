// TTT-Linear inner-loop scan: plain CPU oracle.
//
// TEST INFRASTRUCTURE ONLY. This file is the slow, obviously-correct reference
// that the CUDA path is checked against. Only the tests, the smoke check and the
// benchmark's CPU-baseline leg load it; the product path never does. It shares
// no code, header, table or constant with the CUDA sources.
//
// What it computes, per (batch row, head), in the order the pages give it
// ("Edifice.Recurrent.TTT", section "Equations (TTT-Linear)" and the inner loop
// drawn in section "Architecture"):
//
//     eta_t  = sigmoid(eta_logit_t) / d
//     z_t    = W_{t-1} k_t
//     pred_t = LayerNorm_{gamma,beta}(z_t)
//     err_t  = pred_t - v_t
//     W_t    = W_{t-1} - eta_t * G_t k_t^T
//     o_t    = (W_t q_t) * sigmoid(gate_t)
//
// with the inner gradient G_t (d loss / d z_t, loss = 1/2 ||pred_t - v_t||^2) either
//   * the simplified form of the Equations section:        G_t = err_t, or
//   * the full squared-error gradient through the LayerNorm Jacobian
//     ("Error Correction in Trained TTT Layers", Abstract):
//        g = gamma * err,  G = (g - mean(g) - xhat * mean(g * xhat)) / s.
//
// Mini-batch ("dual-form updates", PonderTTT, section "Technical Architecture"):
// every token of a chunk of b tokens takes its gradient at the chunk-start W_s,
//     o_i = sigmoid(gate_i) * (W_s q_i - sum_{j <= i} eta_j (k_j . q_i) G_j)
//     W   = W_s - sum_j eta_j G_j k_j^T .
// The last chunk may be shorter than b (cortex_rust src/layers/ttt.rs,
// forward_chunkwise: the chunk count is a ceiling division and the last chunk
// takes what is left).
//
// SKIP/UPDATE mask (PonderTTT, section "Core Idea: Binary Gating via
// Gumbel-Softmax"): one byte per chunk of b tokens and per batch row; 0 = SKIP
// sets eta = 0 for every token of that chunk, so W does not change there while
// outputs are still produced.
//
// Readings where the pages are silent:
//   * LayerNorm normalises over the d features of one head, biased variance,
//     eps inside the square root: s = sqrt(mean((z - mu)^2) + eps).
//   * W is stored row-major as W[out][in] so that z = W k.
//   * gate_logit == NULL means no output gate (sigmoid replaced by 1).
//   * The gate is one scalar per token by default. With the per-channel gate
//     option it is a d-vector per token, o_t[r] = sigmoid(gate_t[r]) (W_t q_t)[r]:
//     the elementwise reading of "Sigmoid gate on output (like SwiGLU)"
//     ("Edifice.Recurrent.TTT", section "Paper-Faithful Implementation", item 4).
//   * mask == NULL means every chunk updates.
//   * NO_LN removes the LayerNorm: pred = z and G = z - v (the delta rule of the
//     section "Key Innovations").
//   * The ablation gradient ("Error Correction in Trained TTT Layers", Abstract:
//     the full normalised prediction's contribution removed, the LayerNorm
//     Jacobian retained) is the Jacobian form with the whole prediction
//     gamma * xhat + beta dropped from the error: g = -gamma * v. With per-token
//     norm matching it is rescaled to the L2 norm of the full Jacobian-form
//     gradient of the same token (and is 0 where its own norm is 0).
//
// Arithmetic runs in the template scalar type: double is the oracle; the float
// instantiation exists only to measure how much plain fp32 rounding alone moves
// the result (the conditioning floor of the recurrence).

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// Oracle-local mode bits. Their numeric values follow the public interface of
// the scan so a caller can pass the same integer.
constexpr unsigned kMiniBatch = 1u << 0;
constexpr unsigned kLnJacobian = 1u << 1;
constexpr unsigned kNoLayerNorm = 1u << 2;
constexpr unsigned kGateChannel = 1u << 6;
constexpr unsigned kGradAblate = 1u << 8;
constexpr unsigned kNormMatch = 1u << 9;
// The `:mlp` variant ("Edifice.Recurrent.TTT", `build` options, `:variant`):
// SiLU applied to the keys and the queries before the inner model. Oracle
// only for now; the bit is reserved for the scan's interface.
constexpr unsigned kKqSilu = 1u << 10;

template <typename S>
S sigmoid(S x) {
  return S(1) / (S(1) + std::exp(-x));
}

// SiLU(x) = x * sigmoid(x).
template <typename S>
S silu(S x) {
  return x * sigmoid(x);
}

// Inner LayerNorm forward and the inner gradient with respect to z.
// Writes pred (may be null), G, and xhat (may be null). With the ablation
// gradient, norms (may be null) receives the L2 norms of the full
// Jacobian-form gradient and of the ablated gradient before any norm matching
// (their ratio is the gradient norm ratio of "Error Correction in Trained TTT
// Layers", Abstract).
template <typename S>
void ln_and_grad(const S* z, const S* v, const S* gamma, const S* beta, int d,
                 S eps, unsigned mode, S* pred_out, S* G, S* xhat_out, S* norms = nullptr) {
  std::vector<S> pred(d), xhat(d);
  if (mode & kNoLayerNorm) {
    for (int f = 0; f < d; ++f) {
      pred[f] = z[f];
      xhat[f] = z[f];
      G[f] = z[f] - v[f];
    }
  } else {
    S mu = 0;
    for (int f = 0; f < d; ++f) mu += z[f];
    mu /= S(d);
    S var = 0;
    for (int f = 0; f < d; ++f) var += (z[f] - mu) * (z[f] - mu);
    var /= S(d);
    const S s = std::sqrt(var + eps);
    for (int f = 0; f < d; ++f) {
      xhat[f] = (z[f] - mu) / s;
      pred[f] = gamma[f] * xhat[f] + beta[f];
    }
    if (mode & (kLnJacobian | kGradAblate)) {
      // back through the LayerNorm: G = J^T g with g the gradient at its output
      auto jacobian_t = [&](const std::vector<S>& g, S* out) {
        S mean_g = 0, mean_gx = 0;
        for (int f = 0; f < d; ++f) {
          mean_g += g[f];
          mean_gx += g[f] * xhat[f];
        }
        mean_g /= S(d);
        mean_gx /= S(d);
        for (int f = 0; f < d; ++f) out[f] = (g[f] - mean_g - xhat[f] * mean_gx) / s;
      };
      std::vector<S> g(d), full(d);
      for (int f = 0; f < d; ++f) g[f] = gamma[f] * (pred[f] - v[f]);
      jacobian_t(g, full.data());
      if (mode & kGradAblate) {
        for (int f = 0; f < d; ++f) g[f] = gamma[f] * (-v[f]);
        jacobian_t(g, G);
        S n_full = 0, n_abl = 0;
        for (int f = 0; f < d; ++f) {
          n_full += full[f] * full[f];
          n_abl += G[f] * G[f];
        }
        if (norms) {
          norms[0] = std::sqrt(n_full);
          norms[1] = std::sqrt(n_abl);
        }
        if (mode & kNormMatch) {
          const S scale = n_abl > S(0) ? std::sqrt(n_full / n_abl) : S(0);
          for (int f = 0; f < d; ++f) G[f] *= scale;
        }
      } else {
        for (int f = 0; f < d; ++f) G[f] = full[f];
      }
    } else {
      for (int f = 0; f < d; ++f) G[f] = pred[f] - v[f];
    }
  }
  if (pred_out)
    for (int f = 0; f < d; ++f) pred_out[f] = pred[f];
  if (xhat_out)
    for (int f = 0; f < d; ++f) xhat_out[f] = xhat[f];
}

// y = M x for a d x d row-major M.
template <typename S>
void matvec(const S* M, const S* x, int d, S* y) {
  for (int r = 0; r < d; ++r) {
    S acc = 0;
    for (int c = 0; c < d; ++c) acc += M[r * d + c] * x[c];
    y[r] = acc;
  }
}

template <typename S>
S dot(const S* a, const S* b, int d) {
  S acc = 0;
  for (int f = 0; f < d; ++f) acc += a[f] * b[f];
  return acc;
}

// Output gate of feature r of token t: scalar per token, or one per feature.
template <typename S>
S gate_of(const S* gate_logit, unsigned mode, int t, int d, int r) {
  if (!gate_logit) return S(1);
  if (mode & kGateChannel) return sigmoid(gate_logit[(size_t)t * d + r]);
  return sigmoid(gate_logit[t]);
}

// One (batch row, head) recurrence over all T tokens.
template <typename S>
void scan_one_head(const S* q, const S* k, const S* v, const S* eta_logit,
                   const S* gate_logit, const S* W0, const S* gamma,
                   const S* beta, int T, int d, S eps, unsigned mode, int b,
                   const unsigned char* mask_row, S* o, S* W_T, S* W_chunks,
                   S* gnorms) {
  const int n_chunks = (T + b - 1) / b;
  std::vector<S> W(W0, W0 + (size_t)d * d);
  std::vector<S> z(d), G(d), Wq(d);
  // the `:mlp` variant feeds SiLU(k), SiLU(q) to the inner model
  std::vector<S> ks, qs;
  if (mode & kKqSilu) {
    ks.resize((size_t)T * d);
    qs.resize((size_t)T * d);
    for (size_t i = 0; i < (size_t)T * d; ++i) {
      ks[i] = silu(k[i]);
      qs[i] = silu(q[i]);
    }
    k = ks.data();
    q = qs.data();
  }

  for (int c = 0; c < n_chunks; ++c) {
    const int t0 = c * b;
    const int t1 = (t0 + b < T) ? t0 + b : T;
    const bool update = (mask_row == nullptr) || (mask_row[c] != 0);
    if (W_chunks) std::memcpy(W_chunks + (size_t)c * d * d, W.data(), sizeof(S) * d * d);

    if (!(mode & kMiniBatch)) {
      // Exact per-token recurrence.
      for (int t = t0; t < t1; ++t) {
        const S* kt = k + (size_t)t * d;
        const S* qt = q + (size_t)t * d;
        const S* vt = v + (size_t)t * d;
        const S eta = update ? sigmoid(eta_logit[t]) / S(d) : S(0);
        matvec(W.data(), kt, d, z.data());
        ln_and_grad(z.data(), vt, gamma, beta, d, eps, mode, (S*)nullptr,
                    G.data(), (S*)nullptr, gnorms ? gnorms + (size_t)t * 2 : (S*)nullptr);
        // a SKIP chunk takes no gradient: its tokens report zero norms
        if (gnorms && !update) gnorms[(size_t)t * 2] = gnorms[(size_t)t * 2 + 1] = S(0);
        for (int r = 0; r < d; ++r)
          for (int cc = 0; cc < d; ++cc) W[r * d + cc] -= eta * G[r] * kt[cc];
        matvec(W.data(), qt, d, Wq.data());
        for (int r = 0; r < d; ++r)
          o[(size_t)t * d + r] = gate_of(gate_logit, mode, t, d, r) * Wq[r];
      }
    } else {
      // Mini-batch (dual form): all gradients of the chunk at W_s.
      const int n = t1 - t0;
      std::vector<S> Gs((size_t)n * d), etas(n);
      for (int i = 0; i < n; ++i) {
        const int t = t0 + i;
        etas[i] = update ? sigmoid(eta_logit[t]) / S(d) : S(0);
        matvec(W.data(), k + (size_t)t * d, d, z.data());
        ln_and_grad(z.data(), v + (size_t)t * d, gamma, beta, d, eps, mode,
                    (S*)nullptr, Gs.data() + (size_t)i * d, (S*)nullptr,
                    gnorms ? gnorms + (size_t)t * 2 : (S*)nullptr);
        if (gnorms && !update) gnorms[(size_t)t * 2] = gnorms[(size_t)t * 2 + 1] = S(0);
      }
      for (int i = 0; i < n; ++i) {
        const int t = t0 + i;
        const S* qt = q + (size_t)t * d;
        matvec(W.data(), qt, d, Wq.data());
        for (int j = 0; j <= i; ++j) {
          const S a = etas[j] * dot(k + (size_t)(t0 + j) * d, qt, d);
          for (int r = 0; r < d; ++r) Wq[r] -= a * Gs[(size_t)j * d + r];
        }
        for (int r = 0; r < d; ++r)
          o[(size_t)t * d + r] = gate_of(gate_logit, mode, t, d, r) * Wq[r];
      }
      for (int j = 0; j < n; ++j) {
        const S* kj = k + (size_t)(t0 + j) * d;
        for (int r = 0; r < d; ++r)
          for (int cc = 0; cc < d; ++cc)
            W[r * d + cc] -= etas[j] * Gs[(size_t)j * d + r] * kj[cc];
      }
    }
  }
  if (W_chunks)
    std::memcpy(W_chunks + (size_t)n_chunks * d * d, W.data(), sizeof(S) * d * d);
  std::memcpy(W_T, W.data(), sizeof(S) * d * d);
}

template <typename S>
int forward(const S* q, const S* k, const S* v, const S* eta_logit,
            const S* gate_logit, const S* W0, const S* gamma, const S* beta,
            int B, int H, int T, int d, S eps, unsigned mode, int b,
            const unsigned char* mask, S* o, S* W_T, S* W_chunks, S* grad_norms,
            int nthreads) {
  if (B < 0 || H < 0 || T < 0 || d <= 0 || b <= 0) return -1;
  if (grad_norms && !(mode & kGradAblate)) return -1;
  if ((mode & kGradAblate) && (mode & kNoLayerNorm)) return -1;
  if ((mode & kNormMatch) && !(mode & kGradAblate)) return -1;
  if (!q || !k || !v || !eta_logit || !W0 || !o || !W_T) return -1;
  if (!(mode & kNoLayerNorm) && (!gamma || !beta)) return -1;
  const int n_chunks = (T + b - 1) / b;
  const long long heads = (long long)B * H;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (long long bh = 0; bh < heads; ++bh) {
    const int bi = (int)(bh / H);
    const int h = (int)(bh % H);
    const size_t tok = (size_t)bh * T;
    scan_one_head<S>(q + tok * d, k + tok * d, v + tok * d, eta_logit + tok,
                     gate_logit ? gate_logit + ((mode & kGateChannel) ? tok * d : tok)
                                : nullptr,
                     W0 + (size_t)bh * d * d,
                     gamma ? gamma + (size_t)h * d : nullptr,
                     beta ? beta + (size_t)h * d : nullptr, T, d, eps, mode, b,
                     mask ? mask + (size_t)bi * n_chunks : nullptr,
                     o + tok * d, W_T + (size_t)bh * d * d,
                     W_chunks ? W_chunks + (size_t)bh * (n_chunks + 1) * d * d
                              : nullptr,
                     grad_norms ? grad_norms + tok * 2 : nullptr);
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Backward of the per-token recurrence (reverse mode through every token).
// No page gives this; it is the chain rule applied, in reverse order, to the
// forward steps above: z = W k, the LayerNorm and its gradient G, the update
// W' = W - eta G k^T, the output o = gate * (W' q). Given dO (= dL/do) and
// dW_T (= dL/dW_T) it returns dL/d of every input.
// ---------------------------------------------------------------------------

// dz, and the contributions to dv, dgamma, dbeta, of dG through G(z, v).
template <typename S>
void lngrad_backward(const S* z, const S* v, const S* gamma, const S* beta, int d, S eps,
                     unsigned mode, const S* dG, S* dz, S* dv, S* dgamma, S* dbeta) {
  if (mode & kNoLayerNorm) {  // G = z - v
    for (int f = 0; f < d; ++f) {
      dz[f] = dG[f];
      dv[f] -= dG[f];
    }
    return;
  }
  S mu = 0;
  for (int f = 0; f < d; ++f) mu += z[f];
  mu /= S(d);
  S var = 0;
  for (int f = 0; f < d; ++f) var += (z[f] - mu) * (z[f] - mu);
  var /= S(d);
  const S s = std::sqrt(var + eps);
  std::vector<S> xhat(d), err(d), dxhat(d, S(0));
  for (int f = 0; f < d; ++f) {
    xhat[f] = (z[f] - mu) / s;
    err[f] = gamma[f] * xhat[f] + beta[f] - v[f];
  }
  S ds = 0;  // dL/ds through G's explicit 1/s (the Jacobian forms only)
  std::vector<S> derr(d, S(0));
  const bool ablate = mode & kGradAblate;
  if (mode & (kLnJacobian | kGradAblate)) {
    // G = (g - mean g - xhat mean(g xhat)) / s, g = gamma err (ablation:
    // g = -gamma v, which does not depend on z)
    std::vector<S> g(d), G(d);
    S a = 0, c = 0, mdG = 0, mdGx = 0;
    for (int f = 0; f < d; ++f) {
      g[f] = ablate ? -gamma[f] * v[f] : gamma[f] * err[f];
      a += g[f];
      c += g[f] * xhat[f];
      mdG += dG[f];
      mdGx += dG[f] * xhat[f];
    }
    a /= S(d);
    c /= S(d);
    mdG /= S(d);
    mdGx /= S(d);
    for (int f = 0; f < d; ++f) G[f] = (g[f] - a - xhat[f] * c) / s;
    for (int f = 0; f < d; ++f) {
      const S dg = (dG[f] - mdG - xhat[f] * mdGx) / s;       // J^T is symmetric
      dxhat[f] += (-dG[f] * c - g[f] * mdGx) / s;
      ds -= dG[f] * G[f] / s;
      if (ablate) {
        dgamma[f] -= dg * v[f];
        dv[f] -= dg * gamma[f];
      } else {
        dgamma[f] += dg * err[f];
        derr[f] = dg * gamma[f];
      }
    }
  } else {  // G = err
    for (int f = 0; f < d; ++f) derr[f] = dG[f];
  }
  // err = gamma xhat + beta - v
  for (int f = 0; f < d; ++f) {
    dgamma[f] += derr[f] * xhat[f];
    dbeta[f] += derr[f];
    dv[f] -= derr[f];
    dxhat[f] += derr[f] * gamma[f];
  }
  // xhat = (z - mu) / s, s = sqrt(var + eps), var = mean((z - mu)^2)
  S dxx = 0;
  for (int f = 0; f < d; ++f) dxx += dxhat[f] * xhat[f];
  const S ds_total = ds - dxx / s;
  const S dvar = ds_total / (S(2) * s);
  std::vector<S> dy(d);
  S mdy = 0;
  for (int f = 0; f < d; ++f) {
    dy[f] = dxhat[f] / s + dvar * S(2) * (z[f] - mu) / S(d);
    mdy += dy[f];
  }
  mdy /= S(d);
  for (int f = 0; f < d; ++f) dz[f] = dy[f] - mdy;
}

template <typename S>
void backward_one_head(const S* q, const S* k, const S* v, const S* eta_logit,
                       const S* gate_logit, const S* W0, const S* gamma, const S* beta,
                       int T, int d, S eps, unsigned mode, int b,
                       const unsigned char* mask_row, const S* dO, const S* dW_T,
                       S* dq, S* dk, S* dv, S* deta, S* dgate, S* dW0, S* dgamma,
                       S* dbeta) {
  // forward, keeping the state before every token
  std::vector<S> Ws((size_t)(T + 1) * d * d);
  std::memcpy(Ws.data(), W0, sizeof(S) * d * d);
  std::vector<S> z(d), G(d), y(d), dz(d), dG(d), dy(d), dWk(d);
  auto upd_of = [&](int t) { return (mask_row == nullptr) || (mask_row[t / b] != 0); };
  for (int t = 0; t < T; ++t) {
    const S* W = Ws.data() + (size_t)t * d * d;
    S* Wn = Ws.data() + (size_t)(t + 1) * d * d;
    const S* kt = k + (size_t)t * d;
    const S eta = upd_of(t) ? sigmoid(eta_logit[t]) / S(d) : S(0);
    matvec(W, kt, d, z.data());
    ln_and_grad(z.data(), v + (size_t)t * d, gamma, beta, d, eps, mode, (S*)nullptr,
                G.data(), (S*)nullptr);
    for (int r = 0; r < d; ++r)
      for (int c = 0; c < d; ++c) Wn[r * d + c] = W[r * d + c] - eta * G[r] * kt[c];
  }
  // reverse: dW holds dL/dW_t, starting from dL/dW_T
  std::vector<S> dW(dW_T, dW_T + (size_t)d * d);
  for (int t = T - 1; t >= 0; --t) {
    const S* W = Ws.data() + (size_t)t * d * d;       // W_{t-1}
    const S* Wn = Ws.data() + (size_t)(t + 1) * d * d; // W_t
    const S* kt = k + (size_t)t * d;
    const S* qt = q + (size_t)t * d;
    const S* dOt = dO + (size_t)t * d;
    const bool upd = upd_of(t);
    const S sg = upd ? sigmoid(eta_logit[t]) : S(0);
    const S eta = sg / S(d);
    // o = gate * (W_t q)
    matvec(Wn, qt, d, y.data());
    if (gate_logit && (mode & kGateChannel)) {
      for (int r = 0; r < d; ++r) {
        const S g = sigmoid(gate_logit[(size_t)t * d + r]);
        dy[r] = g * dOt[r];
        dgate[(size_t)t * d + r] = dOt[r] * y[r] * g * (S(1) - g);
      }
    } else if (gate_logit) {
      const S g = sigmoid(gate_logit[t]);
      S acc = 0;
      for (int r = 0; r < d; ++r) {
        dy[r] = g * dOt[r];
        acc += dOt[r] * y[r];
      }
      dgate[t] = acc * g * (S(1) - g);
    } else {
      for (int r = 0; r < d; ++r) dy[r] = dOt[r];
    }
    for (int c = 0; c < d; ++c) {
      S acc = 0;
      for (int r = 0; r < d; ++r) acc += Wn[r * d + c] * dy[r];
      dq[(size_t)t * d + c] = acc;
    }
    for (int r = 0; r < d; ++r)
      for (int c = 0; c < d; ++c) dW[r * d + c] += dy[r] * qt[c];
    // W_t = W_{t-1} - eta G k^T, G = G(z = W_{t-1} k)
    matvec(W, kt, d, z.data());
    ln_and_grad(z.data(), v + (size_t)t * d, gamma, beta, d, eps, mode, (S*)nullptr,
                G.data(), (S*)nullptr);
    matvec(dW.data(), kt, d, dWk.data());               // dW k
    S deta_t = 0;
    for (int r = 0; r < d; ++r) {
      deta_t -= G[r] * dWk[r];
      dG[r] = -eta * dWk[r];
    }
    for (int c = 0; c < d; ++c) {
      S acc = 0;
      for (int r = 0; r < d; ++r) acc += dW[r * d + c] * G[r];
      dk[(size_t)t * d + c] = -eta * acc;
    }
    deta[t] = upd ? deta_t * sg * (S(1) - sg) / S(d) : S(0);
    lngrad_backward(z.data(), v + (size_t)t * d, gamma, beta, d, eps, mode, dG.data(),
                    dz.data(), dv + (size_t)t * d, dgamma, dbeta);
    // z = W_{t-1} k
    for (int c = 0; c < d; ++c) {
      S acc = 0;
      for (int r = 0; r < d; ++r) acc += W[r * d + c] * dz[r];
      dk[(size_t)t * d + c] += acc;
    }
    for (int r = 0; r < d; ++r)
      for (int c = 0; c < d; ++c) dW[r * d + c] += dz[r] * kt[c];
  }
  std::memcpy(dW0, dW.data(), sizeof(S) * d * d);
}

// Backward of the mini-batch (dual-form) recurrence: per chunk, every
// gradient at the chunk-start W_s, the inclusive causal readout
// o_i = gate (W_s q_i - sum_{j<=i} eta_j (k_j.q_i) G_j), one update
// W_e = W_s - sum_j eta_j G_j k_j^T; reverse mode over the chunks.
template <typename S>
void backward_one_head_minibatch(const S* q, const S* k, const S* v, const S* eta_logit,
                                 const S* gate_logit, const S* W0, const S* gamma,
                                 const S* beta, int T, int d, S eps, unsigned mode, int b,
                                 const unsigned char* mask_row, const S* dO, const S* dW_T,
                                 S* dq, S* dk, S* dv, S* deta, S* dgate, S* dW0, S* dgamma,
                                 S* dbeta) {
  const int n_chunks = (T + b - 1) / b;
  std::vector<S> Ws((size_t)(n_chunks + 1) * d * d);
  std::memcpy(Ws.data(), W0, sizeof(S) * d * d);
  std::vector<S> z(d), dz(d), y(d), dy(d), dWk(d);
  // forward: the chunk-start states
  for (int c = 0; c < n_chunks; ++c) {
    const int t0 = c * b, n = std::min(b, T - t0);
    const bool upd = (mask_row == nullptr) || (mask_row[c] != 0);
    const S* W = Ws.data() + (size_t)c * d * d;
    S* Wn = Ws.data() + (size_t)(c + 1) * d * d;
    std::memcpy(Wn, W, sizeof(S) * d * d);
    for (int j = 0; j < n; ++j) {
      const S* kj = k + (size_t)(t0 + j) * d;
      const S eta = upd ? sigmoid(eta_logit[t0 + j]) / S(d) : S(0);
      std::vector<S> G(d);
      matvec(W, kj, d, z.data());
      ln_and_grad(z.data(), v + (size_t)(t0 + j) * d, gamma, beta, d, eps, mode, (S*)nullptr,
                  G.data(), (S*)nullptr);
      for (int r = 0; r < d; ++r)
        for (int cc = 0; cc < d; ++cc) Wn[r * d + cc] -= eta * G[r] * kj[cc];
    }
  }
  std::vector<S> dW(dW_T, dW_T + (size_t)d * d);  // dL/dW_e of the chunk being undone
  for (int c = n_chunks - 1; c >= 0; --c) {
    const int t0 = c * b, n = std::min(b, T - t0);
    const bool upd = (mask_row == nullptr) || (mask_row[c] != 0);
    const S* W = Ws.data() + (size_t)c * d * d;
    std::vector<S> Gs((size_t)n * d), dGs((size_t)n * d, S(0)), etas(n), sgs(n), detas(n, S(0));
    for (int j = 0; j < n; ++j) {
      sgs[j] = upd ? sigmoid(eta_logit[t0 + j]) : S(0);
      etas[j] = sgs[j] / S(d);
      matvec(W, k + (size_t)(t0 + j) * d, d, z.data());
      ln_and_grad(z.data(), v + (size_t)(t0 + j) * d, gamma, beta, d, eps, mode, (S*)nullptr,
                  Gs.data() + (size_t)j * d, (S*)nullptr);
    }
    std::vector<S> dWs(dW);  // W_e = W_s - ...: identity part
    for (int j = 0; j < n; ++j) {
      const S* kj = k + (size_t)(t0 + j) * d;
      const S* Gj = Gs.data() + (size_t)j * d;
      matvec(dW.data(), kj, d, dWk.data());
      for (int r = 0; r < d; ++r) {
        detas[j] -= Gj[r] * dWk[r];
        dGs[(size_t)j * d + r] -= etas[j] * dWk[r];
      }
      for (int cc = 0; cc < d; ++cc) {
        S acc = 0;
        for (int r = 0; r < d; ++r) acc += dW[r * d + cc] * Gj[r];
        dk[(size_t)(t0 + j) * d + cc] = -etas[j] * acc;
      }
    }
    // outputs of the chunk
    for (int i = 0; i < n; ++i) {
      const int t = t0 + i;
      const S* qi = q + (size_t)t * d;
      const S* dOt = dO + (size_t)t * d;
      matvec(W, qi, d, y.data());
      for (int j = 0; j <= i; ++j) {
        const S a = etas[j] * dot(k + (size_t)(t0 + j) * d, qi, d);
        for (int r = 0; r < d; ++r) y[r] -= a * Gs[(size_t)j * d + r];
      }
      if (gate_logit && (mode & kGateChannel)) {
        for (int r = 0; r < d; ++r) {
          const S g = sigmoid(gate_logit[(size_t)t * d + r]);
          dy[r] = g * dOt[r];
          dgate[(size_t)t * d + r] = dOt[r] * y[r] * g * (S(1) - g);
        }
      } else if (gate_logit) {
        const S g = sigmoid(gate_logit[t]);
        S acc = 0;
        for (int r = 0; r < d; ++r) {
          dy[r] = g * dOt[r];
          acc += dOt[r] * y[r];
        }
        dgate[t] = acc * g * (S(1) - g);
      } else {
        for (int r = 0; r < d; ++r) dy[r] = dOt[r];
      }
      // y = W_s q_i - sum_{j<=i} eta_j (k_j . q_i) G_j
      for (int cc = 0; cc < d; ++cc) {
        S acc = 0;
        for (int r = 0; r < d; ++r) acc += W[r * d + cc] * dy[r];
        dq[(size_t)t * d + cc] = acc;
      }
      for (int r = 0; r < d; ++r)
        for (int cc = 0; cc < d; ++cc) dWs[r * d + cc] += dy[r] * qi[cc];
      for (int j = 0; j <= i; ++j) {
        const S* kj = k + (size_t)(t0 + j) * d;
        const S* Gj = Gs.data() + (size_t)j * d;
        const S kq = dot(kj, qi, d);
        const S dyG = dot(dy.data(), Gj, d);
        for (int cc = 0; cc < d; ++cc) {
          dq[(size_t)t * d + cc] -= etas[j] * dyG * kj[cc];
          dk[(size_t)(t0 + j) * d + cc] -= etas[j] * dyG * qi[cc];
        }
        detas[j] -= kq * dyG;
        for (int r = 0; r < d; ++r) dGs[(size_t)j * d + r] -= etas[j] * kq * dy[r];
      }
    }
    // G_j = G(z_j), z_j = W_s k_j
    for (int j = 0; j < n; ++j) {
      const int t = t0 + j;
      const S* kj = k + (size_t)t * d;
      matvec(W, kj, d, z.data());
      lngrad_backward(z.data(), v + (size_t)t * d, gamma, beta, d, eps, mode,
                      dGs.data() + (size_t)j * d, dz.data(), dv + (size_t)t * d, dgamma, dbeta);
      for (int cc = 0; cc < d; ++cc) {
        S acc = 0;
        for (int r = 0; r < d; ++r) acc += W[r * d + cc] * dz[r];
        dk[(size_t)t * d + cc] += acc;
      }
      for (int r = 0; r < d; ++r)
        for (int cc = 0; cc < d; ++cc) dWs[r * d + cc] += dz[r] * kj[cc];
      deta[t] = upd ? detas[j] * sgs[j] * (S(1) - sgs[j]) / S(d) : S(0);
    }
    dW.swap(dWs);
  }
  std::memcpy(dW0, dW.data(), sizeof(S) * d * d);
}

}  // namespace

extern "C" {

// Backward of the per-token scan (SIMPLE, LN-Jacobian or no-LayerNorm
// gradient; scalar or per-feature gate; mask). Inputs as for the forward scan,
// plus dO [B, H, T, d] and dW_T [B, H, d, d]. Writes dq, dk, dv [B, H, T, d],
// deta [B, H, T], dgate (shape of gate_logit; may be null when gate_logit is),
// dW0 [B, H, d, d], dgamma, dbeta [H, d] (summed over the batch rows; ignored
// with NO_LN). Per-token or mini-batch mode, every gradient form but norm
// matching, the SiLU variant. Returns 0, or -1 on an argument it does not take.
int ttt_oracle_backward_f64(const double* q, const double* k, const double* v,
                            const double* eta_logit, const double* gate_logit,
                            const double* W0, const double* gamma, const double* beta,
                            int B, int H, int T, int d, double eps, unsigned mode, int b,
                            const unsigned char* mask, const double* dO, const double* dW_T,
                            double* dq, double* dk, double* dv, double* deta, double* dgate,
                            double* dW0, double* dgamma, double* dbeta) {
  if (B < 0 || H < 0 || T < 0 || d <= 0 || b <= 0) return -1;
  if (mode & kNormMatch) return -1;
  if ((mode & kGradAblate) && (mode & kNoLayerNorm)) return -1;
  if (!q || !k || !v || !eta_logit || !W0 || !dO || !dW_T || !dq || !dk || !dv || !deta ||
      !dW0)
    return -1;
  if (gate_logit && !dgate) return -1;
  const bool no_ln = mode & kNoLayerNorm;
  if (!no_ln && (!gamma || !beta || !dgamma || !dbeta)) return -1;
  const int n_chunks = (T + b - 1) / b;
  std::vector<double> ones((size_t)d, 1.0), zeros((size_t)d, 0.0), sink_g((size_t)d),
      sink_b((size_t)d);
  if (!no_ln) {
    std::memset(dgamma, 0, sizeof(double) * (size_t)H * d);
    std::memset(dbeta, 0, sizeof(double) * (size_t)H * d);
  }
  const size_t gstride = (mode & kGateChannel) ? (size_t)d : 1;
  std::memset(dv, 0, sizeof(double) * (size_t)B * H * T * d);  // accumulated per token
  // the SiLU variant: run on SiLU(q), SiLU(k), then chain dq, dk through SiLU
  const size_t ntok = (size_t)B * H * T * d;
  std::vector<double> qs, ks;
  const double* q_in = q;
  const double* k_in = k;
  if (mode & kKqSilu) {
    qs.resize(ntok);
    ks.resize(ntok);
    for (size_t i = 0; i < ntok; ++i) {
      qs[i] = silu(q[i]);
      ks[i] = silu(k[i]);
    }
    q = qs.data();
    k = ks.data();
  }
  for (long long bh = 0; bh < (long long)B * H; ++bh) {
    const int bi = (int)(bh / H);
    const int h = (int)(bh % H);
    const size_t tok = (size_t)bh * T;
    auto one = (mode & kMiniBatch) ? backward_one_head_minibatch<double>
                                   : backward_one_head<double>;
    one(q + tok * d, k + tok * d, v + tok * d, eta_logit + tok,
        gate_logit ? gate_logit + tok * gstride : nullptr, W0 + (size_t)bh * d * d,
        no_ln ? ones.data() : gamma + (size_t)h * d, no_ln ? zeros.data() : beta + (size_t)h * d,
        T, d, eps, mode, b, mask ? mask + (size_t)bi * n_chunks : nullptr, dO + tok * d,
        dW_T + (size_t)bh * d * d, dq + tok * d, dk + tok * d, dv + tok * d, deta + tok,
        gate_logit ? dgate + tok * gstride : nullptr, dW0 + (size_t)bh * d * d,
        no_ln ? sink_g.data() : dgamma + (size_t)h * d,
        no_ln ? sink_b.data() : dbeta + (size_t)h * d);
  }
  if (mode & kKqSilu) {
    // d SiLU(x) / dx = sigmoid(x) (1 + x (1 - sigmoid(x)))
    for (size_t i = 0; i < ntok; ++i) {
      const double sq = sigmoid(q_in[i]), sk = sigmoid(k_in[i]);
      dq[i] *= sq * (1.0 + q_in[i] * (1.0 - sq));
      dk[i] *= sk * (1.0 + k_in[i] * (1.0 - sk));
    }
  }
  return 0;
}


// Full scan. All arrays are host, contiguous, row-major:
//   q, k, v, o: [B, H, T, d];  eta_logit: [B, H, T];
//   gate_logit: [B, H, T], or [B, H, T, d] with mode bit 1 << 6 (per-channel gate);
//   W0, W_T: [B, H, d, d] with z = W k;  gamma, beta: [H, d];
//   mask: [B, ceil(T/b)] bytes, 1 = UPDATE, 0 = SKIP;
//   W_chunks: [B, H, ceil(T/b) + 1, d, d], W before each chunk and after the last;
//   grad_norms: [B, H, T, 2] (ablation gradient only, may be null): per token the
//     L2 norm of the full Jacobian-form gradient and of the ablated gradient
//     before any norm matching; zeros on the tokens of SKIP chunks, which take
//     no gradient.
// Returns 0, or -1 on an invalid argument. nthreads <= 0 keeps the OpenMP default.
int ttt_oracle_forward_f64(const double* q, const double* k, const double* v,
                           const double* eta_logit, const double* gate_logit,
                           const double* W0, const double* gamma,
                           const double* beta, int B, int H, int T, int d,
                           double eps, unsigned mode, int b,
                           const unsigned char* mask, double* o, double* W_T,
                           double* W_chunks, double* grad_norms, int nthreads) {
  return forward<double>(q, k, v, eta_logit, gate_logit, W0, gamma, beta, B, H,
                         T, d, eps, mode, b, mask, o, W_T, W_chunks, grad_norms, nthreads);
}

// The same definition evaluated in float (conditioning-floor measurement only).
int ttt_oracle_forward_f32(const float* q, const float* k, const float* v,
                           const float* eta_logit, const float* gate_logit,
                           const float* W0, const float* gamma,
                           const float* beta, int B, int H, int T, int d,
                           float eps, unsigned mode, int b,
                           const unsigned char* mask, float* o, float* W_T,
                           float* W_chunks, float* grad_norms, int nthreads) {
  return forward<float>(q, k, v, eta_logit, gate_logit, W0, gamma, beta, B, H,
                        T, d, eps, mode, b, mask, o, W_T, W_chunks, grad_norms, nthreads);
}

// One inner LayerNorm + gradient evaluation on a single d-vector z (for pins);
// norms (may be null, ablation gradient only) as for grad_norms above.
int ttt_oracle_lngrad_f64(const double* z, const double* v, const double* gamma,
                          const double* beta, int d, double eps, unsigned mode,
                          double* pred, double* G, double* xhat, double* norms) {
  if (!z || !v || !G || d <= 0) return -1;
  if (norms && !(mode & kGradAblate)) return -1;
  if ((mode & kGradAblate) && (mode & kNoLayerNorm)) return -1;
  if ((mode & kNormMatch) && !(mode & kGradAblate)) return -1;
  if (!(mode & kNoLayerNorm) && (!gamma || !beta)) return -1;
  ln_and_grad<double>(z, v, gamma, beta, d, eps, mode, pred, G, xhat, norms);
  return 0;
}

int ttt_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
