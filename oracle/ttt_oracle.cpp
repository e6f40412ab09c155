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

}  // namespace

extern "C" {

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
