// Streaming decode step: one token for every (batch row, head), fast weights
// updated in place. This is the per-token recurrence of "Edifice.Recurrent.TTT",
// section "Equations (TTT-Linear)", for a single t, with the state carried
// between calls the way cortex_rust src/layers/ttt.rs (forward_update) takes a
// weight state in and returns the output and the new state.
//
// Per head, from ONE read of W:
//   z = W k and W q (both from the same registers),
//   LayerNorm + gradient G (simplified, LN-Jacobian, no LayerNorm, or the
//     ablation: the Jacobian applied to -gamma v, optionally norm-matched),
//   eta = sigmoid(eta_logit) / d, or 0 when the batch row's update flag is 0,
//   W' = W - eta G k^T, written back in place (not written at all when eta = 0,
//        so a skipped head keeps its W bit for bit),
//   o  = gate * (W' q) = gate * (W q - eta (k . q) G).
// W is read once and written once, so the step is bound by HBM bandwidth
// (2 d^2 x 4 bytes of state per head and token).
//
// Layout: 16 rows of W per warp. In load i a warp reads RPI consecutive rows
// (RPI * d floats = 512 contiguous bytes), lane l taking the float4 at column
// 4 (l % LPR) of row RPI i + l / LPR. The per-row dot products are finished by
// a butterfly that halves the row set at every step (reduce-scatter), leaving
// each row's sums on two adjacent lanes.
#pragma once

#include "common.cuh"

namespace ttt {

struct DecodeParams {
  const void* q;              // [B, H, D]
  const void* k;
  const void* v;
  const void* eta_logit;      // [B, H]
  const void* gate_logit;     // [B, H] or [B, H, D]; may be null
  float* W;                   // [B, H, D, D], in place
  const float* gamma;         // [H, D]; may be null with no_ln
  const float* beta;
  const unsigned char* update;  // [B] or null
  void* o;                    // [B, H, D]
  long long heads;            // B * H
  int H;
  float eps;
  int lnjac, no_ln, gate_channel;
  int ablate, norm_match;   // ablation gradient; per-token norm matching
  int kq_silu;              // the `:mlp` variant: SiLU on k and q as they are loaded
};

template <int D>
struct DecodeShape {
  static constexpr int NT = 128;          // threads per CTA
  static constexpr int WPH = D / 16;      // warps per head (16 rows each)
  static constexpr int HPB = 4 / WPH;     // heads per CTA
  static constexpr int LPR = D / 4;       // lanes per row (4 columns per lane)
  static constexpr int RPI = 32 / LPR;    // rows per warp-wide load
  static constexpr int NI = 16 / RPI;     // loads per lane
  static_assert(NI * 2 == LPR, "reduce-scatter needs NI == LPR / 2");
};

template <typename InT>
__device__ __forceinline__ void load4(const InT* p, float* out);
template <>
__device__ __forceinline__ void load4<float>(const float* p, float* out) {
  const float4 x = __ldg(reinterpret_cast<const float4*>(p));
  out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float* out) {
  const uint2 x = __ldg(reinterpret_cast<const uint2*>(p));
  out[0] = __uint_as_float(x.x << 16); out[1] = __uint_as_float(x.x & 0xffff0000u);
  out[2] = __uint_as_float(x.y << 16); out[3] = __uint_as_float(x.y & 0xffff0000u);
}

// p[0..N) are partial sums of rows i = 0..N-1, spread over 2N lanes (lane bits
// 0..log2(N)). Afterwards p[0] on lane l holds the full sum of row
// (l >> 1) & (N - 1).
template <int N>
__device__ __forceinline__ void reduce_scatter(float (&p)[N], int lane) {
#pragma unroll
  for (int s = N / 2; s >= 1; s >>= 1) {
    const bool up = lane & (2 * s);
#pragma unroll
    for (int j = 0; j < s; ++j) {
      const float send = up ? p[j] : p[j + s];
      const float keep = up ? p[j + s] : p[j];
      p[j] = keep + __shfl_xor_sync(0xffffffffu, send, 2 * s);
    }
  }
  p[0] += __shfl_xor_sync(0xffffffffu, p[0], 1);
}

template <int D, typename InT, typename OutT>
__global__ void __launch_bounds__(DecodeShape<D>::NT) decode_step_kernel(const DecodeParams p) {
  using S = DecodeShape<D>;
  __shared__ float red[5][S::WPH][2];    // per-warp partials of the LayerNorm rounds
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wih = warp % S::WPH;
  const long long bh = (long long)blockIdx.x * S::HPB + warp / S::WPH;
  // Only CTAs holding several heads (one warp each, no block barrier) have a tail.
  if (bh >= p.heads) return;
  const int bi = (int)(bh / p.H);
  const int h = (int)(bh - (long long)bi * p.H);
  const int cg = lane % S::LPR;       // column group: columns 4 cg .. 4 cg + 3
  const int rsub = lane / S::LPR;     // row within one warp-wide load

  // ---- all global loads first: W (this warp's 16 rows), then the token ----
  float* Wp = p.W + (size_t)bh * D * D + (size_t)(16 * wih + rsub) * D + 4 * cg;
  float4 w[S::NI];
#pragma unroll
  for (int i = 0; i < S::NI; ++i)
    w[i] = __ldcs(reinterpret_cast<const float4*>(Wp + (size_t)i * S::RPI * D));
  float kk[4], qq[4];
  load4<InT>(static_cast<const InT*>(p.k) + bh * D + 4 * cg, kk);
  load4<InT>(static_cast<const InT*>(p.q) + bh * D + 4 * cg, qq);
  if (p.kq_silu) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      kk[i] = siluf_(kk[i]);
      qq[i] = siluf_(qq[i]);
    }
  }
  // the head row this lane ends up holding after the reductions
  const int rr = 16 * wih + S::RPI * ((lane >> 1) & (S::NI - 1)) + rsub;
  const float vr = to_f32(static_cast<const InT*>(p.v)[bh * D + rr]);
  const float eta_l = to_f32(static_cast<const InT*>(p.eta_logit)[bh]);
  float gate_l = 0.f;
  if (p.gate_logit)
    gate_l = to_f32(static_cast<const InT*>(p.gate_logit)[p.gate_channel ? bh * D + rr : bh]);
  float gam = 1.f, bet = 0.f;
  if (!p.no_ln) {
    gam = __ldg(p.gamma + (size_t)h * D + rr);
    bet = __ldg(p.beta + (size_t)h * D + rr);
  }
  const bool upd = (p.update == nullptr) || (p.update[bi] != 0);

  // ---- z = W k, W q and k . q ----
  float pz[S::NI], pq[S::NI];
#pragma unroll
  for (int i = 0; i < S::NI; ++i) {
    pz[i] = fmaf(w[i].x, kk[0], fmaf(w[i].y, kk[1], fmaf(w[i].z, kk[2], w[i].w * kk[3])));
    pq[i] = fmaf(w[i].x, qq[0], fmaf(w[i].y, qq[1], fmaf(w[i].z, qq[2], w[i].w * qq[3])));
  }
  float kq = fmaf(kk[0], qq[0], fmaf(kk[1], qq[1], fmaf(kk[2], qq[2], kk[3] * qq[3])));
  reduce_scatter<S::NI>(pz, lane);
  reduce_scatter<S::NI>(pq, lane);
#pragma unroll
  for (int off = 1; off < S::LPR; off <<= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
  const float z = pz[0], wq = pq[0];

  // Sum over the head's D rows: lanes l and l ^ 1 hold the same row, so the
  // warp sum runs over lane bits 1..4 only; then across the head's warps.
  auto head_sum = [&](float a, float b, int round) -> float2 {
#pragma unroll
    for (int off = 2; off < 32; off <<= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, off);
      b += __shfl_xor_sync(0xffffffffu, b, off);
    }
    if constexpr (S::WPH > 1) {
      if (lane == 0) { red[round][wih][0] = a; red[round][wih][1] = b; }
      __syncthreads();
      a = 0.f; b = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < S::WPH; ++w2) { a += red[round][w2][0]; b += red[round][w2][1]; }
    }
    return make_float2(a, b);
  };

  // ---- LayerNorm and the inner gradient of this lane's row ----
  float G;
  if (p.no_ln) {
    G = z - vr;
  } else {
    constexpr float inv_d = 1.0f / (float)D;
    const float mu = head_sum(z, 0.f, 0).x * inv_d;
    const float y = z - mu;
    const float var = head_sum(y * y, 0.f, 1).x * inv_d;
    const float s = sqrtf(var + p.eps);
    const float xh = y / s;
    const float err = fmaf(gam, xh, bet) - vr;
    // back through the LayerNorm: J^T g = (g - mean g - xhat mean(g xhat)) / s
    auto jacobian_t = [&](float g, int round) {
      const float2 m = head_sum(g, g * xh, round);
      return (g - m.x * inv_d - xh * (m.y * inv_d)) / s;
    };
    if (p.ablate) {
      // the prediction removed, the Jacobian kept; optionally rescaled to the
      // full gradient's norm
      G = jacobian_t(-gam * vr, 2);
      if (p.norm_match) {
        const float Gf = jacobian_t(gam * err, 3);
        const float2 n = head_sum(Gf * Gf, G * G, 4);
        G *= n.y > 0.f ? sqrtf(n.x / n.y) : 0.f;
      }
    } else if (p.lnjac) {
      G = jacobian_t(gam * err, 2);
    } else {
      G = err;
    }
  }

  // ---- W' = W - eta G k^T, in place ----
  const float eta = upd ? sigmoidf_(eta_l) / (float)D : 0.f;
  if (eta != 0.f) {
    const float eg = eta * G;
#pragma unroll
    for (int i = 0; i < S::NI; ++i) {
      // G of row RPI i + rsub sits on lane rsub * LPR + 2 i
      const float gi = __shfl_sync(0xffffffffu, eg, rsub * S::LPR + 2 * i);
      float4 x = w[i];
      x.x = fmaf(-gi, kk[0], x.x);
      x.y = fmaf(-gi, kk[1], x.y);
      x.z = fmaf(-gi, kk[2], x.z);
      x.w = fmaf(-gi, kk[3], x.w);
      __stcs(reinterpret_cast<float4*>(Wp + (size_t)i * S::RPI * D), x);
    }
  }

  // ---- o = gate * (W q - eta (k . q) G) ----
  if ((lane & 1) == 0) {
    const float gate = p.gate_logit ? sigmoidf_(gate_l) : 1.f;
    static_cast<OutT*>(p.o)[bh * D + rr] = from_f32<OutT>(gate * fmaf(-eta * kq, G, wq));
  }
}

}  // namespace ttt
