// Backward of the TTT-Linear scan on CUDA cores (fp32): the gradients of
// L = <dO, o> + <dW_T, W_T> with respect to q, k, v, the two logits, W0, gamma
// and beta, in per-token and mini-batch mode.
//
// The forward recurrence ("Edifice.Recurrent.TTT", Equations (TTT-Linear);
// mini-batch: PonderTTT, Technical Architecture, dual-form updates) is, per
// token t of a chunk that starts from W_s,
//     z_t = W_{t-1} k_t,  G_t = G(z_t, v_t),  W_t = W_{t-1} - eta_t G_t k_t^T,
//     o_t = gate_t (W_t q_t)
// (mini-batch: every z_t from W_s, o_t = gate_t (W_s q_t - sum_{j<=t} eta_j
// (k_j.q_t) G_j), one update per chunk). Its reverse, with D = dL/dW at the
// chunk end (D_e), dy_t = gate_t dO_t and the exact chunk identity
// W_t = W_s - sum_{j<=t} eta_j G_j k_j^T, is
//     u_t   = D_e k_t + sum_{j>=t} dy_j (q_j.k_t) + sum_{j>t} dz_j (k_j.k_t)
//     deta_t = -G_t.u_t,   dG_t = -eta_t u_t,   dz_t = G'(z_t)^T dG_t
//     dq_t  = W_s^T dy_t - sum_{j<=t} eta_j (G_j.dy_t) k_j
//     dk_t  = -eta_t (D_e^T G_t + sum_{j>=t} (dy_j.G_t) q_j + sum_{j>t} (dz_j.G_t) k_j)
//             + W_s^T dz_t - sum_{j<t} eta_j (G_j.dz_t) k_j
//     D_s   = D_e + sum_t (dy_t q_t^T + dz_t k_t^T)
// where the terms in dz_j (k_j.k_t) and (G_j.dz_t) are absent in mini-batch
// mode (its z_t do not depend on the chunk's earlier gradients). Only the dz_t
// are sequential (the chain, one warp, right to left through the chunk); the
// d x d work (W_s K^T, W_s Q^T, D_e K^T, W_s^T [dy dz], D_e^T G and the rank-2b
// update of D) is batched per chunk. The chunk-start states W_s come from the
// forward's W_chunks snapshots (one per chunk of b tokens); the forward inside a
// chunk is recomputed from W_s with the same identity.
//
// Every LayerNorm gradient step of the reverse chain takes one warp reduction:
// the sums it needs are closed forms in a few sums over u (formed together)
// and in per-token sums the forward recompute leaves behind. In mini-batch
// mode no token's chain step depends on another's, so all warps take tokens.
//
// One CTA of 4d threads per (batch row, head). gamma / beta gradients are
// summed over the head's tokens in the chain warps' registers, then over the
// warps in a fixed order, and written per head to `gb_part`;
// bwd_reduce_gb_kernel sums them over the batch rows in a fixed order.
#pragma once

#include "common.cuh"
#include "scan_simt.cuh"  // kC, butterfly

namespace ttt {

struct BwdParams {
  const void* q;           // [B, H, T, D] fp32 or bf16 (with eta_logit, gate_logit)
  const void* k;
  const void* v;
  const void* eta_logit;   // [B, H, T]
  const void* gate_logit;  // [B, H, T], [B, H, T, D] (gate_channel) or null
  const float* gamma;      // [H, D]; null with no_ln
  const float* beta;
  const unsigned char* mask;  // [B, n_chunks] or null
  const float* W_chunks;   // [B, H, n_chunks + 1, D, D]: W before every chunk of b tokens
  const float* dO;         // [B, H, T, D]
  const float* dW_T;       // [B, H, D, D] or null (zero)
  float* dq;               // [B, H, T, D]
  float* dk;
  float* dv;
  float* deta;             // [B, H, T]
  float* dgate;            // shape of gate_logit, or null
  float* dW0;              // [B, H, D, D]
  float* gb_part;          // [B * H, 2, D]: per head sum of dgamma, dbeta (null with no_ln)
  int B, H, T;
  int b;                   // chunk (<= kC)
  int n_chunks;            // ceil(T / b)
  float eps;
  int gate_channel;
  int kq_silu;
};

template <int D>
struct BwdLayout {
  static constexpr int NT = 4 * D;   // threads: 256 at d = 64, 64 at d = 16
  static constexpr int C = kC;       // largest chunk
  // padded row stride of every [rows][D] array: rows stay 16-byte aligned
  // (float4 reads along a row), and rows r and r+8 of a column fall in
  // different banks
  static constexpr int LD = D + 4;
  static constexpr int MAT = D * LD; // a d x d matrix
  static constexpr int TOK = C * LD; // a [C][D] token array
  static constexpr int GR = C * C;   // a Gram
  // offsets in floats
  static constexpr int oW = 0;                 // W_s
  static constexpr int oDm = oW + MAT;         // D = dL/dW (chunk end, then chunk start)
  static constexpr int oK = oDm + MAT;         // inner-model keys (after SiLU if asked)
  static constexpr int oQ = oK + TOK;          // inner-model queries
  static constexpr int oV = oQ + TOK;
  static constexpr int oDO = oV + TOK;
  static constexpr int oZ = oDO + TOK;         // W_s k_t, then z_t
  static constexpr int oY = oZ + TOK;          // W_s q_t, then y_t = W_t q_t
  static constexpr int oPB = oY + TOK;         // D_e k_t
  static constexpr int oG = oPB + TOK;         // G_t
  static constexpr int oXh = oG + TOK;         // xhat_t (z_t with no LayerNorm)
  static constexpr int oDy = oXh + TOK;        // dy_t = gate_t dO_t
  static constexpr int oDz = oDy + TOK;        // dz_t
  static constexpr int oT1 = oDz + TOK;        // W_s^T dy_t
  static constexpr int oT2 = oT1 + TOK;        // W_s^T dz_t
  static constexpr int oT3 = oT2 + TOK;        // D_e^T G_t
  static constexpr int oKK = oT3 + TOK;        // k_i . k_j
  static constexpr int oQK = oKK + GR;         // q_i . k_j
  static constexpr int oGDy = oQK + GR;        // G_j . dy_i
  static constexpr int oGDz = oGDy + GR;       // G_j . dz_i
  static constexpr int oEta = oGDz + GR;       // eta_t (0 on SKIP chunks and past the chunk)
  static constexpr int oSg = oEta + C;         // sigmoid(eta_logit_t)
  static constexpr int oGate = oSg + C;        // scalar gate_t
  static constexpr int oS = oGate + C;         // per token of the forward: LayerNorm s_t,
  static constexpr int oA = oS + C;            //   mean(g), mean(g xhat) (Jacobian forms),
  static constexpr int oCg = oA + C;           //   sum gamma^2 xhat, sum gamma^2 xhat^2
  static constexpr int oP1 = oCg + C;          //   (LN Jacobian) and sum xhat
  static constexpr int oP2 = oP1 + C;
  static constexpr int oPx = oP2 + C;
  static constexpr int oRs = oPx + C;          //   and 1 / s_t
  static constexpr int floats = oRs + C;
  static constexpr int bytes = floats * 4;
  static_assert(LD % 4 == 0 && oDm % 4 == 0 && oK % 4 == 0 && oQ % 4 == 0 && oG % 4 == 0 &&
                    oDy % 4 == 0 && oDz % 4 == 0,
                "arrays read as float4 start on 16 bytes");
};

__device__ __forceinline__ float4 ld4(const float* a) { return *reinterpret_cast<const float4*>(a); }
__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
  return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, fmaf(a.x, b.x, acc))));
}

__device__ __forceinline__ float silu_grad(float x) {
  const float s = sigmoidf_(x);
  return s * (1.f + x * (1.f - s));
}

template <typename InT>
__device__ __forceinline__ float ld_in(const void* p, size_t i) {
  return to_f32(static_cast<const InT*>(p)[i]);
}

// GM: 0 simplified (G = err), 1 LN Jacobian, 2 no LayerNorm (G = z - v),
// 3 ablation (the Jacobian applied to -gamma v).
template <int D, typename InT, bool MINIB, int GM>
__global__ void __launch_bounds__(4 * D, 1) scan_bwd_kernel(const BwdParams p) {
  using L = BwdLayout<D>;
  constexpr int NT = L::NT, C = L::C, LD = L::LD;
  constexpr int NW = NT / 32;
  constexpr int EPL = (D + 31) / 32;
  constexpr bool kLN = GM != 2;
  constexpr bool kJac = GM == 1 || GM == 3;
  extern __shared__ __align__(16) float sm[];
  float* sW = sm + L::oW;
  float* sD = sm + L::oDm;
  float* sK = sm + L::oK;
  float* sQ = sm + L::oQ;
  float* sV = sm + L::oV;
  float* sDO = sm + L::oDO;
  float* sZ = sm + L::oZ;
  float* sY = sm + L::oY;
  float* sPB = sm + L::oPB;
  float* sG = sm + L::oG;
  float* sXh = sm + L::oXh;
  float* sDy = sm + L::oDy;
  float* sDz = sm + L::oDz;
  float* sT1 = sm + L::oT1;
  float* sT2 = sm + L::oT2;
  float* sT3 = sm + L::oT3;
  float* sKK = sm + L::oKK;
  float* sQK = sm + L::oQK;
  float* sGDy = sm + L::oGDy;
  float* sGDz = sm + L::oGDz;
  float* sEta = sm + L::oEta;
  float* sSg = sm + L::oSg;
  float* sGate = sm + L::oGate;
  float* sS = sm + L::oS;
  float* sA = sm + L::oA;
  float* sCg = sm + L::oCg;
  float* sP1 = sm + L::oP1;
  float* sP2 = sm + L::oP2;
  float* sPx = sm + L::oPx;
  float* sRs = sm + L::oRs;

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const long long bh = blockIdx.x;
  const int bi = (int)(bh / p.H);
  const int h = (int)(bh - (long long)bi * p.H);
  const int T = p.T, b = p.b, nc = p.n_chunks;
  const size_t tok0 = (size_t)bh * T;
  const float inv_d = 1.0f / (float)D;
  const float* Wc = p.W_chunks + (size_t)bh * (nc + 1) * D * D;

  // chain warps: this lane's features f = lane + 32 e, and gamma / beta sums
  float gam[EPL], bet[EPL], dgam[EPL], dbet[EPL];
  float sg2 = 0.f;  // sum of gamma^2 over the head's features
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int f = lane + 32 * e;
    const bool ok = f < D && kLN;
    gam[e] = ok ? p.gamma[(size_t)h * D + f] : 1.f;
    bet[e] = ok ? p.beta[(size_t)h * D + f] : 0.f;
    dgam[e] = 0.f;
    dbet[e] = 0.f;
    if (f < D) sg2 = fmaf(gam[e], gam[e], sg2);
  }
  {
    float t1[1] = {sg2};
    butterfly<1>(t1);
    sg2 = t1[0];
  }
  // per-token mode: warp 0 walks the tokens in order; mini-batch: every warp
  const bool chain_warp = MINIB || warp == 0;

  // D = dW_T
  for (int idx = tid; idx < D * D; idx += NT) {
    const int r = idx / D, c = idx - r * D;
    sD[r * LD + c] = p.dW_T ? p.dW_T[(size_t)bh * D * D + idx] : 0.f;
  }

  // ---- a chunk's global inputs, loaded into registers one chunk ahead (the
  // loads of chunk ch-1 are in flight while chunk ch finishes): this thread's
  // elements idx = tid + NT i of W_s and of the [C][D] token arrays, and (tid
  // < C) token tid's logits. Rows past the chunk and SKIP chunks' eta are
  // zeroed when the registers are stored. ----
  // (Raw values of the input type: converting at the load would wait for it.)
  constexpr int kWpt = D * D / NT, kTpt = C * D / NT;
  const InT* pk = static_cast<const InT*>(p.k);
  const InT* pq = static_cast<const InT*>(p.q);
  const InT* pv = static_cast<const InT*>(p.v);
  const InT* pel = static_cast<const InT*>(p.eta_logit);
  const InT* pgl = static_cast<const InT*>(p.gate_logit);
  float rw[kWpt], ro[kTpt];
  InT rk[kTpt], rq[kTpt], rv[kTpt], rgc[kTpt], rel, rgl;
  auto fetch = [&](int ch) {
    const int t0 = ch * b;
    const int n = min(b, T - t0);
#pragma unroll
    for (int i = 0; i < kWpt; ++i) rw[i] = Wc[(size_t)ch * D * D + tid + NT * i];
#pragma unroll
    for (int i = 0; i < kTpt; ++i) {
      const int idx = tid + NT * i, t = idx / D;
      const size_t g = (tok0 + t0 + t) * D + (idx - t * D);
      rk[i] = rq[i] = rv[i] = rgc[i] = from_f32<InT>(0.f);
      ro[i] = 0.f;
      if (t < n) {
        rk[i] = pk[g];
        rq[i] = pq[g];
        rv[i] = pv[g];
        ro[i] = p.dO[g];
        if (pgl && p.gate_channel) rgc[i] = pgl[g];
      }
    }
    rel = rgl = from_f32<InT>(0.f);
    if (tid < C && tid < n) {
      rel = pel[tok0 + t0 + tid];
      if (pgl && !p.gate_channel) rgl = pgl[tok0 + t0 + tid];
    }
  };
  if (nc > 0) fetch(nc - 1);

  for (int ch = nc - 1; ch >= 0; --ch) {
    const int t0 = ch * b;
    const int n = min(b, T - t0);
    const bool upd = p.mask == nullptr || p.mask[(size_t)bi * nc + ch] != 0;

    // ---- chunk inputs (rows past n are zero), W_s, scalars ----
#pragma unroll
    for (int i = 0; i < kWpt; ++i) {
      const int idx = tid + NT * i, r = idx / D;
      sW[r * LD + idx - r * D] = rw[i];
    }
#pragma unroll
    for (int i = 0; i < kTpt; ++i) {
      const int idx = tid + NT * i, t = idx / D, f = idx - t * D;
      const bool ok = t < n;
      float kv = to_f32(rk[i]), qv = to_f32(rq[i]);
      if (p.kq_silu && ok) {
        kv = siluf_(kv);
        qv = siluf_(qv);
      }
      sK[t * LD + f] = kv;
      sQ[t * LD + f] = qv;
      sV[t * LD + f] = to_f32(rv[i]);
      const float gch = (ok && p.gate_logit && p.gate_channel) ? sigmoidf_(to_f32(rgc[i])) : 1.f;
      // dy = gate dO (the scalar gate is applied below, once it is known)
      sDO[t * LD + f] = ro[i];
      sDy[t * LD + f] = gch * ro[i];
    }
    if (tid < C) {
      const int t = tid;
      const bool ok = t < n;
      const float sg = (ok && upd) ? sigmoidf_(to_f32(rel)) : 0.f;
      sSg[t] = sg;
      sEta[t] = sg * inv_d;
      sGate[t] = (ok && p.gate_logit && !p.gate_channel) ? sigmoidf_(to_f32(rgl)) : 1.f;
    }
    __syncthreads();
    if (p.gate_logit && !p.gate_channel) {
      for (int idx = tid; idx < C * D; idx += NT) {
        const int t = idx / D, f = idx - t * D;
        sDy[t * LD + f] *= sGate[t];
      }
    }

    // ---- batched: W_s k_t, W_s q_t, D_e k_t (thread: row r, tokens tg + 4m) ----
    {
      const int r = tid % D, tg = tid / D;
      constexpr int NTK = C / 4;
      float az[NTK], ay[NTK], ap[NTK];
#pragma unroll
      for (int m = 0; m < NTK; ++m) az[m] = ay[m] = ap[m] = 0.f;
      for (int c = 0; c < D; c += 4) {
        const float4 w = ld4(sW + r * LD + c), dd = ld4(sD + r * LD + c);
#pragma unroll
        for (int m = 0; m < NTK; ++m) {
          const int t = tg + 4 * m;
          const float4 kc = ld4(sK + t * LD + c);
          az[m] = dot4(w, kc, az[m]);
          ay[m] = dot4(w, ld4(sQ + t * LD + c), ay[m]);
          ap[m] = dot4(dd, kc, ap[m]);
        }
      }
#pragma unroll
      for (int m = 0; m < NTK; ++m) {
        const int t = tg + 4 * m;
        sZ[t * LD + r] = az[m];
        sY[t * LD + r] = ay[m];
        sPB[t * LD + r] = ap[m];
      }
    }
    // ---- Grams k_i.k_j and q_i.k_j ----
    for (int idx = tid; idx < C * C; idx += NT) {
      const int i = idx / C, j = idx - i * C;
      float kk = 0.f, qk = 0.f;
      for (int f = 0; f < D; f += 4) {
        const float4 kj = ld4(sK + j * LD + f);
        kk = dot4(ld4(sK + i * LD + f), kj, kk);
        qk = dot4(ld4(sQ + i * LD + f), kj, qk);
      }
      sKK[idx] = kk;
      sQK[idx] = qk;
    }
    __syncthreads();

    // ---- forward chain: z_t, LayerNorm (one reduction of shifted moments),
    //      G_t, and the per-token sums the reverse chain needs ----
    // One token's LayerNorm and gradient from its z (this lane's features):
    // writes G, xhat and the per-token sums, returns G.
    auto fwd_token = [&](int t, const float (&z)[EPL], float (&G)[EPL]) {
      float v[EPL], xh[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const int f = lane + 32 * e;
        v[e] = f < D ? sV[t * LD + f] : 0.f;
      }
      if (!kLN) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          G[e] = (lane + 32 * e < D) ? z[e] - v[e] : 0.f;
          xh[e] = z[e];
        }
      } else {
        // shift by one element of the token; moments of y = z - shift:
        // sum y, sum y^2 and (Jacobian forms) sum a y, sum a y^2, sum c y, sum c
        // with g = a xhat + c (LN Jacobian: a = gamma^2, c = gamma (beta - v);
        // ablation: a = 0, c = -gamma v)
        const float c0 = __shfl_sync(0xffffffffu, z[0], 0);
        constexpr int NM = kJac ? 6 : 2;
        float m[NM], y[EPL], aa[EPL], cc[EPL];
#pragma unroll
        for (int i = 0; i < NM; ++i) m[i] = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          const bool fv = lane + 32 * e < D;
          y[e] = fv ? z[e] - c0 : 0.f;
          aa[e] = (fv && GM == 1) ? gam[e] * gam[e] : 0.f;
          cc[e] = !fv ? 0.f : (GM == 3 ? -gam[e] * v[e] : gam[e] * (bet[e] - v[e]));
          m[0] += y[e];
          m[1] = fmaf(y[e], y[e], m[1]);
          if (kJac) {
            const float ay = aa[e] * y[e];
            m[2] += ay;
            m[3] = fmaf(ay, y[e], m[3]);
            m[4] = fmaf(cc[e], y[e], m[4]);
            m[5] += cc[e];
          }
        }
        butterfly<NM>(m);
        const float mu1 = m[0] * inv_d;
        const float ve = fmaxf(fmaf(m[1], inv_d, -mu1 * mu1), 0.f) + p.eps;
        const float rs = rsqrtf(ve);  // 1 / s, s = sqrt(var + eps)
        const float s = ve * rs;
#pragma unroll
        for (int e = 0; e < EPL; ++e) xh[e] = (lane + 32 * e < D) ? (y[e] - mu1) * rs : 0.f;
        if (kJac) {
          const float sa = (GM == 1) ? sg2 : 0.f;                                 // sum of a
          const float p1 = (m[2] - mu1 * sa) * rs;                                // sum a xhat
          const float p2 = (m[3] - 2.f * mu1 * m[2] + mu1 * mu1 * sa) * (rs * rs);  // sum a xhat^2
          const float a_ = (p1 + m[5]) * inv_d;                                   // mean g
          const float cg = fmaf(m[4] - mu1 * m[5], rs, p2) * inv_d;               // mean g xhat
#pragma unroll
          for (int e = 0; e < EPL; ++e) {
            const float g = fmaf(aa[e], xh[e], cc[e]);
            G[e] = (lane + 32 * e < D) ? (g - a_ - xh[e] * cg) * rs : 0.f;
          }
          if (lane == 0) {
            sA[t] = a_;
            sCg[t] = cg;
            sP1[t] = p1;
            sP2[t] = p2;
          }
        } else {
#pragma unroll
          for (int e = 0; e < EPL; ++e)
            G[e] = (lane + 32 * e < D) ? fmaf(gam[e], xh[e], bet[e]) - v[e] : 0.f;
        }
        if (lane == 0) {
          sS[t] = s;
          sRs[t] = rs;
          sPx[t] = (m[0] - (float)D * mu1) * rs;  // sum xhat
        }
      }
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const int f = lane + 32 * e;
        if (f < D) {
          sG[t * LD + f] = G[e];
          sXh[t * LD + f] = xh[e];
        }
      }
    };
    auto zero_rows = [&](float* a, int t) {
#pragma unroll
      for (int e = 0; e < EPL; ++e)
        if (lane + 32 * e < D) a[t * LD + lane + 32 * e] = 0.f;
    };
    if (MINIB) {
      // every token's z is W_s k_t: every warp takes tokens
      for (int t = warp; t < C; t += NW) {
        if (t >= n || !upd) {  // SKIP chunks take no gradient (eta = 0)
          zero_rows(sG, t);
          zero_rows(sXh, t);
          continue;
        }
        float z[EPL], G[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) z[e] = (lane + 32 * e < D) ? sZ[t * LD + lane + 32 * e] : 0.f;
        fwd_token(t, z, G);
      }
    } else if (warp == 0) {
      // token by token: z_t = W_s k_t - sum_{j<t} eta_j (k_t . k_j) G_j, the
      // earlier G_j read back from shared memory (this lane wrote them); a
      // rolled loop keeps the chain's code small
#pragma unroll 1
      for (int t = 0; t < C; ++t) {
        if (t < n && upd) {
          float z[EPL], G[EPL];
#pragma unroll
          for (int e = 0; e < EPL; ++e) z[e] = (lane + 32 * e < D) ? sZ[t * LD + lane + 32 * e] : 0.f;
          for (int j = 0; j < t; ++j) {
            const float a = -sEta[j] * sKK[t * C + j];
#pragma unroll
            for (int e = 0; e < EPL; ++e)
              if (lane + 32 * e < D) z[e] = fmaf(a, sG[j * LD + lane + 32 * e], z[e]);
          }
          fwd_token(t, z, G);
        } else {
          zero_rows(sG, t);
          zero_rows(sXh, t);
        }
      }
    }
    __syncthreads();

    // ---- readout y_t = W_s q_t - sum_{j<=t} eta_j (q_t.k_j) G_j and the gate
    //      gradients; the part of u_t that does not wait for the chain,
    //      D_e k_t + sum_{j>=t} dy_j (q_j.k_t), into sPB ----
    for (int idx = tid; idx < C * D; idx += NT) {
      const int t = idx / D, f = idx - t * D;
      float y = sY[t * LD + f];
      if (upd)
        for (int j = 0; j <= t; ++j) y = fmaf(-sEta[j] * sQK[t * C + j], sG[j * LD + f], y);
      sY[t * LD + f] = y;
      if (p.gate_logit && p.gate_channel && t < n) {
        const size_t g = (tok0 + t0 + t) * D + f;
        const float gs = sigmoidf_(ld_in<InT>(p.gate_logit, g));
        p.dgate[g] = sDO[t * LD + f] * y * gs * (1.f - gs);
      }
      float u = sPB[t * LD + f];
      for (int j = t; j < n; ++j) u = fmaf(sQK[j * C + t], sDy[j * LD + f], u);
      sPB[t * LD + f] = u;
    }
    __syncthreads();
    if (p.gate_logit && !p.gate_channel) {
      // one warp per token: dL/dgate_logit = (dO . y) gate (1 - gate)
      for (int t = warp; t < n; t += NT / 32) {
        float acc[1] = {0.f};
        for (int f = lane; f < D; f += 32) acc[0] = fmaf(sDO[t * LD + f], sY[t * LD + f], acc[0]);
        butterfly<1>(acc);
        if (lane == 0) {
          const float gs = sGate[t];
          p.dgate[tok0 + t0 + t] = acc[0] * gs * (1.f - gs);
        }
      }
    }

    // ---- reverse chain: deta_t, dz_t, dv_t from u_t (per-token mode: warp 0,
    //      right to left, u in registers; mini-batch: every warp) ----
    // One token's step: the LayerNorm backward of dG = -eta u in closed form
    // (one warp reduction); writes deta, dz, dv and adds to the gamma / beta sums.
    auto bwd_token = [&](int t, const float (&u)[EPL], float (&dz)[EPL]) {
      const size_t gt = tok0 + t0 + t;
      float G[EPL], xh[EPL], v[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const int f = lane + 32 * e;
        G[e] = f < D ? sG[t * LD + f] : 0.f;
        xh[e] = f < D ? sXh[t * LD + f] : 0.f;
        v[e] = f < D ? sV[t * LD + f] : 0.f;
      }
      // sum G u, sum u, sum u xhat, sum u w, sum u w xhat with w = gamma^2 (LN
      // Jacobian) or gamma (simplified gradient)
      float m[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const float w = GM == 1 ? gam[e] * gam[e] : gam[e];
        m[0] = fmaf(G[e], u[e], m[0]);
        m[1] += u[e];
        m[2] = fmaf(u[e], xh[e], m[2]);
        m[3] = fmaf(u[e], w, m[3]);
        m[4] = fmaf(u[e] * w, xh[e], m[4]);
      }
      butterfly<5>(m);
      const float eta = sEta[t];
      if (lane == 0) p.deta[gt] = -m[0] * sSg[t] * (1.f - sSg[t]) * inv_d;
      float dv[EPL];
      if (!kLN) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          dz[e] = -eta * u[e];
          dv[e] = eta * u[e];
        }
      } else {
        // dG = -eta u; the sums of the LayerNorm backward in closed form
        const float s = sS[t], rs = sRs[t];
        const float mdG = -eta * m[1] * inv_d, mdGx = -eta * m[2] * inv_d;
        float ds = 0.f, s_jx = 0.f, s_j = 0.f, s_ex = 0.f, s_e = 0.f;
        if (kJac) {
          const float a_ = sA[t], cg = sCg[t];
          ds = eta * m[0] * rs;                           // -(sum dG G) / s
          s_jx = -2.f * (float)D * cg * mdGx * rs;        // sum of the Jacobian part of dxhat * xhat
          s_j = -(float)D * (cg * mdG + a_ * mdGx) * rs;  // ... and of that part alone
        }
        if (GM == 1) {         // derr = dg gamma: sums of derr gamma xhat, derr gamma
          s_ex = (-eta * m[4] - mdG * sP1[t] - mdGx * sP2[t]) * rs;
          s_e = (-eta * m[3] - mdG * sg2 - mdGx * sP1[t]) * rs;
        } else if (GM == 0) {  // derr = dG
          s_ex = -eta * m[4];
          s_e = -eta * m[3];
        }
        const float dxx = s_jx + s_ex;
        const float dvar = (ds - dxx * rs) * (0.5f * rs);
        const float mdy = ((s_j + s_e) * rs + dvar * 2.f * s * sPx[t] * inv_d) * inv_d;
        const float cgt = kJac ? sCg[t] : 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          const bool fv = lane + 32 * e < D;
          const float dG = -eta * u[e];
          float derr, dxh = 0.f;
          dv[e] = 0.f;
          if (kJac) {
            const float g = GM == 3 ? -gam[e] * v[e] : gam[e] * (fmaf(gam[e], xh[e], bet[e]) - v[e]);
            const float dg = (dG - mdG - xh[e] * mdGx) * rs;
            dxh = (-dG * cgt - g * mdGx) * rs;
            if (GM == 3) {
              if (fv) {
                dgam[e] -= dg * v[e];
                dv[e] -= dg * gam[e];
              }
              derr = 0.f;
            } else {
              if (fv) dgam[e] = fmaf(dg, fmaf(gam[e], xh[e], bet[e]) - v[e], dgam[e]);
              derr = dg * gam[e];
            }
          } else {
            derr = dG;
          }
          // err = gamma xhat + beta - v
          if (fv) {
            dgam[e] = fmaf(derr, xh[e], dgam[e]);
            dbet[e] += derr;
          }
          dv[e] -= derr;
          dxh = fmaf(derr, gam[e], dxh);
          // xhat = (z - mu) / s, s = sqrt(var + eps), z - mu = xhat s
          dz[e] = fv ? fmaf(dxh, rs, dvar * 2.f * xh[e] * s * inv_d) - mdy : 0.f;
        }
      }
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const int f = lane + 32 * e;
        if (f < D) {
          sDz[t * LD + f] = dz[e];
          p.dv[gt * D + f] = dv[e];
        }
      }
    };
    auto skip_token = [&](int t) {  // a SKIP chunk takes no gradient
      const size_t gt = tok0 + t0 + t;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const int f = lane + 32 * e;
        if (f < D) {
          sDz[t * LD + f] = 0.f;
          p.dv[gt * D + f] = 0.f;
        }
      }
      if (lane == 0) p.deta[gt] = 0.f;
    };
    if (MINIB) {
      for (int t = warp; t < C; t += NW) {
        if (t >= n) {
          zero_rows(sDz, t);
          continue;
        }
        if (!upd) {
          skip_token(t);
          continue;
        }
        float u[EPL], dz[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) u[e] = (lane + 32 * e < D) ? sPB[t * LD + lane + 32 * e] : 0.f;
        bwd_token(t, u, dz);
      }
    } else if (warp == 0) {
      // right to left: u_t = (the part in sPB) + sum_{j>t} (k_j . k_t) dz_j,
      // the later dz_j read back from shared memory (this lane wrote them)
#pragma unroll 1
      for (int i = 0; i < C; ++i) {
        const int t = C - 1 - i;
        if (t >= n) {
          zero_rows(sDz, t);
        } else if (!upd) {
          skip_token(t);
        } else {
          float u[EPL], dz[EPL];
#pragma unroll
          for (int e = 0; e < EPL; ++e) u[e] = (lane + 32 * e < D) ? sPB[t * LD + lane + 32 * e] : 0.f;
          for (int j = n - 1; j > t; --j) {
            const float a = sKK[j * C + t];
#pragma unroll
            for (int e = 0; e < EPL; ++e)
              if (lane + 32 * e < D) u[e] = fmaf(a, sDz[j * LD + lane + 32 * e], u[e]);
          }
          bwd_token(t, u, dz);
        }
      }
    }
    // the next chunk's loads, issued once the chains (whose registers they
    // would crowd) are done
    if (ch > 0) fetch(ch - 1);
    __syncthreads();

    // ---- batched: W_s^T dy_t, W_s^T dz_t, D_e^T G_t (thread: column c, tokens tg + 4m);
    //      Grams G_j.dy_i, G_j.dz_i ----
    {
      const int c = tid % D, tg = tid / D;
      constexpr int NTK = C / 4;
      float a1[NTK], a2[NTK], a3[NTK];
#pragma unroll
      for (int m = 0; m < NTK; ++m) a1[m] = a2[m] = a3[m] = 0.f;
      for (int r = 0; r < D; r += 4) {
        const float4 w = make_float4(sW[r * LD + c], sW[(r + 1) * LD + c], sW[(r + 2) * LD + c],
                                     sW[(r + 3) * LD + c]);
        const float4 dd = make_float4(sD[r * LD + c], sD[(r + 1) * LD + c], sD[(r + 2) * LD + c],
                                      sD[(r + 3) * LD + c]);
#pragma unroll
        for (int m = 0; m < NTK; ++m) {
          const int t = tg + 4 * m;
          a1[m] = dot4(w, ld4(sDy + t * LD + r), a1[m]);
          a2[m] = dot4(w, ld4(sDz + t * LD + r), a2[m]);
          a3[m] = dot4(dd, ld4(sG + t * LD + r), a3[m]);
        }
      }
#pragma unroll
      for (int m = 0; m < NTK; ++m) {
        const int t = tg + 4 * m;
        sT1[t * LD + c] = a1[m];
        sT2[t * LD + c] = a2[m];
        sT3[t * LD + c] = a3[m];
      }
    }
    for (int idx = tid; idx < C * C; idx += NT) {
      const int i = idx / C, j = idx - i * C;
      float gy = 0.f, gz = 0.f;
      for (int f = 0; f < D; f += 4) {
        const float4 gj = ld4(sG + j * LD + f);
        gy = dot4(gj, ld4(sDy + i * LD + f), gy);
        gz = dot4(gj, ld4(sDz + i * LD + f), gz);
      }
      sGDy[idx] = gy;
      sGDz[idx] = gz;
    }
    __syncthreads();

    // ---- dq, dk (chained through SiLU for the `:mlp` variant) ----
    for (int idx = tid; idx < C * D; idx += NT) {
      const int t = idx / D, c = idx - t * D;
      if (t >= n) continue;
      float dq = sT1[t * LD + c];
      float dk = sT2[t * LD + c];
      if (upd) {
        float a = sT3[t * LD + c];
        for (int j = t; j < n; ++j) a = fmaf(sGDy[j * C + t], sQ[j * LD + c], a);
        if (!MINIB)
          for (int j = t + 1; j < n; ++j) a = fmaf(sGDz[j * C + t], sK[j * LD + c], a);
        dk = fmaf(-sEta[t], a, dk);
        for (int j = 0; j <= t; ++j) dq = fmaf(-sEta[j] * sGDy[t * C + j], sK[j * LD + c], dq);
        if (!MINIB)
          for (int j = 0; j < t; ++j) dk = fmaf(-sEta[j] * sGDz[t * C + j], sK[j * LD + c], dk);
      }
      const size_t g = (tok0 + t0 + t) * D + c;
      if (p.kq_silu) {
        dq *= silu_grad(ld_in<InT>(p.q, g));
        dk *= silu_grad(ld_in<InT>(p.k, g));
      }
      p.dq[g] = dq;
      p.dk[g] = dk;
    }
    // ---- D_s = D_e + sum_t (dy_t q_t^T + dz_t k_t^T): a TS x TS tile of D
    //      per thread, so each value read from shared memory feeds TS FMAs ----
    {
      constexpr int TS = (D == 64) ? 4 : 2;  // TS * TS = D * D / NT
      static_assert(TS * TS * NT == D * D, "one tile per thread");
      const int r0 = TS * (tid / (D / TS)), c0 = TS * (tid % (D / TS));
      float acc[TS][TS];
#pragma unroll
      for (int i = 0; i < TS; ++i)
#pragma unroll
        for (int j = 0; j < TS; ++j) acc[i][j] = sD[(r0 + i) * LD + c0 + j];
      for (int t = 0; t < n; ++t) {
        float dy[TS], dz[TS], q[TS], k[TS];
#pragma unroll
        for (int i = 0; i < TS; ++i) {
          dy[i] = sDy[t * LD + r0 + i];
          dz[i] = sDz[t * LD + r0 + i];
          q[i] = sQ[t * LD + c0 + i];
          k[i] = sK[t * LD + c0 + i];
        }
#pragma unroll
        for (int i = 0; i < TS; ++i)
#pragma unroll
          for (int j = 0; j < TS; ++j) acc[i][j] = fmaf(dz[i], k[j], fmaf(dy[i], q[j], acc[i][j]));
      }
#pragma unroll
      for (int i = 0; i < TS; ++i)
#pragma unroll
        for (int j = 0; j < TS; ++j) sD[(r0 + i) * LD + c0 + j] = acc[i][j];
    }
    __syncthreads();
  }

  // ---- dW0 = D, per-head gamma / beta sums ----
  for (int idx = tid; idx < D * D; idx += NT) {
    const int r = idx / D, c = idx - r * D;
    p.dW0[(size_t)bh * D * D + idx] = sD[r * LD + c];
  }
  if (kLN && p.gb_part != nullptr) {
    // the chain warps' sums, added over the warps in warp order
    float* red = sT1;  // [NW][2][D] (free after the last chunk)
    if (chain_warp) {
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const int f = lane + 32 * e;
        if (f < D) {
          red[(warp * 2) * D + f] = dgam[e];
          red[(warp * 2 + 1) * D + f] = dbet[e];
        }
      }
    }
    __syncthreads();
    if (tid < 2 * D) {
      const int which = tid / D, f = tid - which * D;
      float acc = 0.f;
      for (int w = 0; w < (MINIB ? NW : 1); ++w) acc += red[(w * 2 + which) * D + f];
      p.gb_part[((size_t)bh * 2 + which) * D + f] = acc;
    }
  }
}

// dgamma[h][f] = sum over batch rows of the per-head sums (in batch-row order,
// so the result does not depend on scheduling); likewise dbeta.
__global__ void bwd_reduce_gb_kernel(const float* __restrict__ gb_part, int B, int H, int D,
                                     float* __restrict__ dgamma, float* __restrict__ dbeta) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= H * D) return;
  const int h = idx / D, f = idx - h * D;
  float sg = 0.f, sb = 0.f;
  for (int bi = 0; bi < B; ++bi) {
    const size_t bh = (size_t)bi * H + h;
    sg += gb_part[(bh * 2) * D + f];
    sb += gb_part[(bh * 2 + 1) * D + f];
  }
  dgamma[idx] = sg;
  dbeta[idx] = sb;
}

}  // namespace ttt
