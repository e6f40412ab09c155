// CUDA-core (fp32) scan kernel: exact per-token recurrence and mini-batch dual
// form, any input/output dtype, d in {16, 64}.
//
// One CTA per (batch row, head) keeps W in shared memory in fp32 for the whole
// sequence. Tokens are processed in chunks of C tokens using the exact
// chunk identity of the per-token recurrence ("Edifice.Recurrent.TTT",
// Equations (TTT-Linear)): with W_s the state at the chunk start and
// a_ij = eta_j (k_j . k_i),
//
//     z_i = W_{i-1} k_i = W_s k_i - sum_{j<i} a_ij G_j
//     o_i = W_i q_i     = W_s q_i - sum_{j<=i} eta_j (k_j . q_i) G_j
//     W_e = W_s - sum_j eta_j G_j k_j^T
//
// so the d x d work (W_s K^T, W_s Q^T, the rank-C update) runs on all threads
// while only the O(C d) gradient chain stays sequential (one warp). Mini-batch
// mode (PonderTTT, dual-form updates) is the same chunk step without the
// correction of z_i, with C = b.
#pragma once

#include "common.cuh"

namespace ttt {

constexpr int kSimtCMax = 16;

template <int D>
struct SimtLayout {
  static constexpr int NT = 4 * D;           // threads per CTA
  static constexpr int NW = NT / 32;         // warps per CTA
  static constexpr int KP = D + 1;           // padded row stride of the W, K and Q tiles
  // shared-memory carve-up, in floats
  static constexpr int oW = 0;                        // W     [D][KP]
  static constexpr int oK = oW + D * KP;              // K     [CMAX][KP]
  static constexpr int oQ = oK + kSimtCMax * KP;      // Q     [CMAX][KP]
  static constexpr int oV = oQ + kSimtCMax * KP;      // V     [CMAX][D]
  static constexpr int oZ = oV + kSimtCMax * D;       // W_s K^T  [CMAX][D]
  static constexpr int oQ0 = oZ + kSimtCMax * D;      // W_s Q^T  [CMAX][D]
  static constexpr int oG = oQ0 + kSimtCMax * D;      // G     [CMAX][D]
  static constexpr int oAkk = oG + kSimtCMax * D;     // eta_j k_i.k_j, j < i  [CMAX][CMAX]
  static constexpr int oAqk = oAkk + kSimtCMax * kSimtCMax;  // eta_j q_i.k_j, j <= i
  static constexpr int oEta = oAqk + kSimtCMax * kSimtCMax;
  static constexpr int oGate = oEta + kSimtCMax;
  static constexpr int oGam = oGate + kSimtCMax;
  static constexpr int oBet = oGam + D;
  static constexpr int total = oBet + D;
  static constexpr size_t bytes = sizeof(float) * total;
};

// Copy n rows of D elements (row stride D in global memory) into shared
// memory as fp32 rows of stride `stride`, with 16-byte loads.
template <int D, int NT, typename InT>
__device__ __forceinline__ void simt_load_rows(const InT* __restrict__ src, int n,
                                               float* dst, int stride, int tid) {
  constexpr int VW = Vec16<InT>::N;
  constexpr int VPR = D / VW;
  const int nv = n * VPR;
  for (int idx = tid; idx < nv; idx += NT) {
    const int row = idx / VPR;
    const int col = (idx - row * VPR) * VW;
    float tmp[VW];
    Vec16<InT>::load(src + (size_t)row * D + col, tmp);
#pragma unroll
    for (int u = 0; u < VW; ++u) dst[row * stride + col + u] = tmp[u];
  }
}

// Inner LayerNorm + gradient for token i of the chunk, one warp, lane owns
// features lane, lane + 32, ... Writes G_i to sG[i]. With `correct`, z_i is
// W_s k_i minus the contribution of the earlier tokens of the chunk.
template <int D>
__device__ __forceinline__ void simt_grad_token(int i, bool correct, const float* sZ,
                                                const float* sAkk, float* sG,
                                                const float* sV, const float* sGam,
                                                const float* sBet, float eps, int lnjac,
                                                int no_ln, int lane) {
  constexpr int EPL = (D + 31) / 32;
  float z[EPL], vv[EPL], G[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int f = lane + 32 * e;
    float zz = 0.f, v = 0.f;
    if (f < D) {
      zz = sZ[i * D + f];
      if (correct) {
        for (int j = 0; j < i; ++j) zz -= sAkk[i * kSimtCMax + j] * sG[j * D + f];
      }
      v = sV[i * D + f];
    }
    z[e] = zz;
    vv[e] = v;
  }
  if (no_ln) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) G[e] = z[e] - vv[e];
  } else {
    const float inv_d = 1.0f / (float)D;
    float s1 = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) s1 += z[e];  // lanes past D hold 0
    const float mu = warp_sum(s1) * inv_d;
    float s2 = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const float dz = (lane + 32 * e < D) ? z[e] - mu : 0.f;
      s2 += dz * dz;
    }
    const float var = warp_sum(s2) * inv_d;
    const float s = sqrtf(var + eps);
    float xh[EPL], gg[EPL];
    float sg = 0.f, sgx = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int f = lane + 32 * e;
      const bool ok = f < D;
      const float gam = ok ? sGam[f] : 0.f;
      const float bet = ok ? sBet[f] : 0.f;
      xh[e] = ok ? (z[e] - mu) / s : 0.f;
      const float err = ok ? gam * xh[e] + bet - vv[e] : 0.f;
      G[e] = err;
      gg[e] = gam * err;
      sg += gg[e];
      sgx += gg[e] * xh[e];
    }
    if (lnjac) {
      const float mg = warp_sum(sg) * inv_d;
      const float mgx = warp_sum(sgx) * inv_d;
#pragma unroll
      for (int e = 0; e < EPL; ++e) G[e] = (gg[e] - mg - xh[e] * mgx) / s;
    }
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int f = lane + 32 * e;
    if (f < D) sG[i * D + f] = G[e];
  }
}

template <int D, typename InT, typename OutT>
__global__ void __launch_bounds__(4 * D) scan_simt_kernel(const ScanParams p) {
  using L = SimtLayout<D>;
  constexpr int NT = L::NT;
  constexpr int KP = L::KP;
  extern __shared__ float smem[];
  float* sW = smem + L::oW;
  float* sK = smem + L::oK;
  float* sQ = smem + L::oQ;
  float* sV = smem + L::oV;
  float* sZ = smem + L::oZ;
  float* sQ0 = smem + L::oQ0;
  float* sG = smem + L::oG;
  float* sAkk = smem + L::oAkk;
  float* sAqk = smem + L::oAqk;
  float* sEta = smem + L::oEta;
  float* sGate = smem + L::oGate;
  float* sGam = smem + L::oGam;
  float* sBet = smem + L::oBet;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const long long bh = blockIdx.x;
  const int bi = (int)(bh / p.H);
  const int h = (int)(bh - (long long)bi * p.H);
  const size_t tok0 = (size_t)bh * p.T;
  const InT* __restrict__ gq = static_cast<const InT*>(p.q) + tok0 * D;
  const InT* __restrict__ gk = static_cast<const InT*>(p.k) + tok0 * D;
  const InT* __restrict__ gv = static_cast<const InT*>(p.v) + tok0 * D;
  const InT* __restrict__ gel = static_cast<const InT*>(p.eta_logit) + tok0;
  const InT* __restrict__ ggl =
      p.gate_logit ? static_cast<const InT*>(p.gate_logit) + tok0 : nullptr;
  OutT* __restrict__ go = static_cast<OutT*>(p.o) + tok0 * D;
  const float* W0 = p.W0 + (size_t)bh * D * D;  // may alias W_T
  float* Wc = p.W_chunks ? p.W_chunks + (size_t)bh * (p.n_mask_chunks + 1) * D * D : nullptr;

  for (int e = tid; e < D * D; e += NT) sW[(e / D) * KP + (e % D)] = W0[e];
  if (tid < D) {
    sGam[tid] = p.no_ln ? 1.f : p.gamma[(size_t)h * D + tid];
    sBet[tid] = p.no_ln ? 0.f : p.beta[(size_t)h * D + tid];
  }
  __syncthreads();

  const float inv_d = 1.0f / (float)D;
  for (int t0 = 0; t0 < p.T; t0 += p.C) {
    const int n = min(p.C, p.T - t0);
    const int mc = t0 / p.b;
    const bool upd = (p.mask == nullptr) || (p.mask[(size_t)bi * p.n_mask_chunks + mc] != 0);
    if (Wc && (t0 % p.b) == 0) {
      float* dst = Wc + (size_t)mc * D * D;
      for (int e = tid; e < D * D; e += NT) dst[e] = sW[(e / D) * KP + (e % D)];
    }
    simt_load_rows<D, NT>(gk + (size_t)t0 * D, n, sK, KP, tid);
    simt_load_rows<D, NT>(gq + (size_t)t0 * D, n, sQ, KP, tid);
    simt_load_rows<D, NT>(gv + (size_t)t0 * D, n, sV, D, tid);
    if (tid < n) {
      sEta[tid] = upd ? sigmoidf_(to_f32(gel[t0 + tid])) * inv_d : 0.f;
      sGate[tid] = ggl ? sigmoidf_(to_f32(ggl[t0 + tid])) : 1.f;
    }
    __syncthreads();

    // W_s K^T and W_s Q^T: thread owns output feature r for tokens i = g, g + NT/D, ...
    {
      const int r = tid % D;
      for (int i = tid / D; i < n; i += NT / D) {
        float az = 0.f, aq = 0.f;
#pragma unroll 8
        for (int c = 0; c < D; ++c) {
          const float w = sW[r * KP + c];
          az = fmaf(w, sK[i * KP + c], az);
          aq = fmaf(w, sQ[i * KP + c], aq);
        }
        sZ[i * D + r] = az;
        sQ0[i * D + r] = aq;
      }
    }
    // causal Gram terms of the chunk
    for (int e = tid; e < n * n; e += NT) {
      const int i = e / n;
      const int j = e - i * n;
      float akk = 0.f, aqk = 0.f;
      if (j <= i) {
#pragma unroll 8
        for (int c = 0; c < D; ++c) {
          const float kj = sK[j * KP + c];
          akk = fmaf(sK[i * KP + c], kj, akk);
          aqk = fmaf(sQ[i * KP + c], kj, aqk);
        }
      }
      sAkk[i * kSimtCMax + j] = (j < i) ? sEta[j] * akk : 0.f;
      sAqk[i * kSimtCMax + j] = (j <= i) ? sEta[j] * aqk : 0.f;
    }
    __syncthreads();

    // inner gradients: a sequential chain (per-token) or independent (mini-batch)
    if (!p.minibatch) {
      if (warp == 0) {
        for (int i = 0; i < n; ++i) {
          simt_grad_token<D>(i, true, sZ, sAkk, sG, sV, sGam, sBet, p.eps, p.lnjac, p.no_ln, lane);
          __syncwarp();
        }
      }
    } else {
      for (int i = warp; i < n; i += L::NW)
        simt_grad_token<D>(i, false, sZ, sAkk, sG, sV, sGam, sBet, p.eps, p.lnjac, p.no_ln, lane);
    }
    __syncthreads();

    // W_e = W_s - sum_j eta_j G_j k_j^T (skipped chunks leave W untouched)
    if (upd) {
      for (int e = tid; e < D * D; e += NT) {
        const int r = e / D;
        const int c = e - r * D;
        float acc = sW[r * KP + c];
        for (int j = 0; j < n; ++j) acc -= (sEta[j] * sG[j * D + r]) * sK[j * KP + c];
        sW[r * KP + c] = acc;
      }
    }
    // o_i = gate_i (W_s q_i - sum_{j<=i} eta_j (k_j . q_i) G_j)
    for (int e = tid; e < n * D; e += NT) {
      const int i = e / D;
      const int r = e - i * D;
      float acc = sQ0[i * D + r];
      for (int j = 0; j <= i; ++j) acc -= sAqk[i * kSimtCMax + j] * sG[j * D + r];
      go[(size_t)(t0 + i) * D + r] = from_f32<OutT>(sGate[i] * acc);
    }
    __syncthreads();
  }

  if (Wc) {
    float* dst = Wc + (size_t)p.n_mask_chunks * D * D;
    for (int e = tid; e < D * D; e += NT) dst[e] = sW[(e / D) * KP + (e % D)];
  }
  float* WT = p.W_T + (size_t)bh * D * D;
  for (int e = tid; e < D * D; e += NT) WT[e] = sW[(e / D) * KP + (e % D)];
}

}  // namespace ttt
