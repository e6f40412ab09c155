// CUDA-core (fp32) scan kernel: exact per-token recurrence and mini-batch dual
// form, fp32 or bf16 inputs, fp32 or bf16 outputs, d in {16, 64}.
//
// One CTA per (batch row, head) keeps W in fp32 for the whole sequence. Tokens
// run in chunks of C <= 16 through the exact chunk identity of the per-token
// recurrence ("Edifice.Recurrent.TTT", Equations (TTT-Linear)): with W_s the
// state at the chunk start and a_mj = eta_j (k_m . k_j),
//
//     z_m = W_{m-1} k_m = W_s k_m - sum_{j<m} a_mj G_j
//     o_i = W_i q_i     = W_s q_i - sum_{j<=i} eta_j (k_j . q_i) G_j
//     W_e = W_s - sum_j eta_j G_j k_j^T .
//
// Mini-batch mode (PonderTTT, dual-form updates) is the same chunk step
// without the in-chunk correction of z_m (C = b).
//
// Warp roles. The last warp is the gradient CHAIN: for chunk c it walks the
// tokens in order, each needing one LayerNorm reduction (all moments of one
// token in a single butterfly) and a right-looking update of the pending z's.
// The other 2d threads are BULK threads that own W in registers (thread t:
// row r = t % d, columns [d/2 * (t / d), +d/2)) and, while the chain works on
// chunk c, do everything that does not wait for it:
//     W_{s,c} = W_{s,c-1} - eta G_{c-1} K_{c-1}      (rank-C update)
//     Q0_c = Q_c W_{s,c}^T,   P_{c+1} = K_{c+1} W_{s,c}^T
//     O_{c-1} = gate (Q0_{c-1} - S_{c-1} G_{c-1})      (outputs of chunk c-1)
//     S_c = tril(Q_c K_c^T) eta, X_{c+1} = K_{c+1} K_c^T eta, A_{c+1} = strict tril(K K^T) eta
//     cp.async prefetch of the inputs of chunks c+1 / c+2.
// After both finish, the bulk threads apply the look-ahead correction
//     z-input of chunk c+1:  Zpre_{c+1} = P_{c+1} - X_{c+1} G_c
// (because W_{s,c+1} = W_{s,c} - eta G_c K_c), and the next chunk starts.
#pragma once

#include "common.cuh"

namespace ttt {

constexpr int kC = 16;  // largest chunk of the CUDA-core kernel

// IH = 2 doubles the bulk warps (8 at d = 64), so every SM sub-partition runs
// two of them; used when heads are few.
//
// W lives in the bulk threads' registers as RB x CBW blocks: thread
// (row group rg, column group cg) holds rows RB rg .. + RB - 1, columns
// CBW cg .. + CBW - 1. The CG = D / CBW threads of a row group are consecutive
// lanes, so a product's partial sums over column groups finish with a lane
// reduce-scatter, and every input-row segment a thread loads feeds RB rows.
template <int D, typename InT, int IH = 1>
struct PipeLayout {
  static constexpr int NBT = 2 * D * IH;     // bulk threads
  static constexpr int NT = NBT + 32;        // + the chain warp
  static constexpr int KH = D / 2;           // Gram column half
  static constexpr int NG = NBT / 32;        // bulk warps
  static constexpr int CBW = D >= 64 ? 8 : 4;          // columns of a W block
  static constexpr int CG = D / CBW;                   // column groups (lanes per row group)
  static constexpr int RB = D * D / (NBT * CBW);       // rows of a W block
  static_assert(RB * CBW * NBT == D * D && RB >= 2 && 32 % CG == 0, "W block geometry");
  static constexpr int ELT = (int)sizeof(InT);
  static constexpr int ROWB = D * ELT + 16;  // padded row of an input tile (bytes)
  static constexpr int TILE = kC * ROWB;
  // byte offsets into dynamic shared memory
  static constexpr int oK = 0;                         // K tiles, ring of 4
  static constexpr int oQ = oK + 4 * TILE;             // Q tiles, ring of 2
  static constexpr int oV = oQ + 2 * TILE;             // V tiles, ring of 2
  static constexpr int oZ = oV + 2 * TILE;             // P / Zpre   [2][kC][D] f32
  static constexpr int oG = oZ + 2 * kC * D * 4;       // G          [2][kC][D]
  static constexpr int oQ0 = oG + 2 * kC * D * 4;      // Q0         [2][kC][D]
  static constexpr int oA = oQ0 + 2 * kC * D * 4;      // in-chunk K Gram [2][kC][kC]
  static constexpr int oS = oA + 2 * kC * kC * 4;      // Q K Gram   [2][kC][kC]
  static constexpr int oX = oS + 2 * kC * kC * 4;      // cross Gram [kC][kC]
  static constexpr int oEta = oX + kC * kC * 4;        // eta        [4][kC]
  static constexpr int oGate = oEta + 4 * kC * 4;      // gate       [4][kC]
  static constexpr int oMu = oGate + 4 * kC * 4;       // mean of Zpre rows [2][kC]
  static constexpr int oMG = oMu + 2 * kC * 4;         // mean of G rows    [2][kC]
  static constexpr int oFlag = oMG + 2 * kC * 4;       // chunk updates?    [4] int
  static constexpr int bytes = oFlag + 16;
};

__device__ __forceinline__ void bulk_barrier(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int src_bytes) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// 8 consecutive elements of a shared-memory tile row, widened to fp32.
__device__ __forceinline__ void lds8(const unsigned char* p, float (&x)[8], float) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 16);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void lds8(const unsigned char* p, float (&x)[8], __nv_bfloat16) {
  const uint4 a = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ float lds1(const unsigned char* p, float) {
  return *reinterpret_cast<const float*>(p);
}
__device__ __forceinline__ float lds1(const unsigned char* p, __nv_bfloat16) {
  return __uint_as_float((uint32_t)(*reinterpret_cast<const unsigned short*>(p)) << 16);
}

// Asynchronous copy of rows [t0, t0 + n) of a [T][D] head array into a tile
// (rows >= n are zero-filled).
template <int D, typename InT>
__device__ __forceinline__ void tile_load(unsigned char* tile, const InT* src, int t0, int n,
                                          int tid, int nthreads) {
  using L = PipeLayout<D, InT, 1>;
  constexpr int CPR = D * L::ELT / 16;  // 16-byte pieces per row
  for (int idx = tid; idx < kC * CPR; idx += nthreads) {
    const int row = idx / CPR;
    const int piece = idx - row * CPR;
    const bool ok = row < n;
    const InT* g = src + (size_t)(t0 + (ok ? row : 0)) * D + piece * (16 / L::ELT);
    cp_async16(tile + row * L::ROWB + piece * 16, g, ok ? 16 : 0);
  }
}

// SiLU, in place, on the pieces of a tile that tile_load() with the same
// arguments copied for this thread (the `:mlp` variant's keys and queries).
// Call after this thread's copies completed (cp.async.wait) and before the
// barrier that publishes the tile; fp32 tiles only, so every element keeps
// full precision. Rows past n were zero-filled and SiLU(0) = 0.
template <int D, typename InT>
__device__ __forceinline__ void tile_silu(unsigned char* tile, int n, int tid, int nthreads) {
  if constexpr (sizeof(InT) == 4) {
    using L = PipeLayout<D, InT, 1>;
    constexpr int CPR = D * L::ELT / 16;
    for (int idx = tid; idx < kC * CPR; idx += nthreads) {
      const int row = idx / CPR;
      if (row >= n) continue;
      float4* x = reinterpret_cast<float4*>(tile + row * L::ROWB + (idx - row * CPR) * 16);
      float4 v = *x;
      v.x = siluf_(v.x); v.y = siluf_(v.y); v.z = siluf_(v.z); v.w = siluf_(v.w);
      *x = v;
    }
  }
}

// Four consecutive elements of a shared-memory tile row (16 bytes of fp32 or
// 8 bytes of bf16), widened to two fp32 pairs.
template <typename InT>
struct Unit;
template <>
struct Unit<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void ld(const unsigned char* p, float2 (&x)[2]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    x[0] = make_float2(a.x, a.y);
    x[1] = make_float2(a.z, a.w);
  }
};
template <>
struct Unit<__nv_bfloat16> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void ld(const unsigned char* p, float2 (&x)[2]) {
    const uint2 a = *reinterpret_cast<const uint2*>(p);
    x[0] = make_float2(__uint_as_float(a.x << 16), __uint_as_float(a.x & 0xffff0000u));
    x[1] = make_float2(__uint_as_float(a.y << 16), __uint_as_float(a.y & 0xffff0000u));
  }
};

__device__ __forceinline__ float2 dup2(float x) { return make_float2(x, x); }

// Reduce-scatter of V partial sums over the G lanes of one lane group (lane
// bits 0 .. log2 G - 1): each step exchanges half of the values still held
// (S of them) across lane bit B. Afterwards lane g holds the full sums of
// values g (V/G) .. g (V/G) + V/G - 1 in a[0 .. V/G).
template <int V, int S, int B>
__device__ __forceinline__ void reduce_scatter_step(float (&a)[V], int g) {
  if constexpr (B >= 1) {
    const bool up = g & B;
#pragma unroll
    for (int j = 0; j < S; ++j) {
      const float send = up ? a[j] : a[j + S];
      const float keep = up ? a[j + S] : a[j];
      a[j] = keep + __shfl_xor_sync(0xffffffffu, send, B);
    }
    reduce_scatter_step<V, S / 2, B / 2>(a, g);
  }
}
template <int V, int G>
__device__ __forceinline__ void reduce_scatter_lanes(float (&a)[V], int g) {
  reduce_scatter_step<V, V / 2, G / 2>(a, g);
}

// A bulk thread's block of W (see PipeLayout) and the work done on it.
template <int D, typename InT, int IH>
struct WBlock {
  using L = PipeLayout<D, InT, IH>;
  static constexpr int RB = L::RB, CBW = L::CBW, CG = L::CG, NU = CBW / 4;
  float2 w[RB][CBW / 2];  // w[rb][2 u + t]: columns col(u) + 2 t, + 1 of row row0 + rb
  int row0, cg, swap;

  __device__ __forceinline__ void init(int tid) {
    cg = tid % CG;
    row0 = (tid / CG) * RB;
    // fp32 tiles with two units per block: the upper half of the column groups
    // takes its units in swapped order so the broadcast addresses of one load
    // fall in disjoint banks
    swap = (L::ELT == 4 && NU == 2 && cg >= CG / 2) ? 1 : 0;
  }
  __device__ __forceinline__ int col(int u) const { return cg * CBW + 4 * (u ^ swap); }

  __device__ __forceinline__ void load(const float* Wh) {
#pragma unroll
    for (int rb = 0; rb < RB; ++rb)
#pragma unroll
      for (int u = 0; u < NU; ++u) {
        const float4 x = *reinterpret_cast<const float4*>(Wh + (size_t)(row0 + rb) * D + col(u));
        w[rb][2 * u] = make_float2(x.x, x.y);
        w[rb][2 * u + 1] = make_float2(x.z, x.w);
      }
  }
  __device__ __forceinline__ void store(float* Wh) const {
#pragma unroll
    for (int rb = 0; rb < RB; ++rb)
#pragma unroll
      for (int u = 0; u < NU; ++u)
        *reinterpret_cast<float4*>(Wh + (size_t)(row0 + rb) * D + col(u)) =
            make_float4(w[rb][2 * u].x, w[rb][2 * u].y, w[rb][2 * u + 1].x, w[rb][2 * u + 1].y);
  }
  // W -= sum_{j < n} eta_j G_j k_j^T over the rows of tile Kt (rows of G past
  // n may hold anything, so their scale is selected away, not multiplied).
  __device__ __forceinline__ void rank_update(const unsigned char* Kt, const float* Gp,
                                              const float* et, int n) {
#pragma unroll
    for (int j = 0; j < kC; ++j) {
      float g[RB];
      if constexpr (RB == 4) {
        const float4 g4 = *reinterpret_cast<const float4*>(Gp + j * D + row0);
        g[0] = g4.x; g[1] = g4.y; g[2] = g4.z; g[3] = g4.w;
      } else {
        const float2 g2 = *reinterpret_cast<const float2*>(Gp + j * D + row0);
        g[0] = g2.x; g[1] = g2.y;
      }
      const float e = j < n ? -et[j] : 0.f;
      float2 x[NU][2];
#pragma unroll
      for (int u = 0; u < NU; ++u) Unit<InT>::ld(Kt + j * L::ROWB + col(u) * L::ELT, x[u]);
#pragma unroll
      for (int rb = 0; rb < RB; ++rb) {
        const float2 s = dup2(j < n ? e * g[rb] : 0.f);
#pragma unroll
        for (int u = 0; u < NU; ++u) {
          w[rb][2 * u] = __ffma2_rn(s, x[u][0], w[rb][2 * u]);
          w[rb][2 * u + 1] = __ffma2_rn(s, x[u][1], w[rb][2 * u + 1]);
        }
      }
    }
  }
  // (W x_t)_row for the kC rows x_t of tile R and this block's rows, in batches
  // of 8 tokens finished by a reduce-scatter over the CG lanes; stored as
  // out[t][row] (PTS == 0) or transposed, out[row][t] with token stride PTS.
  template <int PTS = 0>
  __device__ __forceinline__ void products(const unsigned char* R, float* out) const {
    constexpr int V = RB * 8, PER = V / CG;
#pragma unroll
    for (int t0 = 0; t0 < kC; t0 += 8) {
      float2 x[8][NU][2];
#pragma unroll
      for (int b = 0; b < 8; ++b)
#pragma unroll
        for (int u = 0; u < NU; ++u) Unit<InT>::ld(R + (t0 + b) * L::ROWB + col(u) * L::ELT, x[b][u]);
      float acc[V];
#pragma unroll
      for (int rb = 0; rb < RB; ++rb)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          float2 a = __fmul2_rn(w[rb][0], x[b][0][0]);
          a = __ffma2_rn(w[rb][1], x[b][0][1], a);
#pragma unroll
          for (int u = 1; u < NU; ++u) {
            a = __ffma2_rn(w[rb][2 * u], x[b][u][0], a);
            a = __ffma2_rn(w[rb][2 * u + 1], x[b][u][1], a);
          }
          acc[rb * 8 + b] = a.x + a.y;
        }
      reduce_scatter_lanes<V, CG>(acc, cg);
      // lane cg now holds values cg * PER .. + PER - 1: one row, PER tokens
      const int i0 = cg * PER, rb = i0 / 8, tb = i0 % 8;
      if constexpr (PTS == 0) {
#pragma unroll
        for (int u = 0; u < PER; ++u) out[(t0 + tb + u) * D + row0 + rb] = acc[u];
      } else {
#pragma unroll
        for (int u = 0; u < PER; ++u) out[(row0 + rb) * PTS + t0 + tb + u] = acc[u];
      }
    }
  }
};

template <int N>
__device__ __forceinline__ void butterfly(float (&v)[N]) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], off);
  }
}

// Gradient chain of one chunk of the one-CTA-per-head kernel (one warp).
// (The cluster kernel uses the Chain struct below, which also applies the
// next chunk's correction; here that stays a separate phase, which keeps this
// kernel's registers low enough for three CTAs per SM when heads are many.)
// GM: 0 = simplified (G = err),
// 1 = through the LayerNorm Jacobian, 2 = no LayerNorm (G = z - v),
// 3 = the ablation gradient (the Jacobian applied to -gamma * v, the
// prediction removed; "Error Correction in Trained TTT Layers", Abstract),
// 4 = the ablation together with the norm of the GM 1 gradient: rescaled per
// token to that norm when nmatch, and both norms (full, ablated before any
// rescaling) written to gnorm[2 i], gnorm[2 i + 1] when gnorm is not null.
// Both Jacobian forms (1, 3, 4) give G a zero feature mean.
// Reads Zpre (z before in-chunk corrections), A (eta_j k_m.k_j, j < m), V,
// mu0 (mean of each Zpre row); writes G and, for GM 0, the mean of each G row.
template <int D, typename InT, bool MINIB, int GM>
__device__ __forceinline__ void chain_chunk(int n, const float* __restrict__ Z,
                                            const float* __restrict__ A,
                                            const unsigned char* __restrict__ V,
                                            const float* __restrict__ mu0, float* __restrict__ Gout,
                                            float* __restrict__ mGout, float eps,
                                            const float (&gam)[(D + 31) / 32],
                                            const float (&bet)[(D + 31) / 32], float Sgb, float Sb,
                                            int lane, float* __restrict__ gnorm = nullptr,
                                            bool nmatch = true) {
  using L = PipeLayout<D, InT>;
  constexpr int EPL = (D + 31) / 32;
  const float inv_d = 1.0f / (float)D;
  float zr[kC][EPL];
  float mup[kC];
#pragma unroll
  for (int i = 0; i < kC; ++i) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int f = lane + 32 * e;
      zr[i][e] = (i < n && f < D) ? Z[i * D + f] : 0.f;
    }
    mup[i] = (i < n) ? mu0[i] : 0.f;
  }
#pragma unroll
  for (int i = 0; i < kC; ++i) {
    if (i >= n) break;
    float v[EPL], G[EPL];
    float mG = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int f = lane + 32 * e;
      v[e] = (f < D) ? lds1(V + i * L::ROWB + f * L::ELT, InT()) : 0.f;
    }
    if (GM == 2) {
#pragma unroll
      for (int e = 0; e < EPL; ++e) G[e] = zr[i][e] - v[e];
    } else {
      float y[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) y[e] = (lane + 32 * e < D) ? zr[i][e] - mup[i] : 0.f;
      if (GM == 3) {
        // g = -gamma v: sum y^2, sum gamma v, sum gamma v y
        float m[3] = {0.f, 0.f, 0.f};
        float gv[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          gv[e] = gam[e] * v[e];
          m[0] = fmaf(y[e], y[e], m[0]);
          m[1] += gv[e];
          m[2] = fmaf(gv[e], y[e], m[2]);
        }
        butterfly<3>(m);
        const float rs = rsqrtf(fmaf(m[0], inv_d, eps));
        const float a = m[1] * inv_d, bq = rs * rs * rs * m[2] * inv_d;
#pragma unroll
        for (int e = 0; e < EPL; ++e) G[e] = fmaf(bq, y[e], rs * (a - gv[e]));
      } else if (GM == 4) {
        // both forms from one butterfly: the GM 1 moments plus sum gamma v y
        float m[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float w[EPL], g2[EPL], gv[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          g2[e] = gam[e] * gam[e];
          w[e] = gam[e] * (bet[e] - v[e]);
          gv[e] = gam[e] * v[e];
          m[0] = fmaf(y[e], y[e], m[0]);
          m[1] = fmaf(g2[e], y[e], m[1]);
          m[2] = fmaf(g2[e] * y[e], y[e], m[2]);
          m[3] = fmaf(w[e], y[e], m[3]);
          m[4] = fmaf(gam[e], v[e], m[4]);
          m[5] = fmaf(gv[e], y[e], m[5]);
        }
        butterfly<6>(m);
        const float rs = rsqrtf(fmaf(m[0], inv_d, eps));
        const float mg = (rs * m[1] + Sgb - m[4]) * inv_d;
        const float mgx = rs * (rs * m[2] + m[3]) * inv_d;
        const float rs2 = rs * rs;
        const float a = m[4] * inv_d, bq = rs2 * rs * m[5] * inv_d;
        float Gf[EPL], nrm[2] = {0.f, 0.f};
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          Gf[e] = rs2 * (g2[e] - mgx) * y[e] + rs * (w[e] - mg);
          G[e] = fmaf(bq, y[e], rs * (a - gv[e]));
          if (lane + 32 * e < D) {  // lanes past the features (d = 16) hold no feature
            nrm[0] = fmaf(Gf[e], Gf[e], nrm[0]);
            nrm[1] = fmaf(G[e], G[e], nrm[1]);
          }
        }
        butterfly<2>(nrm);
        if (gnorm != nullptr && lane == 0) {
          gnorm[2 * i] = sqrtf(nrm[0]);
          gnorm[2 * i + 1] = sqrtf(nrm[1]);
        }
        const float scale = !nmatch ? 1.f : (nrm[1] > 0.f ? sqrtf(nrm[0] / nrm[1]) : 0.f);
#pragma unroll
        for (int e = 0; e < EPL; ++e) G[e] *= scale;
      } else if (GM == 1) {
        // moments of y: sum y^2, sum g2 y, sum g2 y^2, sum w y, sum gamma v
        float m[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
        float w[EPL], g2[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          g2[e] = gam[e] * gam[e];
          w[e] = gam[e] * (bet[e] - v[e]);
          m[0] = fmaf(y[e], y[e], m[0]);
          m[1] = fmaf(g2[e], y[e], m[1]);
          m[2] = fmaf(g2[e] * y[e], y[e], m[2]);
          m[3] = fmaf(w[e], y[e], m[3]);
          m[4] = fmaf(gam[e], v[e], m[4]);
        }
        butterfly<5>(m);
        const float rs = rsqrtf(fmaf(m[0], inv_d, eps));
        const float mg = (rs * m[1] + Sgb - m[4]) * inv_d;
        const float mgx = rs * (rs * m[2] + m[3]) * inv_d;
        const float rs2 = rs * rs;
#pragma unroll
        for (int e = 0; e < EPL; ++e) G[e] = rs2 * (g2[e] - mgx) * y[e] + rs * (w[e] - mg);
      } else {
        float m[3] = {0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          m[0] = fmaf(y[e], y[e], m[0]);
          m[1] = fmaf(gam[e], y[e], m[1]);
          m[2] += v[e];
        }
        butterfly<3>(m);
        const float rs = rsqrtf(fmaf(m[0], inv_d, eps));
#pragma unroll
        for (int e = 0; e < EPL; ++e) G[e] = gam[e] * rs * y[e] + bet[e] - v[e];
        mG = (rs * m[1] + Sb - m[2]) * inv_d;
      }
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int f = lane + 32 * e;
      if (f < D) Gout[i * D + f] = G[e];
    }
    if (GM == 0 && lane == 0) mGout[i] = mG;
    if (!MINIB) {
#pragma unroll
      for (int m2 = i + 1; m2 < kC; ++m2) {
        const float a = A[m2 * kC + i];
#pragma unroll
        for (int e = 0; e < EPL; ++e) zr[m2][e] = fmaf(-a, G[e], zr[m2][e]);
        if (GM == 0) mup[m2] = fmaf(-a, mG, mup[m2]);
      }
    }
  }
  if (GM != 0 && lane < kC) mGout[lane] = 0.f;
}

// Dot products of left rows with one right row per lane pair (16 rows x 2
// column halves); returns eta-weighted entries through `emit(i, j, dot)`.
template <int D, typename InT, int IH, typename Emit>
__device__ __forceinline__ void bulk_gram(const unsigned char* right, const unsigned char* left0,
                                          const unsigned char* left1, int nleft, int tid,
                                          Emit emit) {
  using L = PipeLayout<D, InT, IH>;
  constexpr int KH = L::KH;
  const int j = tid & 15;
  const int kq = (tid >> 4) & 1;
  const int grp = tid >> 5;
  float rk[KH];
#pragma unroll
  for (int k = 0; k < KH; k += 8) {
    float x[8];
    lds8(right + j * L::ROWB + (kq * KH + k) * L::ELT, x, InT());
#pragma unroll
    for (int u = 0; u < 8; ++u) rk[k + u] = x[u];
  }
  // rows s = grp, grp + NG, ... taken two at a time (nleft / NG is even)
  for (int s = grp; s < nleft; s += 2 * L::NG) {
    const int s2 = s + L::NG;
    const unsigned char* row0 = (s < kC ? left0 : left1) + (s & (kC - 1)) * L::ROWB +
                                kq * KH * L::ELT;
    const unsigned char* row1 = (s2 < kC ? left0 : left1) + (s2 & (kC - 1)) * L::ROWB +
                                kq * KH * L::ELT;
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
    for (int k = 0; k < KH; k += 8) {
      float x[8], y[8];
      lds8(row0 + k * L::ELT, x, InT());
      lds8(row1 + k * L::ELT, y, InT());
#pragma unroll
      for (int u = 0; u < 8; u += 2) {
        a0 = fmaf(rk[k + u], x[u], a0);
        a1 = fmaf(rk[k + u + 1], x[u + 1], a1);
        b0 = fmaf(rk[k + u], y[u], b0);
        b1 = fmaf(rk[k + u + 1], y[u + 1], b1);
      }
    }
    float acc = a0 + a1, acc2 = b0 + b1;
    acc += __shfl_xor_sync(0xffffffffu, acc, 16);
    acc2 += __shfl_xor_sync(0xffffffffu, acc2, 16);
    if (kq == 0) {
      emit(s, j, acc);
      emit(s2, j, acc2);
    }
  }
}

// mean of each of the kC rows of a [kC][D] fp32 tile: 8 lanes per row,
// each summing a strided eighth (conflict-free), then a 3-level shuffle.
template <int D>
__device__ __forceinline__ void row_means(const float* Z, float* out, int tid, int nthreads) {
  for (int base = 0; base < kC * 8; base += nthreads) {
    const int idx = base + tid;
    const int m = idx >> 3;
    const int part = idx & 7;
    float s = 0.f;
    if (m < kC) {
#pragma unroll
      for (int f = part; f < D; f += 8) s += Z[m * D + f];
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    if (m < kC && part == 0) out[m] = s * (1.0f / (float)D);
  }
}

// Warp-wide sums of five values; the adds run as pairs.
__device__ __forceinline__ void butterfly5(float (&m)[5]) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    float r[5];
#pragma unroll
    for (int i = 0; i < 5; ++i) r[i] = __shfl_xor_sync(0xffffffffu, m[i], off);
    const float2 a = __fadd2_rn(make_float2(m[0], m[1]), make_float2(r[0], r[1]));
    const float2 b = __fadd2_rn(make_float2(m[2], m[3]), make_float2(r[2], r[3]));
    m[0] = a.x; m[1] = a.y; m[2] = b.x; m[3] = b.y;
    m[4] += r[4];
  }
}

// The sequential gradient chain of one head, shared by the CUDA-core scan
// kernels: one warp, lane l holding features l + 32 e (e < EPL; at d = 16
// lanes 16-31 hold none). For chunk c, z of its tokens is P_c (read from
// PT[feature][token], token stride PTS) plus the correction the previous
// chunk left in `cpr`. Per token i the LayerNorm gradient G_i (GM: 0
// simplified, 1 LN Jacobian, 2 no LayerNorm, 3 ablation, 4 ablation with
// per-token norm matching) goes to Gc[i][feature] and is applied at once to
// the later tokens of the chunk through A^T (per-token mode only) and to every
// token of the next chunk through X^T, accumulated in `cpr`. Token pairs are
// updated with paired FMAs, and tokens past n are masked to G = 0 so the
// unrolled token loop has no branch. The LayerNorm shift is the feature mean
// of z at the chunk start (exact for the Jacobian forms, whose G has zero
// mean; tracked through the chunk for the simplified gradient).
template <int D, typename InT, bool MINIB, int GM, int PTS>
struct Chain {
  static constexpr int EPL = (D + 31) / 32;
  static constexpr int NP = kC / 2;
  static constexpr int ROWB = D * (int)sizeof(InT) + 16;  // V tile row, as the kernels' tiles
  float gam[EPL], bet[EPL], g2c[EPL], gbc[EPL];
  float Sgb, Sb;
  float2 cpr[NP][EPL];

  __device__ __forceinline__ void init(const float* gamma_h, const float* beta_h, bool no_ln,
                                       int lane) {
    float sgb = 0.f, sb = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int f = lane + 32 * e;
      gam[e] = (f < D && !no_ln) ? gamma_h[f] : (f < D ? 1.f : 0.f);
      bet[e] = (f < D && !no_ln) ? beta_h[f] : 0.f;
      g2c[e] = gam[e] * gam[e];
      gbc[e] = gam[e] * bet[e];
      sgb = fmaf(gam[e], bet[e], sgb);
      sb += bet[e];
    }
    float s2[2] = {sgb, sb};
    butterfly<2>(s2);
    Sgb = s2[0];
    Sb = s2[1];
    reset();
  }
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int pp = 0; pp < NP; ++pp)
#pragma unroll
      for (int e = 0; e < EPL; ++e) cpr[pp][e] = make_float2(0.f, 0.f);
  }

  __device__ __forceinline__ void run(int n, const float* PT, const float* AT, const float* XT,
                                      const unsigned char* Vt, float* Gc, float eps, int lane) {
    const float inv_d = 1.0f / (float)D;
    float2 zp[NP][EPL];  // z of token pairs (2 pp, 2 pp + 1)
    float2 mp[NP];       // their LayerNorm shift
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int f = lane + 32 * e;
      const float4* row = reinterpret_cast<const float4*>(PT + (f < D ? f : 0) * PTS);
#pragma unroll
      for (int m4 = 0; m4 < kC / 4; ++m4) {
        float4 x = row[m4];
        if (f >= D) x = make_float4(0.f, 0.f, 0.f, 0.f);
        zp[2 * m4][e] = __fadd2_rn(make_float2(x.x, x.y), cpr[2 * m4][e]);
        zp[2 * m4 + 1][e] = __fadd2_rn(make_float2(x.z, x.w), cpr[2 * m4 + 1][e]);
      }
    }
    reset();
    if (GM != 2) {
      // feature means of the kC rows of z: reduce-scatter over the lanes, after
      // which lanes 2m and 2m + 1 hold token m's sum
      float sm[kC];
#pragma unroll
      for (int pp = 0; pp < NP; ++pp) {
        float2 t = zp[pp][0];
#pragma unroll
        for (int e = 1; e < EPL; ++e) t = __fadd2_rn(t, zp[pp][e]);
        sm[2 * pp] = t.x;
        sm[2 * pp + 1] = t.y;
      }
      reduce_scatter_step<kC, kC / 2, 16>(sm, lane);
      const float mrow = (sm[0] + __shfl_xor_sync(0xffffffffu, sm[0], 1)) * inv_d;
#pragma unroll
      for (int pp = 0; pp < NP; ++pp)
        mp[pp] = make_float2(__shfl_sync(0xffffffffu, mrow, 4 * pp),
                             __shfl_sync(0xffffffffu, mrow, 4 * pp + 2));
    }
#pragma unroll
    for (int i = 0; i < kC; ++i) {
      const int pi = i / 2;
      const bool hi = i & 1;
      float v[EPL], Gv[EPL], zi[EPL];
      bool fv[EPL];
      float mG = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const int f = lane + 32 * e;
        fv[e] = f < D;
        v[e] = fv[e] ? lds1(Vt + i * ROWB + f * (int)sizeof(InT), InT()) : 0.f;
        zi[e] = hi ? zp[pi][e].y : zp[pi][e].x;
      }
      if (GM == 2) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) Gv[e] = zi[e] - v[e];
      } else {
        const float mu = hi ? mp[pi].y : mp[pi].x;
        float y[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) y[e] = fv[e] ? zi[e] - mu : 0.f;
        if (GM == 1) {
          // moments of y: sum y^2, sum g2 y, sum g2 y^2, sum w y, sum gamma v
          float m5[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
          float w[EPL];
#pragma unroll
          for (int e = 0; e < EPL; ++e) {
            w[e] = fmaf(-gam[e], v[e], gbc[e]);
            const float gy = g2c[e] * y[e];
            m5[0] = fmaf(y[e], y[e], m5[0]);
            m5[1] += gy;
            m5[2] = fmaf(gy, y[e], m5[2]);
            m5[3] = fmaf(w[e], y[e], m5[3]);
            m5[4] = fmaf(gam[e], v[e], m5[4]);
          }
          butterfly5(m5);
          const float rs = rsqrtf(fmaf(m5[0], inv_d, eps));
          const float mg = (rs * m5[1] + Sgb - m5[4]) * inv_d;
          const float mgx = rs * (rs * m5[2] + m5[3]) * inv_d;
          const float rs2 = rs * rs;
#pragma unroll
          for (int e = 0; e < EPL; ++e) Gv[e] = rs2 * (g2c[e] - mgx) * y[e] + rs * (w[e] - mg);
        } else if (GM == 3) {
          // g = -gamma v: sum y^2, sum gamma v, sum gamma v y
          float m[3] = {0.f, 0.f, 0.f};
          float gv[EPL];
#pragma unroll
          for (int e = 0; e < EPL; ++e) {
            gv[e] = gam[e] * v[e];
            m[0] = fmaf(y[e], y[e], m[0]);
            m[1] += gv[e];
            m[2] = fmaf(gv[e], y[e], m[2]);
          }
          butterfly<3>(m);
          const float rs = rsqrtf(fmaf(m[0], inv_d, eps));
          const float a = m[1] * inv_d, bq = rs * rs * rs * m[2] * inv_d;
#pragma unroll
          for (int e = 0; e < EPL; ++e) Gv[e] = fmaf(bq, y[e], rs * (a - gv[e]));
        } else if (GM == 4) {
          // both forms from one butterfly (the GM 1 moments and sum gamma v y),
          // then the two norms
          float m[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          float w[EPL], gv[EPL];
#pragma unroll
          for (int e = 0; e < EPL; ++e) {
            w[e] = fmaf(-gam[e], v[e], gbc[e]);
            gv[e] = gam[e] * v[e];
            m[0] = fmaf(y[e], y[e], m[0]);
            m[1] = fmaf(g2c[e], y[e], m[1]);
            m[2] = fmaf(g2c[e] * y[e], y[e], m[2]);
            m[3] = fmaf(w[e], y[e], m[3]);
            m[4] = fmaf(gam[e], v[e], m[4]);
            m[5] = fmaf(gv[e], y[e], m[5]);
          }
          butterfly<6>(m);
          const float rs = rsqrtf(fmaf(m[0], inv_d, eps));
          const float mg = (rs * m[1] + Sgb - m[4]) * inv_d;
          const float mgx = rs * (rs * m[2] + m[3]) * inv_d;
          const float rs2 = rs * rs;
          const float a = m[4] * inv_d, bq = rs2 * rs * m[5] * inv_d;
          float nrm[2] = {0.f, 0.f};
#pragma unroll
          for (int e = 0; e < EPL; ++e) {
            const float gf = rs2 * (g2c[e] - mgx) * y[e] + rs * (w[e] - mg);
            Gv[e] = fmaf(bq, y[e], rs * (a - gv[e]));
            if (fv[e]) {
              nrm[0] = fmaf(gf, gf, nrm[0]);
              nrm[1] = fmaf(Gv[e], Gv[e], nrm[1]);
            }
          }
          butterfly<2>(nrm);
          const float scale = nrm[1] > 0.f ? sqrtf(nrm[0] / nrm[1]) : 0.f;
#pragma unroll
          for (int e = 0; e < EPL; ++e) Gv[e] *= scale;
        } else {
          float m3[3] = {0.f, 0.f, 0.f};
#pragma unroll
          for (int e = 0; e < EPL; ++e) {
            m3[0] = fmaf(y[e], y[e], m3[0]);
            m3[1] = fmaf(gam[e], y[e], m3[1]);
            m3[2] += v[e];
          }
          butterfly<3>(m3);
          const float rs = rsqrtf(fmaf(m3[0], inv_d, eps));
#pragma unroll
          for (int e = 0; e < EPL; ++e) Gv[e] = gam[e] * rs * y[e] + bet[e] - v[e];
          mG = (rs * m3[1] + Sb - m3[2]) * inv_d;
        }
      }
      const bool valid = i < n;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        Gv[e] = (valid && fv[e]) ? Gv[e] : 0.f;
        if (fv[e]) Gc[i * D + lane + 32 * e] = Gv[e];
      }
      mG = valid ? mG : 0.f;
      float2 nG[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) nG[e] = dup2(-Gv[e]);
      if (!MINIB) {
        // into the later tokens of this chunk (A^T row i, zero for m <= i)
#pragma unroll
        for (int m4 = (i + 1) / 4; m4 < kC / 4; ++m4) {
          const float4 a4 = reinterpret_cast<const float4*>(AT + i * kC)[m4];
          const float2 a2[2] = {make_float2(a4.x, a4.y), make_float2(a4.z, a4.w)};
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int pp = 2 * m4 + h2;
            if (pp < (i + 1) / 2) continue;
#pragma unroll
            for (int e = 0; e < EPL; ++e) zp[pp][e] = __ffma2_rn(a2[h2], nG[e], zp[pp][e]);
            if (GM == 0) mp[pp] = __ffma2_rn(a2[h2], dup2(-mG), mp[pp]);
          }
        }
      }
      // into every token of the next chunk (X^T row i)
#pragma unroll
      for (int m4 = 0; m4 < kC / 4; ++m4) {
        const float4 x4 = reinterpret_cast<const float4*>(XT + i * kC)[m4];
        const float2 x2[2] = {make_float2(x4.x, x4.y), make_float2(x4.z, x4.w)};
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
          for (int e = 0; e < EPL; ++e)
            cpr[2 * m4 + h2][e] = __ffma2_rn(x2[h2], nG[e], cpr[2 * m4 + h2][e]);
      }
    }
  }
};

// IH = 1 runs three CTAs per SM when heads are many (the bound caps registers
// accordingly); IH = 2 is the few-heads form, one CTA per SM.
template <int D, typename InT, typename OutT, bool MINIB, int GM, int IH>
__global__ void __launch_bounds__(2 * D * IH + 32, IH == 1 ? 3 : 1)
    scan_simt_kernel(const ScanParams p) {
  using L = PipeLayout<D, InT, IH>;
  constexpr int NBT = L::NBT;
  constexpr int EPL = (D + 31) / 32;
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned char* sK = smem + L::oK;
  unsigned char* sQ = smem + L::oQ;
  unsigned char* sV = smem + L::oV;
  float* sZ = reinterpret_cast<float*>(smem + L::oZ);
  float* sG = reinterpret_cast<float*>(smem + L::oG);
  float* sQ0 = reinterpret_cast<float*>(smem + L::oQ0);
  float* sA = reinterpret_cast<float*>(smem + L::oA);
  float* sS = reinterpret_cast<float*>(smem + L::oS);
  float* sX = reinterpret_cast<float*>(smem + L::oX);
  float* sEta = reinterpret_cast<float*>(smem + L::oEta);
  float* sGate = reinterpret_cast<float*>(smem + L::oGate);
  float* sMu = reinterpret_cast<float*>(smem + L::oMu);
  float* sMG = reinterpret_cast<float*>(smem + L::oMG);
  int* sFlag = reinterpret_cast<int*>(smem + L::oFlag);

  const int tid = threadIdx.x;
  const bool chain = tid >= NBT;
  const int lane = tid & 31;
  const long long bh = blockIdx.x;
  const int bi = (int)(bh / p.H);
  const int h = (int)(bh - (long long)bi * p.H);
  const int T = p.T;
  const int C = p.C;
  const int nc = (T + C - 1) / C;
  const size_t tok0 = (size_t)bh * T;
  const InT* gq = static_cast<const InT*>(p.q) + tok0 * D;
  const InT* gk = static_cast<const InT*>(p.k) + tok0 * D;
  const InT* gv = static_cast<const InT*>(p.v) + tok0 * D;
  const InT* gel = static_cast<const InT*>(p.eta_logit) + tok0;
  // per-token gates (scalars staged with eta) or per-feature gates (read by the
  // threads that write the outputs)
  const InT* ggl = (p.gate_logit && !p.gate_channel) ? static_cast<const InT*>(p.gate_logit) + tok0
                                                      : nullptr;
  const InT* gch = (p.gate_logit && p.gate_channel)
                       ? static_cast<const InT*>(p.gate_logit) + tok0 * D : nullptr;
  OutT* go = static_cast<OutT*>(p.o) + tok0 * D;
  float* Wc = p.W_chunks ? p.W_chunks + (size_t)bh * (p.n_mask_chunks + 1) * D * D : nullptr;
  const float inv_d = 1.0f / (float)D;

  auto chunk_len = [&](int c) { return min(C, T - c * C); };
  // per-token gradient norms of chunk c ([n][2]), or null
  auto gnorm_of = [&](int c) -> float* {
    return p.grad_norms ? p.grad_norms + (tok0 + (size_t)c * C) * 2 : nullptr;
  };
  auto tileK = [&](int c) { return sK + (c & 3) * L::TILE; };
  auto tileQ = [&](int c) { return sQ + (c & 1) * L::TILE; };
  auto tileV = [&](int c) { return sV + (c & 1) * L::TILE; };
  // eta (with the mask folded in), gate and the update flag of chunk c: the raw
  // values are fetched early (issue) and consumed after the bulk work (finish)
  // so the global-load latency stays off the critical path.
  struct RawScalars {
    InT e, g;
    unsigned char m;
  };
  auto issue_scalars = [&](int c) {
    RawScalars s;
    s.e = InT();
    s.g = InT();
    s.m = 1;
    if (tid < kC) {
      const int t0 = c * C;
      if (p.mask != nullptr) s.m = p.mask[(size_t)bi * p.n_mask_chunks + t0 / p.b];
      if (tid < chunk_len(c)) {
        s.e = gel[t0 + tid];
        if (ggl) s.g = ggl[t0 + tid];
      }
    }
    return s;
  };
  auto finish_scalars = [&](int c, const RawScalars& s) {
    if (tid < kC) {
      const bool upd = s.m != 0;
      const bool ok = tid < chunk_len(c);
      sEta[(c & 3) * kC + tid] = (ok && upd) ? sigmoidf_(to_f32(s.e)) * inv_d : 0.f;
      sGate[(c & 3) * kC + tid] = (ok && ggl) ? sigmoidf_(to_f32(s.g)) : 1.f;
      if (tid == 0) sFlag[c & 3] = upd ? 1 : 0;
    }
  };

  // ---------------- prologue ----------------
  WBlock<D, InT, IH> wb;
  wb.init(tid);
  // (token, row) work of the outputs and the look-ahead correction
  const int r = tid % D;
  const int part = tid / D;  // 0 .. 2 IH - 1
  float gam[EPL], bet[EPL];
  float Sgb = 0.f, Sb = 0.f;
  if (!chain) {
    wb.load(p.W0 + (size_t)bh * D * D);  // may alias W_T
    if (nc > 0) {
      tile_load<D>(tileK(0), gk, 0, chunk_len(0), tid, NBT);
      tile_load<D>(tileQ(0), gq, 0, chunk_len(0), tid, NBT);
      tile_load<D>(tileV(0), gv, 0, chunk_len(0), tid, NBT);
      if (nc > 1) tile_load<D>(tileK(1), gk, C, chunk_len(1), tid, NBT);
      cp_async_commit();
      finish_scalars(0, issue_scalars(0));
      if (nc > 1) finish_scalars(1, issue_scalars(1));
      cp_async_wait_all();
      if (p.kq_silu) {
        tile_silu<D, InT>(tileK(0), chunk_len(0), tid, NBT);
        tile_silu<D, InT>(tileQ(0), chunk_len(0), tid, NBT);
        if (nc > 1) tile_silu<D, InT>(tileK(1), chunk_len(1), tid, NBT);
      }
    }
  } else {
    float sgb = 0.f, sb = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int f = lane + 32 * e;
      gam[e] = (f < D && !p.no_ln) ? p.gamma[(size_t)h * D + f] : (f < D ? 1.f : 0.f);
      bet[e] = (f < D && !p.no_ln) ? p.beta[(size_t)h * D + f] : 0.f;
      sgb = fmaf(gam[e], bet[e], sgb);
      sb += bet[e];
    }
    float s2[2] = {sgb, sb};
    butterfly<2>(s2);
    Sgb = s2[0];
    Sb = s2[1];
  }
  __syncthreads();
  if (!chain && nc > 0) {
    // P_0 = K_0 W0^T (no correction), its row means, and A_0
    wb.products(tileK(0), sZ);
    if (!MINIB) {
      const int n0 = chunk_len(0);
      bulk_gram<D, InT, IH>(tileK(0), tileK(0), nullptr, kC, tid, [&](int m, int j, float dot) {
        sA[m * kC + j] = (j < m && m < n0) ? sEta[j] * dot : 0.f;
      });
    }
    bulk_barrier(NBT);
    row_means<D>(sZ, sMu, tid, NBT);
  }
  __syncthreads();

  // ---------------- chunk loop ----------------
  for (int c = 0; c < nc; ++c) {
    const int n = chunk_len(c);
    const bool has_next = c + 1 < nc;
    if (chain) {
      // ===== gradient chain of chunk c =====
      float* Gc = sG + (c & 1) * kC * D;
      float* mGc = sMG + (c & 1) * kC;
      if (sFlag[c & 3]) {
        chain_chunk<D, InT, MINIB, GM>(n, sZ + (c & 1) * kC * D, sA + (c & 1) * kC * kC,
                                       tileV(c), sMu + (c & 1) * kC, Gc, mGc, p.eps, gam, bet,
                                       Sgb, Sb, lane, gnorm_of(c), p.norm_match != 0);
      } else {
        for (int e = lane; e < kC * D; e += 32) Gc[e] = 0.f;
        if (lane < kC) mGc[lane] = 0.f;
        // a SKIP chunk takes no gradient: zero norms for its tokens
        if (float* gn = gnorm_of(c); gn != nullptr && lane < 2 * n) gn[lane] = 0.f;
      }
    } else {
      // ===== bulk work that does not wait for the chain =====
      // prefetch: K_{c+2}, Q_{c+1}, V_{c+1}; raw logits of chunk c+2
      if (c + 2 < nc) tile_load<D>(tileK(c + 2), gk, (c + 2) * C, chunk_len(c + 2), tid, NBT);
      if (has_next) {
        tile_load<D>(tileQ(c + 1), gq, (c + 1) * C, chunk_len(c + 1), tid, NBT);
        tile_load<D>(tileV(c + 1), gv, (c + 1) * C, chunk_len(c + 1), tid, NBT);
      }
      cp_async_commit();
      RawScalars pre{};
      if (c + 2 < nc) pre = issue_scalars(c + 2);

      // W_{s,c} = W_{s,c-1} - sum_j eta_j G_j k_j^T over chunk c-1
      if (c >= 1 && sFlag[(c - 1) & 3])
        wb.rank_update(tileK(c - 1), sG + ((c - 1) & 1) * kC * D, sEta + ((c - 1) & 3) * kC,
                       chunk_len(c - 1));
      if (Wc && ((c * C) % p.b) == 0) wb.store(Wc + (size_t)((c * C) / p.b) * D * D);

      // outputs of chunk c-1
      if (c >= 1) {
        const int np = chunk_len(c - 1);
        const float* Q0p = sQ0 + ((c - 1) & 1) * kC * D;
        const float* Sp = sS + ((c - 1) & 1) * kC * kC;
        const float* Gp = sG + ((c - 1) & 1) * kC * D;
        const float* gt = sGate + ((c - 1) & 3) * kC;
        const bool upd = sFlag[(c - 1) & 3];
        OutT* dst = go + (size_t)(c - 1) * C * D;
        // (a rolled loop: unrolling it costs the registers of a third CTA per SM)
        for (int i = part; i < np; i += 2 * IH) {
          float acc = Q0p[i * D + r], acc2 = 0.f;
          if (upd) {
            int j = 0;
            for (; j + 1 <= i; j += 2) {
              acc = fmaf(-Sp[i * kC + j], Gp[j * D + r], acc);
              acc2 = fmaf(-Sp[i * kC + j + 1], Gp[(j + 1) * D + r], acc2);
            }
            if (j == i) acc = fmaf(-Sp[i * kC + j], Gp[j * D + r], acc);
          }
          const float gate = gch ? sigmoidf_(to_f32(gch[((size_t)(c - 1) * C + i) * D + r])) : gt[i];
          dst[(size_t)i * D + r] = from_f32<OutT>(gate * (acc + acc2));
        }
      }

      // Grams: S_c (Q_c K_c^T), X_{c+1} (K_{c+1} K_c^T), A_{c+1} (K_{c+1} K_{c+1}^T)
      {
        const float* et = sEta + (c & 3) * kC;
        float* Sc = sS + (c & 1) * kC * kC;
        const int n1 = has_next ? chunk_len(c + 1) : 0;
        bulk_gram<D, InT, IH>(tileK(c), tileQ(c), has_next ? tileK(c + 1) : nullptr,
                          has_next ? 2 * kC : kC, tid, [&](int s, int j, float dot) {
                            if (s < kC) {
                              Sc[s * kC + j] = (j <= s && s < n) ? et[j] * dot : 0.f;
                            } else {
                              const int m = s - kC;
                              sX[m * kC + j] = (j < n && m < n1) ? et[j] * dot : 0.f;
                            }
                          });
        if (!MINIB && has_next) {
          const float* et1 = sEta + ((c + 1) & 3) * kC;
          float* An = sA + ((c + 1) & 1) * kC * kC;
          bulk_gram<D, InT, IH>(tileK(c + 1), tileK(c + 1), nullptr, kC, tid,
                            [&](int m, int j, float dot) {
                              An[m * kC + j] = (j < m && m < n1) ? et1[j] * dot : 0.f;
                            });
        }
      }

      // Q0_c = Q_c W_{s,c}^T and P_{c+1} = K_{c+1} W_{s,c}^T
      wb.products(tileQ(c), sQ0 + (c & 1) * kC * D);
      if (has_next) wb.products(tileK(c + 1), sZ + ((c + 1) & 1) * kC * D);
      if (has_next) {
        bulk_barrier(NBT);
        row_means<D>(sZ + ((c + 1) & 1) * kC * D, sMu + ((c + 1) & 1) * kC, tid, NBT);
      }
      if (c + 2 < nc) finish_scalars(c + 2, pre);
      cp_async_wait_all();
      if (p.kq_silu) {
        if (c + 2 < nc) tile_silu<D, InT>(tileK(c + 2), chunk_len(c + 2), tid, NBT);
        if (has_next) tile_silu<D, InT>(tileQ(c + 1), chunk_len(c + 1), tid, NBT);
      }
    }
    __syncthreads();

    // ===== look-ahead correction: Zpre_{c+1} = P_{c+1} - X_{c+1} G_c =====
    if (!chain && has_next && sFlag[c & 3]) {
      const int n1 = chunk_len(c + 1);
      float* Zn = sZ + ((c + 1) & 1) * kC * D;
      const float* Gc = sG + (c & 1) * kC * D;
      for (int m = part; m < n1; m += 2 * IH) {
        float acc = Zn[m * D + r], acc2 = 0.f;
        int j = 0;
        for (; j + 1 < n; j += 2) {
          acc = fmaf(-sX[m * kC + j], Gc[j * D + r], acc);
          acc2 = fmaf(-sX[m * kC + j + 1], Gc[(j + 1) * D + r], acc2);
        }
        if (j < n) acc = fmaf(-sX[m * kC + j], Gc[j * D + r], acc);
        Zn[m * D + r] = acc + acc2;
      }
      if (tid < n1) {
        const float* mGc = sMG + (c & 1) * kC;
        float mu = sMu[((c + 1) & 1) * kC + tid];
        for (int j = 0; j < n; ++j) mu = fmaf(-sX[tid * kC + j], mGc[j], mu);
        sMu[((c + 1) & 1) * kC + tid] = mu;
      }
    }
    __syncthreads();
  }

  // ---------------- epilogue ----------------
  if (!chain) {
    if (nc > 0) {
      const int c = nc - 1;
      const int np = chunk_len(c);
      if (sFlag[c & 3]) wb.rank_update(tileK(c), sG + (c & 1) * kC * D, sEta + (c & 3) * kC, np);
      const float* Q0p = sQ0 + (c & 1) * kC * D;
      const float* Sp = sS + (c & 1) * kC * kC;
      const float* Gp = sG + (c & 1) * kC * D;
      const float* gt = sGate + (c & 3) * kC;
      const bool upd = sFlag[c & 3];
      OutT* dst = go + (size_t)c * C * D;
      for (int i = part; i < np; i += 2 * IH) {
        float acc = Q0p[i * D + r];
        if (upd)
          for (int j = 0; j <= i; ++j) acc = fmaf(-Sp[i * kC + j], Gp[j * D + r], acc);
        const float gate = gch ? sigmoidf_(to_f32(gch[((size_t)c * C + i) * D + r])) : gt[i];
        dst[(size_t)i * D + r] = from_f32<OutT>(gate * acc);
      }
    }
    if (Wc) wb.store(Wc + (size_t)p.n_mask_chunks * D * D);
    wb.store(p.W_T + (size_t)bh * D * D);
  }
}

}  // namespace ttt
