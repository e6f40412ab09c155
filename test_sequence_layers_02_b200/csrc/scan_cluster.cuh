// CUDA-core (fp32) per-token scan with one head spread over a cluster of CS
// CTAs, for the case of few heads (fewer than the SMs / CS).
//
// Same exact chunk identity as scan_simt.cuh ("Edifice.Recurrent.TTT",
// Equations (TTT-Linear)): with W_s the state at the start of chunk c and
// eta-weighted Grams A (in-chunk, j < m), X (next chunk against this one) and
// S (queries against keys, j <= i),
//
//     z_{c,m}   = P_{c,m} - sum_{j<m} A_mj G_{c,j},        P_c = K_c W_{s,c-1}^T - X_c G_{c-1}
//     o_{c,i}   = Q0_{c,i} - sum_{j<=i} S_ij G_{c,j},      Q0_c = Q_c W_{s,c}^T
//     W_{s,c+1} = W_{s,c} - sum_j eta_j G_{c,j} k_{c,j}^T .
//
// Work split. CTA q of the cluster owns rows [q RS, (q+1) RS) of W (RS = 64 / CS)
// in the registers of its four bulk warps (thread = one row x 8 columns). Per
// chunk period the bulk warps apply the rank-C update to their rows, compute
// their rows of Q0_c and of K_{c+1} W_{s,c}^T, and rows [4q, 4q+4) of the
// Grams A_{c+1} and X_{c+2} (those three sent to EVERY CTA of the cluster),
// form S_c, write this CTA's rows of the outputs of chunk c-1 and prefetch
// the next tiles and scalars.
// Warp 0 of every CTA runs the same sequential gradient chain over the full 64
// features (replicated, so G never crosses CTAs); besides the in-chunk
// right-looking update it applies each G_{c,j} to the NEXT chunk's z's (the
// -X G_c term above), so the next chunk starts from P + that correction with
// no separate correction phase.
//
// Hand-off. Within a CTA, one block barrier ends every chunk period (buffers
// written in period c are read in period c+1 and are double-buffered). Across
// the cluster the chain's inputs move: each CTA keeps four delivery slots
// (P^T, A^T, X^T of one chunk), each with an mbarrier that expects the slot's
// 6144 bytes; producers write with
// asynchronous remote stores that complete those bytes on the consumer's
// barrier, the chain waits (bounded) for the slot and re-arms it for its next
// use. The chain waits for every chunk, so no CTA runs more than two periods
// ahead of another and four slots are enough for a slot never to be rewritten
// while it is read. A slot holds P transposed, [feature][token] with a padded
// token stride, so the chain reads its two features' 16 tokens with
// conflict-free 16-byte loads.
#pragma once

#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"
#include "scan_simt.cuh"

namespace ttt {

template <typename InT, int CS>
struct ClusterLayout {
  static constexpr int D = 64;
  static constexpr int RS = D / CS;         // rows of W per CTA
  static constexpr int NW = 128;            // bulk threads (warps 0-3)
  static constexpr int NT = NW + 32;        // + the chain warp (warp 4)
  static constexpr int G = NW / RS;         // threads per row of W
  static constexpr int KW = D / G;          // columns of W per thread
  static constexpr int ELT = (int)sizeof(InT);
  static constexpr int ROWB = D * ELT + 16; // padded tile row (bytes), as scan_simt.cuh
  static constexpr int TILE = kC * ROWB;
  static constexpr int oK = 0;                        // K tiles, ring of 8
  static constexpr int oQ = oK + 8 * TILE;            // Q tiles, ring of 2
  static constexpr int oV = oQ + 2 * TILE;            // V tiles, ring of 2
  static constexpr int NPS = 4;                       // P slots
  static constexpr int PTS = kC + 4;                  // padded token stride of a P slot
  static constexpr int SAT = D * PTS;                 // offset of A^T[j][m] in a slot (floats)
  static constexpr int SXT = SAT + kC * kC;           // offset of X^T[j][m]
  static constexpr int PSLOT = SXT + kC * kC;         // floats per delivery slot
  static constexpr int oP = oV + 2 * TILE;            // delivery slots [NPS][PSLOT]
  static constexpr int oG = oP + NPS * PSLOT * 4;     // G                     [2][kC][D]
  static constexpr int oQ0 = oG + 2 * kC * D * 4;     // own rows of Q0        [2][kC][RS]
  static constexpr int oS = oQ0 + 2 * kC * RS * 4;    // S[i][j]               [2][kC][kC]
  static constexpr int oEta = oS + 2 * kC * kC * 4;   // eta  [4][kC]
  static constexpr int oGate = oEta + 4 * kC * 4;     // gate [4][kC]
  static constexpr int oFlag = oGate + 4 * kC * 4;    // chunk updates? [4]
  static constexpr int oBar = oFlag + 16;              // P-slot mbarriers [NPS]
  static constexpr int bytes = oBar + NPS * 8;
  // one delivery, all CTAs together: P (kC x D) and the two Grams (kC x kC each)
  static constexpr uint32_t kSlotBytes = (kC * D + 2 * kC * kC) * 4;
  static_assert(RS == 16 && NW == 128, "each CTA computes four Gram rows with two threads per dot");
  // Requested dynamic shared memory: more than half an SM's, so that one CTA
  // of a cluster runs per SM.
  static constexpr int launch_bytes = bytes > 120 * 1024 ? bytes : 120 * 1024;
  static_assert(KW == 8, "a W thread holds two 4-element units of its row");
};

// Set when a bounded wait of this kernel gave up; read and cleared by
// ttt_check_device_status(). One word per device in this module.
__device__ int g_cluster_status;

// Polls of the second, fixed bound a chain wait keeps using after the caller's
// limit ran out (the flag is then already set): it keeps the P slots'
// barrier bookkeeping in step, so no delivery is still in flight at exit.
constexpr long long kDrainPolls = 1LL << 24;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint32_t cluster_addr(uint32_t local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
  return remote;
}
__device__ __forceinline__ void pbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void pbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// The one expected arrival of a slot phase, announcing its byte count.
__device__ __forceinline__ void pbar_arm(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool pbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}
// Asynchronous 16-byte store into another CTA's shared memory; its completion
// counts 16 bytes on that CTA's barrier (both addresses in the cluster window).
__device__ __forceinline__ void st_async_v4(uint32_t remote_dst, float a, float b, float c,
                                            float d, uint32_t remote_bar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::
          "r"(remote_dst),
      "f"(a), "f"(b), "f"(c), "f"(d), "r"(remote_bar)
      : "memory");
}

// One CTA per SM, as the shared memory request already forces: the explicit
// minimum in the launch bounds lets the compiler give every thread up to 255
// registers.
template <typename InT, typename OutT, int GM, int CS>
__global__ void __launch_bounds__(ClusterLayout<InT, CS>::NT, 1)
    scan_cluster_kernel(const ScanParams p) {
  namespace cg = cooperative_groups;
  using L = ClusterLayout<InT, CS>;
  constexpr int D = 64;
  constexpr int RS = L::RS, G = L::G, KW = L::KW;
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned char* sK = smem + L::oK;
  unsigned char* sQ = smem + L::oQ;
  unsigned char* sV = smem + L::oV;
  float* sP = reinterpret_cast<float*>(smem + L::oP);
  float* sG = reinterpret_cast<float*>(smem + L::oG);
  float* sQ0 = reinterpret_cast<float*>(smem + L::oQ0);
  float* sS = reinterpret_cast<float*>(smem + L::oS);
  float* sEta = reinterpret_cast<float*>(smem + L::oEta);
  float* sGate = reinterpret_cast<float*>(smem + L::oGate);
  int* sFlag = reinterpret_cast<int*>(smem + L::oFlag);
  uint64_t* pbar = reinterpret_cast<uint64_t*>(smem + L::oBar);

  cg::cluster_group cluster = cg::this_cluster();
  const int q = (int)cluster.block_rank();
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const bool chain = tid >= L::NW;
  const long long bh = blockIdx.x / CS;
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

  auto chunk_len = [&](int c) { return (c < nc) ? min(C, T - c * C) : 0; };
  auto tileK = [&](int c) { return sK + (c & 7) * L::TILE; };
  auto tileQ = [&](int c) { return sQ + (c & 1) * L::TILE; };
  auto tileV = [&](int c) { return sV + (c & 1) * L::TILE; };

  const int at = tid;  // bulk thread index for prefetch, scalars and outputs
  struct RawScalars {
    InT e, g;
    unsigned char m;
  };
  auto issue_scalars = [&](int c) {
    RawScalars s;
    s.e = InT();
    s.g = InT();
    s.m = 1;
    if (at < kC) {
      const int t0 = c * C;
      if (p.mask != nullptr) s.m = p.mask[(size_t)bi * p.n_mask_chunks + t0 / p.b];
      if (at < chunk_len(c)) {
        s.e = gel[t0 + at];
        if (ggl) s.g = ggl[t0 + at];
      }
    }
    return s;
  };
  auto finish_scalars = [&](int c, const RawScalars& s) {
    if (at < kC) {
      const bool upd = s.m != 0;
      const bool ok = at < chunk_len(c);
      sEta[(c & 3) * kC + at] = (ok && upd) ? sigmoidf_(to_f32(s.e)) * inv_d : 0.f;
      sGate[(c & 3) * kC + at] = (ok && ggl) ? sigmoidf_(to_f32(s.g)) : 1.f;
      if (at == 0) sFlag[c & 3] = upd ? 1 : 0;
    }
  };

  // ---- bulk thread wt = 0..127 holds W[grow][8 g .. 8 g + 7] ----
  const int wt = tid;
  const int rl = wt / G;
  const int g = wt % G;
  const int grow = q * RS + rl;
  // fp32 tiles: the upper half of the column groups takes its two 4-column
  // units in swapped order, so the 8 broadcast addresses of one load hit
  // disjoint banks
  const int swap = (L::ELT == 4 && g >= G / 2) ? 1 : 0;
  auto ucol = [&](int u) { return g * KW + 4 * (u ^ swap); };  // first column of unit u
  float2 W2[4];  // unit u: W2[2 u], W2[2 u + 1] = columns ucol(u) .. + 3

  // W_{s} -= sum_j eta_j G_j[grow] k_j^T over the kC rows of tile Kt (rows past
  // the chunk have eta = 0 and G = 0). All scales are loaded first; keys go in
  // groups of 4 so the loads of a group overlap the FMAs of the previous one.
  auto rank_update = [&](const unsigned char* Kt, const float* Gp, const float* et) {
    float nge[kC];
#pragma unroll
    for (int j = 0; j < kC; ++j) nge[j] = -et[j] * Gp[j * D + grow];
#pragma unroll
    for (int j0 = 0; j0 < kC; j0 += 4) {
      float2 x[4][2][2];
#pragma unroll
      for (int b = 0; b < 4; ++b)
#pragma unroll
        for (int u = 0; u < 2; ++u) Unit<InT>::ld(Kt + (j0 + b) * L::ROWB + ucol(u) * L::ELT, x[b][u]);
#pragma unroll
      for (int b = 0; b < 4; ++b)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          W2[2 * u] = __ffma2_rn(dup2(nge[j0 + b]), x[b][u][0], W2[2 * u]);
          W2[2 * u + 1] = __ffma2_rn(dup2(nge[j0 + b]), x[b][u][1], W2[2 * u + 1]);
        }
    }
  };
  // Rows [0, kC) of Q0 from rowsA (may be null) and of P from rowsB (may be
  // null), for this CTA's rows; P goes to slot `pslot` of every CTA of the cluster.
  auto products = [&](const unsigned char* rowsA, const unsigned char* rowsB, float* q0dst,
                      int pslot) {
    float acc[2 * kC];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const unsigned char* R = half == 0 ? rowsA : rowsB;
      if (R != nullptr) {
#pragma unroll
        for (int t0 = 0; t0 < kC; t0 += 4) {
          float2 x[4][2][2];
#pragma unroll
          for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int u = 0; u < 2; ++u) Unit<InT>::ld(R + (t0 + b) * L::ROWB + ucol(u) * L::ELT, x[b][u]);
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            float2 a0 = __fmul2_rn(W2[0], x[b][0][0]);
            float2 a1 = __fmul2_rn(W2[1], x[b][0][1]);
            a0 = __ffma2_rn(W2[2], x[b][1][0], a0);
            a1 = __ffma2_rn(W2[3], x[b][1][1], a1);
            const float2 a = __fadd2_rn(a0, a1);
            acc[half * kC + t0 + b] = a.x + a.y;
          }
        }
      } else {
#pragma unroll
        for (int t = 0; t < kC; ++t) acc[half * kC + t] = 0.f;
      }
    }
    reduce_scatter_lanes<2 * kC, G>(acc, g);
    constexpr int PER = 2 * kC / G;
    static_assert(PER == 4, "four tokens per thread after the reduce-scatter");
    const int t0 = g * PER;
    if (t0 < kC) {
      if (q0dst != nullptr) {
#pragma unroll
        for (int v = 0; v < PER; ++v) q0dst[(t0 + v) * RS + rl] = acc[v];
      }
    } else if (pslot >= 0) {
      // tokens t0 - kC .. + 3 of row grow, into P^T of every CTA
      const uint32_t dst = smem_addr(sP + pslot * L::PSLOT + grow * L::PTS + (t0 - kC));
      const uint32_t bar = smem_addr(pbar + pslot);
#pragma unroll
      for (int rk = 0; rk < CS; ++rk)
        st_async_v4(cluster_addr(dst, rk), acc[0], acc[1], acc[2], acc[3], cluster_addr(bar, rk));
    }
  };
  const int gt = tid;
  // Dot products of NL left rows (left0 rows, then left1 rows) with the kC rows
  // of `right`: Gram thread (j, half) holds right row j's half in registers; the
  // result of (left row s, right row j) goes to emit(s, j, dot).
  auto gram = [&](auto nl_tag, const unsigned char* right, const unsigned char* left0,
                  const unsigned char* left1, auto emit) {
    constexpr int NL = decltype(nl_tag)::value;
    constexpr int NG = L::NW / 32;  // bulk warps
    static_assert(NL % (2 * NG) == 0, "left rows go two per warp at a time");
    const int j = gt & 15, kq = (gt >> 4) & 1, grp = gt >> 5;
    float2 rk[D / 4];
#pragma unroll
    for (int u = 0; u < (D / 2) / 4; ++u) {
      float2 x[2];
      Unit<InT>::ld(right + j * L::ROWB + (kq * (D / 2) + u * 4) * L::ELT, x);
      rk[2 * u] = x[0];
      rk[2 * u + 1] = x[1];
    }
    // two left rows at a time, each with two accumulator chains
#pragma unroll
    for (int it = 0; it < NL / NG; it += 2) {
      int s[2];
      const unsigned char* row[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        s[r] = grp + NG * (it + r);
        row[r] = (s[r] < kC ? left0 + s[r] * L::ROWB : left1 + (s[r] - kC) * L::ROWB) +
                 kq * (D / 2) * L::ELT;
      }
      float2 acc[2][2];
#pragma unroll
      for (int r = 0; r < 2; ++r) acc[r][0] = acc[r][1] = make_float2(0.f, 0.f);
#pragma unroll
      for (int u = 0; u < (D / 2) / 4; ++u) {
        float2 x[2][2];
#pragma unroll
        for (int r = 0; r < 2; ++r) Unit<InT>::ld(row[r] + u * 4 * L::ELT, x[r]);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          acc[r][0] = __ffma2_rn(rk[2 * u], x[r][0], acc[r][0]);
          acc[r][1] = __ffma2_rn(rk[2 * u + 1], x[r][1], acc[r][1]);
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const float2 a = __fadd2_rn(acc[r][0], acc[r][1]);
        float dot = a.x + a.y;
        dot += __shfl_xor_sync(0xffffffffu, dot, 16);
        if (kq == 0) emit(s[r], j, dot);
      }
    }
  };
  // Rows [4q, 4q+4) of the eta-weighted Grams feeding the chain of chunk c,
  // A_c (K_c against K_c) and X_{c+1} (K_{c+1} against K_c), sent transposed
  // into delivery slot c % NPS of every CTA. Thread (j, r, half): right row j,
  // left row 4q + r, half the features; four threads' values per j travel as
  // one 16-byte store.
  auto split_grams = [&](int c) {
    const int pr = wt >> 1, kq = wt & 1;
    const int j = pr >> 2, r = pr & 3, Lrow = 4 * q + r;
    const float* et = sEta + (c & 3) * kC;
    const int n0 = chunk_len(c), n1 = chunk_len(c + 1);
    const unsigned char* right = tileK(c) + j * L::ROWB + kq * (D / 2) * L::ELT;
    const unsigned char* la = tileK(c) + Lrow * L::ROWB + kq * (D / 2) * L::ELT;
    const unsigned char* lx = tileK(c + 1) + Lrow * L::ROWB + kq * (D / 2) * L::ELT;
    float2 aa[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float2 ax[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int u = 0; u < (D / 2) / 4; ++u) {
      float2 xr[2], xa[2], xx[2];
      Unit<InT>::ld(right + u * 4 * L::ELT, xr);
      Unit<InT>::ld(la + u * 4 * L::ELT, xa);
      Unit<InT>::ld(lx + u * 4 * L::ELT, xx);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        aa[t] = __ffma2_rn(xr[t], xa[t], aa[t]);
        ax[t] = __ffma2_rn(xr[t], xx[t], ax[t]);
      }
    }
    const float2 sa = __fadd2_rn(aa[0], aa[1]), sx = __fadd2_rn(ax[0], ax[1]);
    float da = sa.x + sa.y, dx = sx.x + sx.y;
    da += __shfl_xor_sync(0xffffffffu, da, 1);
    dx += __shfl_xor_sync(0xffffffffu, dx, 1);
    da = (j < Lrow && Lrow < n0) ? et[j] * da : 0.f;
    dx = (j < n0 && Lrow < n1) ? et[j] * dx : 0.f;
    // lanes 8 j' + 2 r hold r = 0..3 of one j: gather them on lane 8 j'
    float va[4], vx[4];
    va[0] = da;
    vx[0] = dx;
#pragma unroll
    for (int k = 1; k < 4; ++k) {
      va[k] = __shfl_down_sync(0xffffffffu, da, 2 * k);
      vx[k] = __shfl_down_sync(0xffffffffu, dx, 2 * k);
    }
    if ((lane & 7) == 0) {
      float* slot = sP + (c % L::NPS) * L::PSLOT;
      const uint32_t dA = smem_addr(slot + L::SAT + j * kC + 4 * q);
      const uint32_t dX = smem_addr(slot + L::SXT + j * kC + 4 * q);
      const uint32_t bar = smem_addr(pbar + (c % L::NPS));
#pragma unroll
      for (int rk = 0; rk < CS; ++rk) {
        const uint32_t rb = cluster_addr(bar, rk);
        st_async_v4(cluster_addr(dA, rk), va[0], va[1], va[2], va[3], rb);
        st_async_v4(cluster_addr(dX, rk), vx[0], vx[1], vx[2], vx[3], rb);
      }
    }
  };
  auto store_W = [&](float* dst_row) {
#pragma unroll
    for (int u = 0; u < 2; ++u)
      *reinterpret_cast<float4*>(dst_row + ucol(u)) =
          make_float4(W2[2 * u].x, W2[2 * u].y, W2[2 * u + 1].x, W2[2 * u + 1].y);
  };

  // ---- outputs of chunk c, this CTA's rows ----
  constexpr int NOUT = (kC * RS) / L::NW;
  // per-feature gate logits of this thread's outputs of chunk c
  auto gate_logits = [&](int c, float (&g)[NOUT]) {
#pragma unroll
    for (int k = 0; k < NOUT; ++k) {
      const int idx = at + L::NW * k;
      const int i = idx / RS, rr = idx % RS;
      g[k] = (gch && i < chunk_len(c)) ? to_f32(gch[((size_t)c * C + i) * D + q * RS + rr]) : 0.f;
    }
  };
  auto outputs = [&](int c, const float (&gpre)[NOUT]) {
    const int np = chunk_len(c);
    const float* Q0p = sQ0 + (c & 1) * kC * RS;
    const float* Sp = sS + (c & 1) * kC * kC;
    const float* Gp = sG + (c & 1) * kC * D + q * RS;
    const float* gt = sGate + (c & 3) * kC;
    const bool upd = sFlag[c & 3];
    OutT* dst = go + (size_t)c * C * D + q * RS;
#pragma unroll
    for (int k = 0; k < NOUT; ++k) {
      const int idx = at + L::NW * k;
      const int i = idx / RS, rr = idx % RS;
      float acc = Q0p[i * RS + rr], acc2 = 0.f;
      if (upd) {
        const float4* srow = reinterpret_cast<const float4*>(Sp + i * kC);
#pragma unroll
        for (int j4 = 0; j4 < kC / 4; ++j4) {
          const float4 s4 = srow[j4];
          acc = fmaf(-s4.x, Gp[(4 * j4) * D + rr], acc);
          acc2 = fmaf(-s4.y, Gp[(4 * j4 + 1) * D + rr], acc2);
          acc = fmaf(-s4.z, Gp[(4 * j4 + 2) * D + rr], acc);
          acc2 = fmaf(-s4.w, Gp[(4 * j4 + 3) * D + rr], acc2);
        }
      }
      const float gate = gch ? sigmoidf_(gpre[k]) : gt[i];
      if (i < np) dst[(size_t)i * D + rr] = from_f32<OutT>(gate * (acc + acc2));
    }
  };

  // ---- chain state (warp 4) ----
  Chain<D, InT, false, GM, L::PTS> ch;
  unsigned dead = 0;  // P slots whose bookkeeping was lost after a failed drain

  // ---------------- prologue ----------------
  if (chain) {
    if (lane == 0) {
#pragma unroll
      for (int sl = 0; sl < L::NPS; ++sl) {
        pbar_init(pbar + sl, 1);
        if (sl < nc) pbar_arm(pbar + sl, L::kSlotBytes);  // deliveries of chunks 0..3
      }
      pbar_init_fence();
    }
    ch.init(p.gamma + (size_t)h * D, p.beta + (size_t)h * D, p.no_ln, lane);
  } else {
    const float* W0 = p.W0 + ((size_t)bh * D + grow) * D;  // may alias W_T
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float4 w4 = *reinterpret_cast<const float4*>(W0 + ucol(u));
      W2[2 * u] = make_float2(w4.x, w4.y);
      W2[2 * u + 1] = make_float2(w4.z, w4.w);
    }
    if (nc > 0) {
      tile_load<D>(tileK(0), gk, 0, chunk_len(0), at, L::NW);
      tile_load<D>(tileQ(0), gq, 0, chunk_len(0), at, L::NW);
      tile_load<D>(tileV(0), gv, 0, chunk_len(0), at, L::NW);
      if (nc > 1) tile_load<D>(tileK(1), gk, C, chunk_len(1), at, L::NW);
      if (nc > 2) tile_load<D>(tileK(2), gk, 2 * C, chunk_len(2), at, L::NW);
      cp_async_commit();
      finish_scalars(0, issue_scalars(0));
      if (nc > 1) finish_scalars(1, issue_scalars(1));
      cp_async_wait_all();
      if (p.kq_silu) {
        tile_silu<D, InT>(tileK(0), chunk_len(0), at, L::NW);
        tile_silu<D, InT>(tileQ(0), chunk_len(0), at, L::NW);
        if (nc > 1) tile_silu<D, InT>(tileK(1), chunk_len(1), at, L::NW);
        if (nc > 2) tile_silu<D, InT>(tileK(2), chunk_len(2), at, L::NW);
      }
    }
  }
  // every CTA has started and armed its barriers before any remote access
  cluster.sync();
  if (!chain && nc > 0) {
    products(nullptr, tileK(0), nullptr, 0);  // P_0 = K_0 W0^T, into slot 0 everywhere
    split_grams(0);                           // A_0, X_1
  }
  __syncthreads();

  // ---------------- chunk loop ----------------
  for (int c = 0; c < nc; ++c) {
    const int n = chunk_len(c);
    const bool has_next = c + 1 < nc;
    if (chain) {
      // ===== gradient chain of chunk c =====
      // P_c from every CTA of the cluster, waited for even on a SKIP chunk
      // (that keeps the CTAs paced), then the slot is re-armed for chunk c + 4
      const int sl = c % L::NPS;
      if (!((dead >> sl) & 1u)) {
        const uint32_t parity = (uint32_t)((c / L::NPS) & 1);
        bool ok = false;
        for (long long it = 0; it < p.wait_limit && !ok; ++it) ok = pbar_try_wait(pbar + sl, parity);
        if (!ok) {
          if (lane == 0) atomicExch(&g_cluster_status, (int)kStatusTimeout);
          for (long long it = 0; it < kDrainPolls && !ok; ++it) ok = pbar_try_wait(pbar + sl, parity);
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) dead |= 1u << sl;
        else if (lane == 0 && c + L::NPS < nc) pbar_arm(pbar + sl, L::kSlotBytes);
      }
      if (!sFlag[c & 3]) {
        ch.reset();  // a SKIP chunk leaves the next chunk uncorrected (its X is zero)
      } else {
        const float* PT = sP + sl * L::PSLOT;
        ch.run(n, PT, PT + L::SAT, PT + L::SXT, tileV(c), sG + (c & 1) * kC * D, p.eps, lane);
      }
    } else {
      // ===== bulk work of period c =====
      if (c + 3 < nc) tile_load<D>(tileK(c + 3), gk, (c + 3) * C, chunk_len(c + 3), at, L::NW);
      if (has_next) {
        tile_load<D>(tileQ(c + 1), gq, (c + 1) * C, chunk_len(c + 1), at, L::NW);
        tile_load<D>(tileV(c + 1), gv, (c + 1) * C, chunk_len(c + 1), at, L::NW);
      }
      cp_async_commit();
      RawScalars pre{};
      if (c + 2 < nc) pre = issue_scalars(c + 2);
      float gpre[NOUT];
      if (c >= 1) gate_logits(c - 1, gpre);
      // W_{s,c} = W_{s,c-1} - sum_j eta_j G_{c-1,j} k_{c-1,j}^T on this CTA's rows
      if (c >= 1 && sFlag[(c - 1) & 3])
        rank_update(tileK(c - 1), sG + ((c - 1) & 1) * kC * D, sEta + ((c - 1) & 3) * kC);
      if (Wc && ((c * C) % p.b) == 0) store_W(Wc + ((size_t)((c * C) / p.b) * D + grow) * D);
      // Q0_c (own rows) and K_{c+1} W_{s,c}^T (own rows, to every CTA)
      products(tileQ(c), has_next ? tileK(c + 1) : nullptr, sQ0 + (c & 1) * kC * RS,
               has_next ? ((c + 1) % L::NPS) : -1);
      // this CTA's rows of the Grams of the chain of chunk c+1, then S_c
      if (has_next) split_grams(c + 1);
      {
        const float* et = sEta + (c & 3) * kC;
        float* Sc = sS + (c & 1) * kC * kC;
        gram(std::integral_constant<int, kC>(), tileK(c), tileQ(c), nullptr,
             [&](int s, int j, float dot) {
               Sc[s * kC + j] = (j <= s && s < n) ? et[j] * dot : 0.f;
             });
      }
      if (c >= 1) outputs(c - 1, gpre);
      if (c + 2 < nc) finish_scalars(c + 2, pre);
      cp_async_wait_all();
      if (p.kq_silu) {
        if (c + 3 < nc) tile_silu<D, InT>(tileK(c + 3), chunk_len(c + 3), at, L::NW);
        if (has_next) tile_silu<D, InT>(tileQ(c + 1), chunk_len(c + 1), at, L::NW);
      }
    }
    __syncthreads();
  }

  // ---------------- epilogue ----------------
  if (nc > 0) {
    const int c = nc - 1;
    if (!chain && sFlag[c & 3]) rank_update(tileK(c), sG + (c & 1) * kC * D, sEta + (c & 3) * kC);
    if (!chain) {
      float gpre[NOUT];
      gate_logits(c, gpre);
      outputs(c, gpre);
    }
  }
  if (!chain) {
    if (Wc) store_W(Wc + ((size_t)p.n_mask_chunks * D + grow) * D);
    store_W(p.W_T + ((size_t)bh * D + grow) * D);
  }
  cluster.sync();  // no CTA leaves while a peer could still address its shared memory
}

}  // namespace ttt
