// Tensor-core (tcgen05) mini-batch scan: d = 64, b = 16, bf16 q/k/v/logits,
// fp32 state W in TMEM, bf16 or fp32 outputs.
//
// Chunk step (PonderTTT, "Technical Architecture": dual-form updates; every
// gradient of a chunk taken at the chunk-start state W_s):
//     z_i = W_s k_i,  G_i = LayerNorm gradient ("Error Correction in Trained
//     TTT Layers", Abstract),  o_i = W_s q_i - sum_{j<=i} eta_j (k_j.q_i) G_j,
//     W_e = W_s - sum_j eta_j G_j k_j^T.
//
// Look-ahead. With Aneg_c[f][j] = -eta_j G_j[f] and W_{s,c+1} = W_{s,c} + Aneg_c K_c,
//     Z_{c+1} = K_{c+1} W_{s,c+1}^T = P_{c+1} - X_{c+1} G_c,
//     P_{c+1} = K_{c+1} W_{s,c}^T,   X_{c+1}[m][j] = eta_{c,j} (k_{c+1,m} . k_{c,j}),
// so P_{c+1} is produced by the tensor core a whole chunk early and only the
// 16x16x64 correction X G stays between two LayerNorms.
//
// Warp roles (256 threads):
//   chain warps 0-3: correction Z_k = P_k - X_k G_{k-1} (feature-major, from
//     TMEM), transpose through shared memory, token-major LayerNorm + gradient
//     (8 lanes per token, 3-level shuffles), write G_k and Aneg_k.
//   bulk warps 4-7 (thread 128 issues every MMA and TMA):
//     MMA2  O_c^T += Aneg_c . M_c^T   (M_c = tril(Q_c K_c^T), bf16)
//     MMA3  W     += Aneg_c . K_c      (fp32 W in TMEM; K tile as MN-major operand)
//     W (TMEM fp32) -> bf16 W_s operand; o_c = gate * O_c^T -> HBM
//     Grams X_{c+2}, M_{c+1}; MMA1 P_{c+2}^T = W_s K_{c+2}^T, Q0_{c+1}^T = W_s Q_{c+1}^T
//     TMA of chunk c+4 into a 4-stage ring (K, Q 128B-swizzled; V plain).
// M = 128 everywhere: A operands stack two copies of their 64 rows, so TMEM
// lanes 0-63 and 64-127 hold identical results and any warp quarter can read.
//
// Handoffs use mbarriers in rings of two, so a producer is never two phases
// ahead of its consumer. Every wait is bounded; on expiry the CTA records the
// timeout status, both warp groups leave their loops, the MMA-issuing thread
// drains its MMAs and copies (with a bound of its own), and TMEM is freed.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace ttt {

struct TcMaps {
  CUtensorMap q, k, v;  // [B*H][T][64] bf16 as {64, T, B*H}, box {64, 16, 1}
};

namespace tc {

constexpr int D = 64;
constexpr int CB = 16;             // chunk (b)
constexpr int NT = 256;            // 4 chain + 4 bulk warps
constexpr int NST = 4;             // TMA stages
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kTmemGramCols = 32;  // second allocation: X (16 cols) | M (16 cols), lanes 0-15
constexpr uint32_t kColW = 0;      // W accumulator, 64 columns
// slot s (s = 0, 1): P^T at 64 + 32 s, Q0^T / O^T at 80 + 32 s (16 columns each)
__device__ __forceinline__ uint32_t col_p(int s) { return 64u + 32u * (uint32_t)s; }
__device__ __forceinline__ uint32_t col_o(int s) { return 80u + 32u * (uint32_t)s; }
constexpr int kTile = CB * D * 2;  // 2048 bytes
constexpr int kZS = 72;            // row stride (floats) of the token-major Z / G tiles

// shared-memory carve-up (bytes from a 1024-aligned base)
constexpr int oStage = 0;                          // [NST][K | Q | V]
constexpr int kStageBytes = 3 * kTile;
constexpr int oWb = oStage + NST * kStageBytes;    // W_s bf16, 128 rows x 128 B, SW128
constexpr int oAneg = oWb + 128 * 128;             // [2] 128 rows x 16 bf16 (core matrices)
constexpr int oM = oAneg + 2 * 128 * 32;           // [2] 16 x 16 bf16 (core matrices)
constexpr int oZ = oM + 2 * 512;                   // [2][16][kZS] f32
constexpr int oG = oZ + 2 * CB * kZS * 4;          // [2][16][kZS] f32
constexpr int oX = oG + 2 * CB * kZS * 4;          // [2][16][16] f32
constexpr int kSR = 32;                            // scalar ring (chunks)
constexpr int oEta = oX + 2 * CB * CB * 4;         // [kSR][16] f32 (mask folded in)
constexpr int oGate = oEta + kSR * CB * 4;         // [kSR][16] f32
constexpr int oFlag = oGate + kSR * CB * 4;        // [kSR] int
constexpr int oGam = oFlag + kSR * 4;              // gamma, beta [2][64] f32
constexpr int oBar = oGam + 2 * D * 4;             // mbarriers
constexpr int kBars = NST + 2 + 2 + 1 + 1 + 1;     // tma[4], px[2], g[2], w, pro, gram
constexpr int oTmem = oBar + kBars * 8;            // two TMEM base addresses
constexpr int oAbort = oTmem + 8;
constexpr int kSmemUsed = oAbort + 4;
constexpr int kSmemBytes = kSmemUsed + 1024;       // + alignment slack
static_assert(kSmemBytes <= 75 * 1024, "three CTAs per SM must fit");
static_assert(3 * (kTmemCols + kTmemGramCols) <= 512, "three CTAs per SM must fit in TMEM");

__device__ __forceinline__ int core_off(int row, int k) {
  return (row >> 3) * 256 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}
__device__ __forceinline__ int sw128_off(int row, int chunk) {
  return row * 128 + ((chunk ^ (row & 7)) << 4);
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ void bf16x8_to_f32(uint4 u, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
// Barrier over a 128-thread warp group that returns whether any member passed true.
__device__ __forceinline__ bool group_any(int bar_id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.b32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, 128, pi;\n\t"
      "selp.b32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((int)v), "r"(bar_id)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void group_sync(int bar_id) {
  asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(sm100::smem_u32(bar))
               : "memory");
}
constexpr int kBarChain = 2;  // named barrier ids (0 is __syncthreads)
constexpr int kBarBulk = 3;

}  // namespace tc

template <typename OutT, int GM>
__global__ void __launch_bounds__(tc::NT, 3)
    scan_tc_kernel(const ScanParams p, const __grid_constant__ TcMaps maps) {
  using namespace tc;
  using namespace sm100;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sStage = smem + oStage;
  unsigned char* sWb = smem + oWb;
  float* sZ = reinterpret_cast<float*>(smem + oZ);
  float* sG = reinterpret_cast<float*>(smem + oG);
  float* sX = reinterpret_cast<float*>(smem + oX);
  float* sEta = reinterpret_cast<float*>(smem + oEta);
  float* sGate = reinterpret_cast<float*>(smem + oGate);
  int* sFlag = reinterpret_cast<int*>(smem + oFlag);
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(smem + oBar);  // [NST]
  uint64_t* bar_px = bar_tma + NST;  // [2]: delivery k = {P_k, Q0_{k-1}, X_k} on px[k & 1]
  uint64_t* bar_g = bar_px + 2;      // [2]: G_k / Aneg_k written, on g[k & 1]
  uint64_t* bar_w = bar_g + 2;       // bulk MMAs of a chunk complete
  uint64_t* bar_pro = bar_w + 1;     // prologue MMAs complete
  uint64_t* bar_gram = bar_pro + 1;  // Gram MMAs complete
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + oTmem);
  float* sGam = reinterpret_cast<float*>(smem + oGam);
  float* sBet = sGam + D;
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + oAbort);
  auto tK = [&](int c) { return sStage + (c & (NST - 1)) * kStageBytes; };
  auto tQ = [&](int c) { return sStage + (c & (NST - 1)) * kStageBytes + kTile; };
  auto tV = [&](int c) { return sStage + (c & (NST - 1)) * kStageBytes + 2 * kTile; };
  auto aneg = [&](int c) { return smem + oAneg + (c & 1) * 4096; };
  auto mmat = [&](int c) { return smem + oM + (c & 1) * 512; };

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const bool chain = warp < 4;
  const int wq = warp & 3;                     // TMEM lane quarter
  const uint32_t tlane = (uint32_t)(wq * 32) << 16;
  const int fm = (wq & 1) * 32 + lane;         // feature-major role: feature
  const int half = wq >> 1;                    // feature-major role: tokens 8*half .. +8
  const int gt = tid & 127;                    // index within the warp group
  const long long bh = blockIdx.x;
  const int bi = (int)(bh / p.H);
  const int h = (int)(bh - (long long)bi * p.H);
  const int T = p.T;
  const int nc = (T + CB - 1) / CB;
  const size_t tok0 = (size_t)bh * T;
  const __nv_bfloat16* gel = static_cast<const __nv_bfloat16*>(p.eta_logit) + tok0;
  const __nv_bfloat16* ggl =
      p.gate_logit ? static_cast<const __nv_bfloat16*>(p.gate_logit) + tok0 : nullptr;
  OutT* go = static_cast<OutT*>(p.o) + tok0 * D;
  float* Wc = p.W_chunks ? p.W_chunks + (size_t)bh * (p.n_mask_chunks + 1) * D * D : nullptr;
  const long long lim = p.wait_limit;
  const long long drain_lim = 1LL << 24;
  const bool mma_thread = (tid == 128);
  auto chunk_len = [&](int c) { return min(CB, T - c * CB); };

  // ---- per-chunk scalars (eta with the mask folded in, gate, update flag) in
  // a ring of kSR chunks. The bulk group loads them in blocks of 8 chunks,
  // 16 chunks ahead: fetch_block() issues the global loads into registers and
  // store_block(), four iterations later, writes the ring.
  struct Raw {
    __nv_bfloat16 e, g;
    unsigned char m;
  };
  auto fetch_block = [&](int x0) {
    Raw r;
    r.e = __float2bfloat16(0.f);
    r.g = __float2bfloat16(0.f);
    r.m = 1;
    const int x = x0 + (gt >> 4), i = gt & 15;
    if (x < nc) {
      if (p.mask) r.m = p.mask[(size_t)bi * p.n_mask_chunks + x];
      const int t = x * CB + i;
      if (t < T) {
        r.e = gel[t];
        if (ggl) r.g = ggl[t];
      }
    }
    return r;
  };
  auto store_block = [&](int x0, const Raw& r) {
    const int x = x0 + (gt >> 4), i = gt & 15;
    if (x < nc) {
      const bool ok = x * CB + i < T;
      sEta[(x & (kSR - 1)) * CB + i] =
          (ok && r.m) ? sigmoidf_(__bfloat162float(r.e)) * (1.0f / D) : 0.f;
      sGate[(x & (kSR - 1)) * CB + i] = ggl ? sigmoidf_(__bfloat162float(r.g)) : 1.f;
      if (i == 0) sFlag[x & (kSR - 1)] = r.m ? 1 : 0;
    }
  };
  int tma_issued = 0;  // chunks [0, tma_issued) loaded or loading (MMA thread's count)
  int w_issued = 0;    // commits to bar_w (MMA thread's count)
  auto issue_tma = [&](int c) {
    uint64_t* bar = &bar_tma[c & (NST - 1)];
    mbar_arrive_expect_tx(bar, 3 * kTile);
    tma_load_3d(tK(c), &maps.k, bar, 0, c * CB, (int)bh);
    tma_load_3d(tQ(c), &maps.q, bar, 0, c * CB, (int)bh);
    tma_load_3d(tV(c), &maps.v, bar, 0, c * CB, (int)bh);
    tma_issued = c + 1;
  };
  auto tma_parity = [&](int c) { return (uint32_t)((c >> 2) & 1); };
  const uint32_t idescN16 = idesc_bf16_f32(128, 16, false, false);
  const uint32_t idescW = idesc_bf16_f32(128, 64, false, true);
  const uint32_t aWb = smem_u32(sWb);
  // W_s . R^T for 16 rows R (K-major, SW128) into TMEM column `col`
  auto mma_ws_rows = [&](uint32_t tmem, uint32_t col, const unsigned char* rows) {
    const uint32_t ar = smem_u32(rows);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16_ss(tmem + col, smem_desc(aWb + kk * 32, 16, 1024, kLayoutSw128),
                  smem_desc(ar + kk * 32, 16, 1024, kLayoutSw128), idescN16, kk > 0 ? 1u : 0u);
  };
  // Gram products on the tensor core (thread 128): with a 128-row A operand
  // that starts at a 16-row tile (rows 16-127 read whatever follows in shared
  // memory and land in TMEM lanes that are never read),
  //   lanes 0-15, cols 0-15 : k_{cx,m} . k_{cx-1,j}   (X before eta)
  //   lanes 0-15, cols 16-31: q_{cm,i} . k_{cm,j}      (M before the causal mask)
  auto gram_issue = [&](uint32_t tmem2, int cx, int cm) {
    if (cx < nc) {
      const uint32_t a = smem_u32(tK(cx)), b = smem_u32(tK(cx - 1));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tmem2, smem_desc(a + kk * 32, 16, 1024, kLayoutSw128),
                    smem_desc(b + kk * 32, 16, 1024, kLayoutSw128), idescN16, kk > 0 ? 1u : 0u);
    }
    if (cm < nc) {
      const uint32_t a = smem_u32(tQ(cm)), b = smem_u32(tK(cm));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tmem2 + 16, smem_desc(a + kk * 32, 16, 1024, kLayoutSw128),
                    smem_desc(b + kk * 32, 16, 1024, kLayoutSw128), idescN16, kk > 0 ? 1u : 0u);
    }
    mma_commit(bar_gram);
  };
  // warp with TMEM lane quarter 0 (lanes 0-15 hold the rows): X_{cx} (eta-weighted,
  // fp32) and M_{cm} (causal, bf16 in the B-operand layout) into shared memory
  auto gram_extract = [&](uint32_t tmem2, int cx, int cm) {
    float xr[16], mr[16];
    tmem_ld16(tmem2, xr);
    tmem_ld16(tmem2 + 16, mr);
    tmem_wait_ld();
    if (lane < CB) {
      if (cx < nc) {
        const float* et = sEta + ((cx - 1) & (kSR - 1)) * CB;
        const int n1 = chunk_len(cx), n0 = chunk_len(cx - 1);
        float* X = sX + (cx & 1) * CB * CB + lane * CB;
#pragma unroll
        for (int j = 0; j < CB; j += 4) {
          float4 v;
          v.x = (lane < n1 && j + 0 < n0) ? et[j + 0] * xr[j + 0] : 0.f;
          v.y = (lane < n1 && j + 1 < n0) ? et[j + 1] * xr[j + 1] : 0.f;
          v.z = (lane < n1 && j + 2 < n0) ? et[j + 2] * xr[j + 2] : 0.f;
          v.w = (lane < n1 && j + 3 < n0) ? et[j + 3] * xr[j + 3] : 0.f;
          *reinterpret_cast<float4*>(X + j) = v;
        }
      }
      if (cm < nc) {
        const int n = chunk_len(cm);
        const int i = lane;
        unsigned char* Mt = mmat(cm);
#pragma unroll
        for (int j0 = 0; j0 < CB; j0 += 8) {
          uint4 u;
          float m8[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) m8[jj] = (j0 + jj <= i && i < n) ? mr[j0 + jj] : 0.f;
          u.x = pack_bf16(m8[0], m8[1]);
          u.y = pack_bf16(m8[2], m8[3]);
          u.z = pack_bf16(m8[4], m8[5]);
          u.w = pack_bf16(m8[6], m8[7]);
          *reinterpret_cast<uint4*>(Mt + core_off(i, j0)) = u;
        }
        fence_proxy_async_smem();
      }
    }
  };
  auto fail = [&]() {
    if (gt == 0) {
      *sAbort = 1;
      atomicExch(&g_ttt_status, (int)kStatusTimeout);
    }
  };

  // =========================== prologue ===========================
  if (warp == 0) {
    tmem_alloc(sTmem, kTmemCols);
    tmem_alloc(sTmem + 1, kTmemGramCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) mbar_init(&bar_tma[s], 1);
    mbar_init(&bar_px[0], 129);  // 128 bulk threads (X written) + the MMA commit
    mbar_init(&bar_px[1], 129);
    mbar_init(&bar_g[0], 128);   // 128 chain threads
    mbar_init(&bar_g[1], 128);
    mbar_init(bar_w, 1);
    mbar_init(bar_pro, 1);
    mbar_init(bar_gram, 1);
    mbar_init_fence();
    *sAbort = 0;
  }
  if (!chain) {
    store_block(0, fetch_block(0));
    store_block(8, fetch_block(8));
  } else if (gt < D) {
    sGam[gt] = p.no_ln ? 1.f : p.gamma[(size_t)h * D + gt];
    sBet[gt] = p.no_ln ? 0.f : p.beta[(size_t)h * D + gt];
  }
  // chain threads, token-major role: token tm_m, features tm_p + 8u
  const int tm_m = gt >> 3, tm_p = gt & 7;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sTmem[0];
  const uint32_t tmem2 = sTmem[1];
  if (mma_thread) {
    prefetch_tensormap(&maps.q);
    prefetch_tensormap(&maps.k);
    prefetch_tensormap(&maps.v);
    for (int c = 0; c < NST && c < nc; ++c) issue_tma(c);
  }
  if (!chain) {
    // W0 -> TMEM (both row copies, lanes 0-127) and the bf16 operand W_s
    const int row = wq * 32 + lane;
    const float* src = p.W0 + ((size_t)bh * D + (row & 63)) * D;  // may alias W_T
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float w[32];
#pragma unroll
      for (int k = 0; k < 32; k += 4) {
        const float4 w4 = *reinterpret_cast<const float4*>(src + 32 * hf + k);
        w[k] = w4.x; w[k + 1] = w4.y; w[k + 2] = w4.z; w[k + 3] = w4.w;
      }
      tmem_st32(tmem + tlane + kColW + 32 * hf, w);
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint4 u;
        u.x = pack_bf16(w[8 * ch + 0], w[8 * ch + 1]);
        u.y = pack_bf16(w[8 * ch + 2], w[8 * ch + 3]);
        u.z = pack_bf16(w[8 * ch + 4], w[8 * ch + 5]);
        u.w = pack_bf16(w[8 * ch + 6], w[8 * ch + 7]);
        *reinterpret_cast<uint4*>(sWb + sw128_off(row, 4 * hf + ch)) = u;
      }
      if (Wc && row < 64) {
        float* dst = Wc + (size_t)row * D + 32 * hf;
#pragma unroll
        for (int k = 0; k < 32; k += 4)
          *reinterpret_cast<float4*>(dst + k) = make_float4(w[k], w[k + 1], w[k + 2], w[k + 3]);
      }
    }
    tmem_wait_st();
    fence_proxy_async_smem();
  }
  // tiles of chunks 0 and 1, then X_1 and M_0
  bool bad = false;
  if (nc > 0 && !mbar_wait_bounded(&bar_tma[0], 0, lim)) bad = true;
  if (nc > 1 && !mbar_wait_bounded(&bar_tma[1], 0, lim)) bad = true;
  tc_fence_before();
  const bool pro_bad = __syncthreads_or(bad);
  if (pro_bad && tid == 0) {
    *sAbort = 1;
    atomicExch(&g_ttt_status, (int)kStatusTimeout);
  }
  tc_fence_after();
  if (mma_thread && !pro_bad) {
    // Grams X_1, M_0; delivery 0 = {P_0} in slot 0; delivery 1 = {P_1, Q0_0} in slot 1
    gram_issue(tmem2, 1, 0);
    mma_ws_rows(tmem, col_p(0), tK(0));
    if (nc > 1) mma_ws_rows(tmem, col_p(1), tK(1));
    mma_ws_rows(tmem, col_o(1), tQ(0));
    mma_commit(bar_pro);
  }
  if (warp == 4 && !pro_bad) {
    if (mbar_wait_bounded(bar_gram, 0, lim)) {
      tc_fence_after();
      gram_extract(tmem2, 1, 0);
    } else if (lane == 0) {
      *sAbort = 1;
      atomicExch(&g_ttt_status, (int)kStatusTimeout);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const bool run = !*sAbort;
  __syncthreads();

  if (chain && run) {
    // =========================== chain group ===========================
    bool prev_upd = false;
    for (int k = 0; k < nc; ++k) {
      const int n = chunk_len(k);
      const bool upd = sFlag[k & (kSR - 1)] != 0;
      // ---- wait for delivery k (P_k, X_k) ----
      bool ok;
      if (k < 2) ok = mbar_wait_bounded(bar_pro, 0, lim);
      else ok = mbar_wait_bounded(&bar_px[k & 1], (uint32_t)(((k - 2) >> 1) & 1), lim);
      if (group_any(kBarChain, !ok || *sAbort)) {
        fail();
        break;
      }
      tc_fence_after();
      if (upd) {
        // ---- correction, feature-major: Z_k[m][f] = P_k[f][m] - sum_j X_k[m][j] G_{k-1}[j][f] ----
        float z[8];
        tmem_ld8(tmem + tlane + col_p(k & 1) + 8 * half, z);
        tmem_wait_ld();
        if (k >= 1 && prev_upd) {
          // X rows are zero past the previous chunk's length, so all 16 columns run
          const float* X = sX + (k & 1) * CB * CB + 8 * half * CB;
          const float* Gp = sG + ((k - 1) & 1) * CB * kZS + fm;
#pragma unroll
          for (int j4 = 0; j4 < CB; j4 += 4) {
            float g[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) g[jj] = Gp[(j4 + jj) * kZS];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float4 x4 = *reinterpret_cast<const float4*>(X + u * CB + j4);
              z[u] = fmaf(-x4.x, g[0], z[u]);
              z[u] = fmaf(-x4.y, g[1], z[u]);
              z[u] = fmaf(-x4.z, g[2], z[u]);
              z[u] = fmaf(-x4.w, g[3], z[u]);
            }
          }
        }
        float* Zk = sZ + (k & 1) * CB * kZS + 8 * half * kZS + fm;
#pragma unroll
        for (int u = 0; u < 8; ++u) Zk[u * kZS] = z[u];
      }
      group_sync(kBarChain);
      if (upd) {
        // ---- token-major LayerNorm + gradient: token tm_m, features tm_p + 8u ----
        const float* Zk = sZ + (k & 1) * CB * kZS + tm_m * kZS;
        const unsigned char* Vt = tV(k) + tm_m * D * 2;
        float z[8], v[8], G[8], gam[8], bet[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int f = tm_p + 8 * u;
          z[u] = Zk[f];
          v[u] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(Vt + f * 2));
          gam[u] = sGam[f];
          bet[u] = sBet[f];
        }
        if (GM == 2) {
#pragma unroll
          for (int u = 0; u < 8; ++u) G[u] = z[u] - v[u];
        } else {
          float s = 0.f;
#pragma unroll
          for (int u = 0; u < 8; ++u) s += z[u];
          s += __shfl_xor_sync(0xffffffffu, s, 1);
          s += __shfl_xor_sync(0xffffffffu, s, 2);
          s += __shfl_xor_sync(0xffffffffu, s, 4);
          const float mu = s * (1.0f / D);
          float y[8], s2 = 0.f;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            y[u] = z[u] - mu;
            s2 = fmaf(y[u], y[u], s2);
          }
          s2 += __shfl_xor_sync(0xffffffffu, s2, 1);
          s2 += __shfl_xor_sync(0xffffffffu, s2, 2);
          s2 += __shfl_xor_sync(0xffffffffu, s2, 4);
          const float rs = rsqrtf(fmaf(s2, 1.0f / D, p.eps));
          float xh[8], err[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            xh[u] = y[u] * rs;
            err[u] = fmaf(gam[u], xh[u], bet[u]) - v[u];
          }
          if (GM == 1) {
            float a = 0.f, b = 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float g = gam[u] * err[u];
              a += g;
              b = fmaf(g, xh[u], b);
            }
            a += __shfl_xor_sync(0xffffffffu, a, 1);
            b += __shfl_xor_sync(0xffffffffu, b, 1);
            a += __shfl_xor_sync(0xffffffffu, a, 2);
            b += __shfl_xor_sync(0xffffffffu, b, 2);
            a += __shfl_xor_sync(0xffffffffu, a, 4);
            b += __shfl_xor_sync(0xffffffffu, b, 4);
            const float mg = a * (1.0f / D), mgx = b * (1.0f / D);
#pragma unroll
            for (int u = 0; u < 8; ++u) G[u] = (gam[u] * err[u] - mg - xh[u] * mgx) * rs;
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) G[u] = err[u];
          }
        }
        if (tm_m >= n) {
#pragma unroll
          for (int u = 0; u < 8; ++u) G[u] = 0.f;
        }
        const float eta = sEta[(k & (kSR - 1)) * CB + tm_m];
        float* Gk = sG + (k & 1) * CB * kZS + tm_m * kZS;
        unsigned char* An = aneg(k);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int f = tm_p + 8 * u;
          Gk[f] = G[u];
          const __nv_bfloat16 a = __float2bfloat16_rn(-eta * G[u]);
          *reinterpret_cast<__nv_bfloat16*>(An + core_off(f, tm_m)) = a;
          *reinterpret_cast<__nv_bfloat16*>(An + core_off(f + 64, tm_m)) = a;
        }
        fence_proxy_async_smem();
      }
      prev_upd = upd;
      tc_fence_before();  // TMEM reads of P_k done before the bulk may overwrite its slot
      mbar_arrive(&bar_g[k & 1]);
      group_sync(kBarChain);  // G_k visible to the next correction
    }
  } else if (!chain && run) {
    // =========================== bulk group ===========================
    Raw pre{};
    for (int c = 0; c < nc; ++c) {
      const bool upd = sFlag[c & (kSR - 1)] != 0;
      if ((c & 7) == 0) pre = fetch_block(c + 16);
      // ---- tiles of chunk c+2, then the Gram MMAs for X_{c+2}, M_{c+1} ----
      bool ok = true;
      if (c + 2 < nc) ok = mbar_wait_bounded(&bar_tma[(c + 2) & (NST - 1)], tma_parity(c + 2), lim);
      tc_fence_before();
      if (group_any(kBarBulk, !ok || *sAbort)) {
        fail();
        break;
      }
      if (mma_thread) {
        tc_fence_after();
        gram_issue(tmem2, c + 2, c + 1);
      }
      // ---- wait for G_c / Aneg_c ----
      ok = mbar_wait_bounded(&bar_g[c & 1], (uint32_t)((c >> 1) & 1), lim);
      tc_fence_before();
      if (group_any(kBarBulk, !ok || *sAbort)) {
        fail();
        break;
      }
      // ---- MMA2 (outputs) + MMA3 (W update), or just a commit ----
      if (mma_thread) {
        tc_fence_after();
        if (upd) {
          const uint64_t da = smem_desc(smem_u32(aneg(c)), 128, 256, kLayoutNone);
          mma_bf16_ss(tmem + col_o((c + 1) & 1), da,
                      smem_desc(smem_u32(mmat(c)), 128, 256, kLayoutNone), idescN16, 1u);
          mma_bf16_ss(tmem + kColW, da, smem_desc(smem_u32(tK(c)), 2048, 1024, kLayoutSw128),
                      idescW, 1u);
        }
        mma_commit(bar_w);
        ++w_issued;
      }
      ok = mbar_wait_bounded(bar_w, (uint32_t)(c & 1), lim);
      tc_fence_before();
      if (group_any(kBarBulk, !ok || *sAbort)) {
        fail();
        break;
      }
      tc_fence_after();
      // ---- W_{s,c+1} (fp32 TMEM) -> bf16 operand; snapshot ----
      const int row = wq * 32 + lane;
      if (upd) {
#pragma unroll
        for (int qt = 0; qt < 4; ++qt) {
          float w[16];
          tmem_ld16(tmem + tlane + kColW + 16 * qt, w);
          tmem_wait_ld();
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            uint4 u;
            u.x = pack_bf16(w[8 * ch + 0], w[8 * ch + 1]);
            u.y = pack_bf16(w[8 * ch + 2], w[8 * ch + 3]);
            u.z = pack_bf16(w[8 * ch + 4], w[8 * ch + 5]);
            u.w = pack_bf16(w[8 * ch + 6], w[8 * ch + 7]);
            *reinterpret_cast<uint4*>(sWb + sw128_off(row, 2 * qt + ch)) = u;
          }
          if (Wc && row < 64) {
            float* dst = Wc + ((size_t)(c + 1) * D + row) * D + 16 * qt;
#pragma unroll
            for (int k = 0; k < 16; k += 4)
              *reinterpret_cast<float4*>(dst + k) = make_float4(w[k], w[k + 1], w[k + 2], w[k + 3]);
          }
        }
        fence_proxy_async_smem();
      } else if (Wc && row < 64) {
        // W unchanged: the next snapshot repeats this one
        const float* srcw = Wc + ((size_t)c * D + row) * D;
        float* dst = Wc + ((size_t)(c + 1) * D + row) * D;
        for (int k = 0; k < 64; k += 4)
          *reinterpret_cast<float4*>(dst + k) = *reinterpret_cast<const float4*>(srcw + k);
      }
      // ---- Gram results -> X_{c+2}, M_{c+1} ----
      if (wq == 0) {
        ok = mbar_wait_bounded(bar_gram, (uint32_t)((c + 1) & 1), lim);
        if (ok) {
          tc_fence_after();
          gram_extract(tmem2, c + 2, c + 1);
        }
      }
      tc_fence_before();
      if (group_any(kBarBulk, !ok || *sAbort)) {  // W_s bf16 and M_{c+1} written
        fail();
        break;
      }
      // ---- MMA1: delivery c+2 = {P_{c+2}, Q0_{c+1}} into slot (c+2) & 1 ----
      if (mma_thread) {
        tc_fence_after();
        if (c + 2 < nc) mma_ws_rows(tmem, col_p((c + 2) & 1), tK(c + 2));
        if (c + 1 < nc) mma_ws_rows(tmem, col_o((c + 2) & 1), tQ(c + 1));
        if (c + 2 < nc) mma_commit(&bar_px[(c + 2) & 1]);
      }
      if (c + 2 < nc) mbar_arrive(&bar_px[(c + 2) & 1]);
      // ---- outputs o_c = gate * O_c^T ----
      {
        float ov[8];
        tmem_ld8(tmem + tlane + col_o((c + 1) & 1) + 8 * half, ov);
        tmem_wait_ld();
        const float* gte = sGate + (c & (kSR - 1)) * CB + 8 * half;
        const int n = chunk_len(c);
        OutT* dst = go + (size_t)c * CB * D;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int t = 8 * half + u;
          if (t < n) dst[(size_t)t * D + fm] = from_f32<OutT>(gte[u] * ov[u]);
        }
      }
      // ---- refill stage c & 3 with chunk c + 4, scalars of chunk c + 4 ----
      if (mma_thread && c + NST < nc) {
        fence_proxy_async_smem();
        issue_tma(c + NST);
      }
      if ((c & 7) == 4) store_block(c + 12, pre);
    }
  }

  // =========================== teardown ===========================
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*sAbort) {
    if (mma_thread) {
      // all MMAs this thread issued (one commit tracks them all), then every
      // TMA stage that may still be loading; each wait has its own bound
      mma_commit(bar_w);
      if (w_issued > 0) mbar_wait_bounded(bar_w, (uint32_t)((w_issued - 1) & 1), drain_lim);
      mbar_wait_bounded(bar_w, (uint32_t)(w_issued & 1), drain_lim);
      for (int c = (tma_issued > NST ? tma_issued - NST : 0); c < tma_issued; ++c)
        mbar_wait_bounded(&bar_tma[c & (NST - 1)], tma_parity(c), drain_lim);
    }
  } else if (!chain && wq < 2) {
    // W_T (rows of copy 0)
    const int row = wq * 32 + lane;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float w[32];
      tmem_ld32(tmem + tlane + kColW + 32 * hf, w);
      tmem_wait_ld();
      float* dst = p.W_T + ((size_t)bh * D + row) * D + 32 * hf;
#pragma unroll
      for (int k = 0; k < 32; k += 4)
        *reinterpret_cast<float4*>(dst + k) = make_float4(w[k], w[k + 1], w[k + 2], w[k + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    tmem_dealloc(tmem, kTmemCols);
    tmem_dealloc(tmem2, kTmemGramCols);
  }
}

}  // namespace ttt
