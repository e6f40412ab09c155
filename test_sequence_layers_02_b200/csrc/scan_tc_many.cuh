// Tensor-core (tcgen05) mini-batch scan built for three CTAs per SM: d = 64,
// b = 16, bf16 q/k/v/logits, fp32 state W in TMEM, bf16 or fp32 outputs.
//
// The launcher takes this kernel when a launch has between two and three heads
// per SM: it needs 160 TMEM columns and under 75 KB of shared memory per CTA,
// so three heads share an SM and the launch runs in one wave. The kernel of
// scan_tc.cuh (two-chunk look-ahead, a Gram warp, deeper TMA staging) has a
// shorter chunk loop but fits only two CTAs per SM.
//
// Chunk step (PonderTTT, "Technical Architecture": dual-form updates; every
// gradient of a chunk taken at the chunk-start state W_s):
//     z_i = W_s k_i,  G_i = LayerNorm gradient ("Error Correction in Trained
//     TTT Layers", Abstract),  o_i = W_s q_i - sum_{j<=i} eta_j (k_j.q_i) G_j,
//     W_e = W_s - sum_j eta_j G_j k_j^T.
//
// Look-ahead. With Aneg_c[f][j] = -eta_j G_j[f] and W_{s,c+1} = W_{s,c} + Aneg_c K_c,
//     Z_{c+1}^T = W_{s,c+1} K_{c+1}^T = P_{c+1}^T + Aneg_c Xg_{c+1}^T,
//     P_{c+1}^T = W_{s,c} K_{c+1}^T,   Xg_{c+1}[m][j] = k_{c+1,m} . k_{c,j},
// so P_{c+1} comes from the tensor core a chunk early and the correction is
// one more small MMA accumulated into the same TMEM columns. Between two
// LayerNorms only: the chain's Aneg -> three MMAs -> TMEM read of the next Z.
//
// Warps (288 threads):
//   chain 0-3   read Z_k^T (TMEM, feature-major), transpose through shared
//               memory, token-major LayerNorm + gradient (8 lanes per token,
//               one shuffle round of shifted moments), write Aneg_k (bf16).
//   bulk 4-7    W (fp32 TMEM) -> bf16 operand W_s; Gram products two chunks
//               ahead -> bf16 operand [Xg_{c+3}; M_{c+2}]; outputs o_c = gate * O_c^T;
//               per-chunk scalars; one thread issues every TMA load of chunk
//               x = {K_x, Q_{x-1}, V_x}, NST chunks ahead.
//   issuer 8    (one thread) every tcgen05.mma, per chunk c in this order:
//               MMAc [P_{c+1} | O_c]^T += Aneg_c [Xg_{c+1}; M_c]^T (one N = 32 MMA,
//               committed alone: the chain's next Z waits for nothing else);
//               MMA3 W += Aneg_c K_c (K as an MN-major operand); the Gram
//               [K_{c+3}; Q_{c+2}] K_{c+2}^T; once W_s is refreshed, MMA1
//               [P_{c+2} | Q0_{c+1}]^T = W_s [K_{c+2}; Q_{c+1}]^T.
// One chunk period is then the longer of two loops from MMAc: the chain's
// (Z -> LayerNorm -> Aneg) and the W refresh's (MMA3 -> bf16 W_s -> MMA1,
// which must precede the next MMAc); the Grams and the outputs stay off both.
// M = 128 everywhere: A operands stack two copies of their 64 rows, so TMEM
// lanes 0-63 and 64-127 hold identical d-row results and every warp quarter
// reads its own lanes.
//
// Handoffs are mbarriers in rings of two (a producer can never run two phases
// ahead of its consumer). Every wait is bounded: on expiry the CTA records the
// timeout status, all warps leave their loops, the issuer drains its MMAs and
// the TMA thread its copies (each with a bound of its own) and TMEM is freed.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace ttt {
namespace tcm {

// Set to a nonzero code by a kernel whose bounded wait gave up; read and
// cleared through tc_many_status_take(). One word per device, allocated with
// the module of the one translation unit that includes this header.
__device__ int g_tcm_status;

struct TcMaps {
  CUtensorMap q, k, v;  // [B*H][T][64] bf16 as {64, T, B*H}, box {64, 16, 1}
  CUtensorMap o;        // [B*H][T][64] of the output type, the same view and box
};

namespace tc {

constexpr int D = 64;
constexpr int CB = 16;              // chunk (b)
constexpr int NT = 288;             // 4 chain + 4 bulk + 1 issuer warps
constexpr int kMinbMany = 3;        // CTAs per SM of the build for more heads than SMs
constexpr int NST = 5;              // TMA stages
constexpr int kSR = 32;             // scalar ring (chunks)
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kTmemGramCols = 32;
constexpr uint32_t kColW = 0;       // W accumulator (64 columns)
// slot s = 0, 1: [P^T | Q0^T / O^T] at 64 + 32 s (16 + 16 columns); the Gram
// of chunk x in columns 16 (x & 1) of the second allocation
__device__ __forceinline__ uint32_t col_p(int s) { return 64u + 32u * (uint32_t)s; }
__device__ __forceinline__ uint32_t col_o(int s) { return 80u + 32u * (uint32_t)s; }
constexpr int kTile = CB * D * 2;   // 2048 bytes
constexpr int kZS = 72;             // row stride (floats) of the token-major Z tile

// shared memory (bytes from a 1024-aligned base)
constexpr int oKQ = 0;                             // [NST][K_x | Q_{x-1}] 128B-swizzled
constexpr int oV = oKQ + NST * 2 * kTile;          // [NST] V_x, row-major
constexpr int oWb = oV + NST * kTile;              // W_s bf16, 128 rows x 128 B, 128B-swizzled
constexpr int oAneg = oWb + 128 * 128;             // [2] 128 rows x 16 bf16 (core matrices)
constexpr int oXM = oAneg + 2 * 128 * 32;          // [2] [Xg_{x+1}; M_x] 32 x 16 bf16 (core matrices)
constexpr int oZ = oXM + 2 * 1024;                 // [2][16][kZS] f32
constexpr int oEta = oZ + 2 * CB * kZS * 4;        // [kSR][16] f32 (mask folded in)
constexpr int oGate = oEta + kSR * CB * 4;         // [kSR][16] f32
constexpr int oFlag = oGate + kSR * CB * 4;        // [kSR] int
constexpr int oGam = oFlag + kSR * 4;              // gamma, beta [2][64] f32, sum gamma^2, sum gamma*beta
constexpr int oBar = oGam + 2 * D * 4 + 16;        // mbarriers
// tma[NST], g[2], z[2], xm[2], w, wb, gram, pro, rdy[NST]
constexpr int kBars = NST + 2 + 2 + 2 + 4 + NST;
constexpr int oTmem = oBar + kBars * 8;            // two TMEM base addresses
constexpr int oAbort = oTmem + 8;
// [2][16][64] bf16 outputs (bf16 output only), TMA-stored a chunk later; a
// tensor copy's shared-memory operand starts on 128 bytes
constexpr int oOut = (oAbort + 4 + 127) & ~127;
constexpr int kSmemUsed = oOut + 2 * CB * D * 2;
static_assert(oOut % 128 == 0 && (CB * D * 2) % 128 == 0, "TMA store source on 128 bytes");
constexpr int kSmemBytes = kSmemUsed + 1024;       // + alignment slack
static_assert(kSmemBytes <= 75 * 1024, "three CTAs per SM must fit in shared memory");
template <int MINB>
constexpr int smem_bytes() { return kSmemBytes; }
static_assert(oWb % 1024 == 0, "128B-swizzled operands are 1024-aligned");
static_assert(3 * (kTmemCols + kTmemGramCols) <= 512, "three CTAs per SM must fit in TMEM");
// The 128-row A operand of the Gram MMA starts at a stage's K tile and runs
// 16 KB forward: it must stay inside this CTA's shared memory.
static_assert(oKQ + (NST - 1) * 2 * kTile + 128 * 128 <= kSmemUsed, "Gram operand in bounds");

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
// Barrier over `count` threads of a named barrier that returns whether any
// member passed true.
__device__ __forceinline__ bool bar_any(int bar_id, int count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.b32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.b32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((int)v), "r"(bar_id), "r"(count)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bar_sync(int bar_id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(sm100::smem_u32(bar))
               : "memory");
}
constexpr int kBarChain = 2;  // named barriers (0 is __syncthreads)
constexpr int kBarBulk = 3;

}  // namespace tc

// MINB = 3: three CTAs share an SM (heads above the SM count; 72 registers);
// MINB = 1: one CTA per SM, for up to one head per SM (more registers).
template <typename OutT, int GM, int MINB>
__global__ void __launch_bounds__(tc::NT, MINB)
    scan_tc_kernel(const ScanParams p, const __grid_constant__ TcMaps maps) {
  using namespace tc;
  using namespace sm100;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sWb = smem + oWb;
  float* sZ = reinterpret_cast<float*>(smem + oZ);
  float* sEta = reinterpret_cast<float*>(smem + oEta);
  float* sGate = reinterpret_cast<float*>(smem + oGate);
  int* sFlag = reinterpret_cast<int*>(smem + oFlag);
  float* sGam = reinterpret_cast<float*>(smem + oGam);
  float* sBet = sGam + D;
  float* sGamSums = sGam + 2 * D;  // [0] sum gamma^2, [1] sum gamma*beta
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(smem + oBar);  // [NST] chunk x -> x % NST
  uint64_t* bar_g = bar_tma + NST;   // [2] Aneg_k written (chain, 128 arrivals)
  uint64_t* bar_z = bar_g + 2;       // [2] Z_k complete in TMEM (commit)
  uint64_t* bar_xm = bar_z + 2;      // [2] [Xg_{x+1}; M_x] written (bulk warp 4, 32 arrivals)
  uint64_t* bar_w = bar_xm + 2;      // a chunk's MMAc and MMA3 complete (commit)
  uint64_t* bar_wb = bar_w + 1;      // W_s bf16 refreshed (bulk, 128 arrivals)
  uint64_t* bar_gram = bar_wb + 1;   // Gram MMA complete (commit)
  uint64_t* bar_pro = bar_gram + 1;  // prologue MMAs complete (commit)
  // [NST] stage x ready for the MMAs: with the SiLU variant, K_x and Q_{x-1}
  // transformed in place (bulk, 128 arrivals); otherwise the TMA barrier is used
  uint64_t* bar_rdy = bar_pro + 1;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + oTmem);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + oAbort);
  auto tKQ = [&](int x) { return smem + oKQ + (x % NST) * 2 * kTile; };  // K_x, then Q_{x-1}
  auto tV = [&](int x) { return smem + oV + (x % NST) * kTile; };
  auto aneg = [&](int c) { return smem + oAneg + (c & 1) * 4096; };
  auto xm = [&](int x) { return smem + oXM + (x & 1) * 1024; };  // [Xg_{x+1}; M_x]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const bool is_chain = warp < 4;
  const bool is_bulk = warp >= 4 && warp < 8;
  const bool issuer = (tid == 256);
  const bool tma_thread = (tid == 224);        // bulk warp 7, lane 0
  const int wq = warp & 3;                     // TMEM lane quarter of this warp
  const uint32_t tlane = (uint32_t)(wq * 32) << 16;
  const int fm = (wq & 1) * 32 + lane;         // feature-major role: feature
  const int half = wq >> 1;                    // feature-major role: tokens 8*half .. +8
  const int gt = tid & 127;
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
  // bf16 outputs go through a shared-memory tile and a TMA store (one thread,
  // one store per chunk, issued after the next chunk's first bulk barrier);
  // fp32 outputs (whose tile would not fit three CTAs per SM) are stored directly
  constexpr bool kTileOut = sizeof(OutT) == 2;
  auto out_tile = [&](int x) {
    return reinterpret_cast<OutT*>(smem + oOut) + (x & 1) * CB * D;
  };
  float* Wc = p.W_chunks ? p.W_chunks + (size_t)bh * (p.n_mask_chunks + 1) * D * D : nullptr;
  const long long lim = p.wait_limit;
  const long long drain_lim = 1LL << 24;
  auto chunk_len = [&](int c) { return min(CB, T - c * CB); };
  auto fail = [&]() {
    *sAbort = 1;
    atomicExch(&g_tcm_status, (int)kStatusTimeout);
  };

  // ---- per-chunk scalars in a ring of kSR chunks, loaded by the bulk warps
  // in blocks of 8 chunks, 16 chunks ahead; raw values wait in registers ----
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
        r.e = gel[t];  // (read whatever the mask says: a load that waited for the
                       // mask byte would stall these warps once per 8 chunks)
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

  // ---- issuer helpers ----
  int tma_issued = 0;  // TMA loads [0, tma_issued) issued (chunk x = {K_x, Q_{x-1}, V_x})
  int w_issued = 0;    // commits to bar_w
  // A SKIP chunk's keys and values are never used (its z, gradient and update
  // are not formed), so only its queries are loaded; the K_x / V_x slots keep
  // stale data that only reaches TMEM columns nobody reads (P_x; the Gram rows
  // of Xg_x and M_x are zeroed by gram_extract).
  auto issue_tma = [&](int x) {
    uint64_t* bar = &bar_tma[x % NST];
    const bool kv = x < nc && sFlag[x & (kSR - 1)] != 0;
    const uint32_t bytes = (kv ? 2 * kTile : 0) + (x >= 1 ? kTile : 0);
    mbar_arrive_expect_tx(bar, bytes);
    if (kv) {
      tma_load_3d(tKQ(x), &maps.k, bar, 0, x * CB, (int)bh);
      tma_load_3d(tV(x), &maps.v, bar, 0, x * CB, (int)bh);
    }
    if (x >= 1) tma_load_3d(tKQ(x) + kTile, &maps.q, bar, 0, (x - 1) * CB, (int)bh);
    tma_issued = x + 1;
  };
  auto tma_parity = [&](int x) { return (uint32_t)((x / NST) & 1); };
  // stage x ready for the MMAs (see bar_rdy)
  auto wait_stage = [&](int x) {
    return mbar_wait_bounded(p.kq_silu ? &bar_rdy[x % NST] : &bar_tma[x % NST], tma_parity(x),
                             lim);
  };
  // The `:mlp` variant: SiLU in place on stage x (K_x and Q_{x-1}; bulk
  // threads, 32 bytes each). The operands stay bf16, as the MMAs read them.
  auto silu_stage = [&](int x) {
    unsigned char* st = tKQ(x);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      uint4* ptr = reinterpret_cast<uint4*>(st + (gt + 128 * u) * 16);
      uint4 w = *ptr;
      uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        wv[e] = pack_bf16(siluf_(__uint_as_float(wv[e] << 16)),
                          siluf_(__uint_as_float(wv[e] & 0xffff0000u)));
      *ptr = w;
    }
    fence_proxy_async_smem();
  };
  const uint32_t idescN16 = idesc_bf16_f32(128, 16, false, false);
  const uint32_t idescN32 = idesc_bf16_f32(128, 32, false, false);
  const uint32_t idescW = idesc_bf16_f32(128, 64, false, true);
  const uint32_t aWb = smem_u32(sWb);
  // D (+)= W_s . R^T, R = `n` rows (16 or 32) of a 128B-swizzled K-major tile
  auto mma_ws = [&](uint32_t d, const unsigned char* rows, int n) {
    const uint32_t ar = smem_u32(rows);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16_ss(d, smem_desc(aWb + kk * 32, 16, 1024, kLayoutSw128),
                  smem_desc(ar + kk * 32, 16, 1024, kLayoutSw128), n == 32 ? idescN32 : idescN16,
                  kk > 0 ? 1u : 0u);
  };
  // Gram for chunk x into TMEM columns 16 (x & 1) of the second allocation:
  // A = [K_{x+1}; Q_x] (stage x+1; the 128-row operand reads on into the
  // following shared memory, whose rows land in TMEM lanes that are never
  // read), B = K_x:  lanes 0-15 k_{x+1,m}.k_{x,j}, lanes 16-31 q_{x,i}.k_{x,j}
  auto mma_gram = [&](uint32_t tmem2, int x) {
    const uint32_t a = smem_u32(tKQ(x + 1)), b = smem_u32(tKQ(x));
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16_ss(tmem2 + 16u * (uint32_t)(x & 1), smem_desc(a + kk * 32, 16, 1024, kLayoutSw128),
                  smem_desc(b + kk * 32, 16, 1024, kLayoutSw128), idescN16, kk > 0 ? 1u : 0u);
  };
  // bulk warp with TMEM lane quarter 0: Gram rows -> the 32-row operand
  // [Xg_{x+1}; M_x] (bf16): rows 0-15 Xg_{x+1}[m][j] (zero past the chunk
  // lengths), rows 16-31 M_x[i][j] (causal), row = lane
  auto gram_extract = [&](uint32_t tmem2, int x) {
    float r[16];
    tmem_ld16(tmem2 + 16u * (uint32_t)(x & 1), r);
    tmem_wait_ld();
    // Xg_{x+1} and M_x are used only when chunk x updates (Xg also needs
    // chunk x+1 to update); the rows of a SKIP chunk are zero, which also
    // discards the stale keys its stage holds
    const int n0 = sFlag[x & (kSR - 1)] ? chunk_len(x) : 0;
    float v[16];
    if (lane < CB) {
      const int n1 = (x + 1 < nc && sFlag[(x + 1) & (kSR - 1)]) ? chunk_len(x + 1) : 0;
#pragma unroll
      for (int j = 0; j < CB; ++j) v[j] = (lane < n1 && j < n0) ? r[j] : 0.f;
    } else {
      const int i = lane - CB;
#pragma unroll
      for (int j = 0; j < CB; ++j) v[j] = (j <= i && i < n0) ? r[j] : 0.f;
    }
    unsigned char* dst = xm(x);
#pragma unroll
    for (int j0 = 0; j0 < CB; j0 += 8) {
      uint4 u;
      u.x = pack_bf16(v[j0 + 0], v[j0 + 1]);
      u.y = pack_bf16(v[j0 + 2], v[j0 + 3]);
      u.z = pack_bf16(v[j0 + 4], v[j0 + 5]);
      u.w = pack_bf16(v[j0 + 6], v[j0 + 7]);
      *reinterpret_cast<uint4*>(dst + core_off(lane, j0)) = u;
    }
    fence_proxy_async_smem();
  };

  // =========================== prologue ===========================
  if (warp == 0) {
    tmem_alloc(sTmem, kTmemCols);
    tmem_alloc(sTmem + 1, kTmemGramCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) mbar_init(&bar_tma[s], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_g[s], 128);
      mbar_init(&bar_z[s], 1);
      mbar_init(&bar_xm[s], 32);
    }
    mbar_init(bar_w, 1);
    mbar_init(bar_wb, 128);
    mbar_init(bar_gram, 1);
    mbar_init(bar_pro, 1);
    for (int s = 0; s < NST; ++s) mbar_init(&bar_rdy[s], 128);
    mbar_init_fence();
    *sAbort = 0;
  }
  if (is_bulk) {
    store_block(0, fetch_block(0));
    store_block(8, fetch_block(8));
  } else if (is_chain && gt < D) {
    sGam[gt] = p.no_ln ? 1.f : p.gamma[(size_t)h * D + gt];
    sBet[gt] = p.no_ln ? 0.f : p.beta[(size_t)h * D + gt];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sTmem[0];
  const uint32_t tmem2 = sTmem[1];
  if (tma_thread) {
    prefetch_tensormap(&maps.q);
    prefetch_tensormap(&maps.k);
    prefetch_tensormap(&maps.v);
    for (int x = 0; x < NST && x <= nc; ++x) issue_tma(x);
  }
  if (tid == 32) {
    float s2 = 0.f, sgb = 0.f;
    for (int f = 0; f < D; ++f) {
      s2 = fmaf(sGam[f], sGam[f], s2);
      sgb = fmaf(sGam[f], sBet[f], sgb);
    }
    sGamSums[0] = s2;
    sGamSums[1] = sgb;
  }
  if (is_bulk) {
    // W0 -> TMEM (both row copies) and the bf16 operand W_s
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
  // tiles of chunks 0, 1 (chunk 1 carries Q_0) and, for the Gram of chunk 1, 2
  bool bad = false;
  if (!mbar_wait_bounded(&bar_tma[0], 0, lim)) bad = true;
  if (!mbar_wait_bounded(&bar_tma[1], 0, lim)) bad = true;
  if (nc > 1 && !mbar_wait_bounded(&bar_tma[2], 0, lim)) bad = true;
  if (p.kq_silu && is_bulk) {
    // stages 0 .. min(3, nc) (the prologue MMAs and the first Gram read them)
    for (int x = 0; x <= nc && x < 4; ++x) {
      if (x == 3 && !mbar_wait_bounded(&bar_tma[3], 0, lim)) bad = true;
      if (bad) break;
      silu_stage(x);
      mbar_arrive(&bar_rdy[x]);
    }
  }
  tc_fence_before();
  const bool pro_bad = __syncthreads_or(bad);
  tc_fence_after();
  if (pro_bad && tid == 0) fail();
  if (issuer && !pro_bad) {
    mma_gram(tmem2, 0);                        // Xg_1, M_0
    if (nc > 1) mma_gram(tmem2, 1);            // Xg_2, M_1
    mma_ws(tmem + col_p(0), tKQ(0), 16);       // P_0
    mma_ws(tmem + col_p(1), tKQ(1), 32);       // [P_1 | Q0_0]
    mma_commit(bar_pro);
  }
  if (warp == 4 && !pro_bad) {
    if (mbar_wait_bounded(bar_pro, 0, lim)) {
      tc_fence_after();
      gram_extract(tmem2, 0);
      if (nc > 1) gram_extract(tmem2, 1);
    } else if (lane == 0) {
      fail();
    }
  }
  if (warp == 4 && !pro_bad) {
    mbar_arrive(&bar_xm[0]);
    mbar_arrive(&bar_xm[1]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const bool run = !*sAbort;
  __syncthreads();

  if (is_chain && run) {
    // =========================== chain ===========================
    const float sg2 = sGamSums[0], sgb = sGamSums[1];
    const int tm_m = gt >> 3, tm_p = gt & 7;  // token-major role: token, feature part
    for (int k = 0; k < nc; ++k) {
      const int n = chunk_len(k);
      const bool upd = sFlag[k & (kSR - 1)] != 0;
      // per-feature coefficients that do not depend on Z_k, formed before
      // waiting for it: LNJAC a = gamma^2, c = gamma (beta - v);
      // simplified a = gamma, c = beta - v; no LayerNorm c = -v
      // ablation (GM 3, and GM 4 next to the full Jacobian form): a = 0, c = -gamma v
      float a8[8], c8[8], cb8[8];
      {
        const unsigned char* Vt = tV(k) + tm_m * D * 2;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int f = tm_p + 8 * u;
          const float v = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(Vt + f * 2));
          const float g = sGam[f];
          cb8[u] = -g * v;
          if (GM == 1 || GM == 4) {
            a8[u] = g * g;
            c8[u] = g * (sBet[f] - v);
          } else if (GM == 3) {
            a8[u] = 0.f;
            c8[u] = cb8[u];
          } else if (GM == 0) {
            a8[u] = g;
            c8[u] = sBet[f] - v;
          } else {
            a8[u] = 0.f;
            c8[u] = -v;
          }
        }
      }
      const float eta = (tm_m < n) ? sEta[(k & (kSR - 1)) * CB + tm_m] : 0.f;
      bool ok;
      if (k == 0) ok = mbar_wait_bounded(bar_pro, 0, lim);
      else ok = mbar_wait_bounded(&bar_z[k & 1], (uint32_t)(((k - 1) >> 1) & 1), lim);
      if (upd && ok) {
        // Z_k^T (feature-major) -> token-major tile
        tc_fence_after();
        float z[8];
        tmem_ld8(tmem + tlane + col_p(k & 1) + 8 * half, z);
        tmem_wait_ld();
        float* Zk = sZ + (k & 1) * CB * kZS + 8 * half * kZS + fm;
#pragma unroll
        for (int u = 0; u < 8; ++u) Zk[u * kZS] = z[u];
      }
      tc_fence_before();
      if (bar_any(kBarChain, 128, !ok || *sAbort)) {
        if (gt == 0) fail();
        break;
      }
      if (upd) {
        // token-major LayerNorm + gradient: token tm_m, features tm_p + 8u
        const float* Zk = sZ + (k & 1) * CB * kZS + tm_m * kZS;
        float z[8], G[8];
        (void)sgb;
#pragma unroll
        for (int u = 0; u < 8; ++u) z[u] = Zk[tm_p + 8 * u];
        if (GM == 2) {
#pragma unroll
          for (int u = 0; u < 8; ++u) G[u] = z[u] + c8[u];
        } else {
          // shift by one element of the token, then all moments in one round
          // (Jacobian forms: sums of a y, a y^2, c y, c; GM 4 also c_b y, c_b)
          constexpr bool kJac = GM == 1 || GM == 3 || GM == 4;
          constexpr int NM = GM == 4 ? 8 : (kJac ? 6 : 2);
          const float c0 = __shfl_sync(0xffffffffu, z[0], lane & ~7);
          float m[NM];
#pragma unroll
          for (int i = 0; i < NM; ++i) m[i] = 0.f;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float y = z[u] - c0;
            z[u] = y;
            m[0] += y;
            m[1] = fmaf(y, y, m[1]);
            if (kJac) {
              const float ay = a8[u] * y;
              m[2] += ay;
              m[3] = fmaf(ay, y, m[3]);
              m[4] = fmaf(c8[u], y, m[4]);
              m[5] += c8[u];
            }
            if (GM == 4) {
              m[6] = fmaf(cb8[u], y, m[6]);
              m[7] += cb8[u];
            }
          }
#pragma unroll
          for (int off = 1; off < 8; off <<= 1) {
#pragma unroll
            for (int i = 0; i < NM; ++i) m[i] += __shfl_xor_sync(0xffffffffu, m[i], off);
          }
          const float inv_d = 1.0f / D;
          const float mu1 = m[0] * inv_d;                    // mean of the shifted values
          const float var = fmaxf(fmaf(m[1], inv_d, -mu1 * mu1), 0.f);
          const float rs = rsqrtf(var + p.eps);
          if (kJac) {
            // J^T g with g = a xhat / rs + c (a = gamma^2, c = gamma (beta - v): the
            // full form; a = 0, c = -gamma v: the ablation), from the moments of
            // the centred values y - mu1
            const float sa = (GM == 3) ? 0.f : sg2;          // sum of a
            const float say = m[2] - mu1 * sa;
            const float sayy = m[3] - 2.f * mu1 * m[2] + mu1 * mu1 * sa;
            const float scy = m[4] - mu1 * m[5];
            const float mg = (rs * say + m[5]) * inv_d;      // mean of g
            const float mgx = rs * (rs * sayy + scy) * inv_d;
            const float rs2 = rs * rs;
#pragma unroll
            for (int u = 0; u < 8; ++u)
              G[u] = rs2 * (a8[u] - mgx) * (z[u] - mu1) + rs * (c8[u] - mg);
            if (GM == 4) {
              // the ablation (a = 0) next to the full form: both norms, then
              // the ablation, rescaled to the full norm with norm matching
              const float mgb = m[7] * inv_d;
              const float mgxb = rs * (m[6] - mu1 * m[7]) * inv_d;
              float nf = 0.f, nb = 0.f;
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const float gb = -rs2 * mgxb * (z[u] - mu1) + rs * (cb8[u] - mgb);
                nf = fmaf(G[u], G[u], nf);
                nb = fmaf(gb, gb, nb);
                G[u] = gb;
              }
#pragma unroll
              for (int off = 1; off < 8; off <<= 1) {
                nf += __shfl_xor_sync(0xffffffffu, nf, off);
                nb += __shfl_xor_sync(0xffffffffu, nb, off);
              }
              if (p.grad_norms != nullptr && tm_p == 0 && tm_m < n) {
                float* gn = p.grad_norms + (tok0 + (size_t)k * CB + tm_m) * 2;
                gn[0] = sqrtf(nf);
                gn[1] = sqrtf(nb);
              }
              const float scale = !p.norm_match ? 1.f : (nb > 0.f ? sqrtf(nf / nb) : 0.f);
#pragma unroll
              for (int u = 0; u < 8; ++u) G[u] *= scale;
            }
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) G[u] = fmaf(a8[u] * rs, z[u] - mu1, c8[u]);
          }
        }
        unsigned char* An = aneg(k);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int f = tm_p + 8 * u;
          const __nv_bfloat16 a = __float2bfloat16_rn(-eta * G[u]);
          *reinterpret_cast<__nv_bfloat16*>(An + core_off(f, tm_m)) = a;
          *reinterpret_cast<__nv_bfloat16*>(An + core_off(f + 64, tm_m)) = a;
        }
        fence_proxy_async_smem();
      } else if (GM == 4 && p.grad_norms != nullptr && tm_p == 0 && tm_m < n) {
        // a SKIP chunk takes no gradient: zero norms for its tokens
        float* gn = p.grad_norms + (tok0 + (size_t)k * CB + tm_m) * 2;
        gn[0] = 0.f;
        gn[1] = 0.f;
      }
      mbar_arrive(&bar_g[k & 1]);
    }
  } else if (is_bulk && run) {
    // =========================== bulk ===========================
    Raw pre{};
    bool finished = true;
    for (int c = 0; c < nc; ++c) {
      const bool upd = sFlag[c & (kSR - 1)] != 0;
      if ((c & 7) == 0) pre = fetch_block(c + 16);
      // the store of chunk c-2 has read its tile (chunk c writes it again)
      if (kTileOut && tma_thread) bulk_wait_group_read<0>();
      // ---- MMAc and MMA3 of chunk c complete ----
      bool ok = mbar_wait_bounded(bar_w, (uint32_t)(c & 1), lim);
      if (bar_any(kBarBulk, 128, !ok || *sAbort)) {
        if (gt == 0) fail();
        finished = false;
        break;
      }
      tc_fence_after();
      // chunk c-1's outputs, written to its tile before the barrier above
      if (kTileOut && tma_thread && c >= 1) {
        tma_store_3d(&maps.o, out_tile(c - 1), 0, (c - 1) * CB, (int)bh);
        bulk_commit_group();
      }
      // ---- W_{s,c+1} (fp32 TMEM) -> bf16 operand; snapshot ----
      const int row = wq * 32 + lane;
      if (upd) {
        // two 32-column TMEM loads; the second is in flight while the first
        // half is packed to bf16 and stored
        float w[32];
        uint4 packed[4];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          tmem_ld32(tmem + tlane + kColW + 32 * hf, w);
          if (hf == 1) {
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
              *reinterpret_cast<uint4*>(sWb + sw128_off(row, ch)) = packed[ch];
          }
          tmem_wait_ld();
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            packed[ch].x = pack_bf16(w[8 * ch + 0], w[8 * ch + 1]);
            packed[ch].y = pack_bf16(w[8 * ch + 2], w[8 * ch + 3]);
            packed[ch].z = pack_bf16(w[8 * ch + 4], w[8 * ch + 5]);
            packed[ch].w = pack_bf16(w[8 * ch + 6], w[8 * ch + 7]);
          }
          if (Wc && row < 64) {
            float* dst = Wc + ((size_t)(c + 1) * D + row) * D + 32 * hf;
#pragma unroll
            for (int k = 0; k < 32; k += 4)
              *reinterpret_cast<float4*>(dst + k) = make_float4(w[k], w[k + 1], w[k + 2], w[k + 3]);
          }
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
          *reinterpret_cast<uint4*>(sWb + sw128_off(row, 4 + ch)) = packed[ch];
        fence_proxy_async_smem();
      } else if (Wc && row < 64) {
        const float* srcw = Wc + ((size_t)c * D + row) * D;  // W unchanged: repeat the snapshot
        float* dst = Wc + ((size_t)(c + 1) * D + row) * D;
        for (int k = 0; k < 64; k += 4)
          *reinterpret_cast<float4*>(dst + k) = *reinterpret_cast<const float4*>(srcw + k);
      }
      tc_fence_before();
      mbar_arrive(bar_wb);
      // refill stage c % NST with load c + NST: every reader of its tiles (MMA1
      // and the Grams of chunks c-1 and c, MMA3 of chunk c, the chain's V_c)
      // completed before bar_w of this chunk
      if (tma_thread && c + NST <= nc) {
        fence_proxy_async_smem();
        issue_tma(c + NST);
      }
      // SiLU variant: stage c+4, read first by the issuer's next iteration
      if (p.kq_silu && c + 4 <= nc) {
        if (mbar_wait_bounded(&bar_tma[(c + 4) % NST], tma_parity(c + 4), lim)) {
          silu_stage(c + 4);
          mbar_arrive(&bar_rdy[(c + 4) % NST]);
        } else if (lane == 0) {
          fail();
        }
      }
      // ---- Gram of chunk c+2 -> [Xg_{c+3}; M_{c+2}]. Its buffer held the
      // operand of chunk c's MMAc, complete since bar_w ----
      // (warp 4 alone: the other bulk warps go on to the outputs; a failed
      // wait is seen by all at the next bar_any)
      if (c + 2 < nc && wq == 0) {
        if (mbar_wait_bounded(bar_gram, (uint32_t)(c & 1), lim)) {
          tc_fence_after();
          gram_extract(tmem2, c + 2);
          mbar_arrive(&bar_xm[c & 1]);
        } else if (lane == 0) {
          fail();
        }
      }
      // ---- outputs o_c = gate * O_c^T ----
      {
        float ov[8];
        tmem_ld8(tmem + tlane + col_o((c + 1) & 1) + 8 * half, ov);
        tmem_wait_ld();
        const float* gte = sGate + (c & (kSR - 1)) * CB + 8 * half;
        if (kTileOut) {  // rows past the sequence are outside the tensor map
          OutT* tile = out_tile(c);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            tile[(8 * half + u) * D + fm] = from_f32<OutT>(gte[u] * ov[u]);
          fence_proxy_async_smem();
        } else {
          const int n = chunk_len(c);
          OutT* dst = go + (size_t)c * CB * D;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int t = 8 * half + u;
            if (t < n) dst[(size_t)t * D + fm] = from_f32<OutT>(gte[u] * ov[u]);
          }
        }
      }
      if ((c & 7) == 4) store_block(c + 12, pre);
    }
    if (kTileOut) {
      bar_sync(kBarBulk, 128);  // every bulk thread's last tile written
      if (tma_thread) {
        if (finished && nc > 0) {
          tma_store_3d(&maps.o, out_tile(nc - 1), 0, (nc - 1) * CB, (int)bh);
          bulk_commit_group();
        }
        bulk_wait_group<0>();  // every output store complete before the CTA ends
      }
    }
  } else if (issuer && run) {
    // =========================== issuer ===========================
    for (int c = 0; c < nc; ++c) {
      const bool upd = sFlag[c & (kSR - 1)] != 0;
      const bool next = c + 1 < nc;
      // the operand [Xg_{c+1}; M_c] (its Gram has left TMEM slot c & 1), Aneg_c
      bool ok = mbar_wait_bounded(&bar_xm[c & 1], (uint32_t)((c >> 1) & 1), lim) &&
                mbar_wait_bounded(&bar_g[c & 1], (uint32_t)((c >> 1) & 1), lim);
      if (!ok || *sAbort) {
        fail();
        break;
      }
      tc_fence_after();
      const uint64_t da = smem_desc(smem_u32(aneg(c)), 128, 256, kLayoutNone);
      if (upd)
        mma_bf16_ss(tmem + col_p((c + 1) & 1), da,
                    smem_desc(smem_u32(xm(c)), 128, 256, kLayoutNone), idescN32, 1u);
      if (next) mma_commit(&bar_z[(c + 1) & 1]);
      if (upd)
        mma_bf16_ss(tmem + kColW, da, smem_desc(smem_u32(tKQ(c)), 2048, 1024, kLayoutSw128),
                    idescW, 1u);
      mma_commit(bar_w);
      ++w_issued;

      if (c + 2 < nc) {
        // Gram of chunk c+2 (stages c+2, c+3) into TMEM slot c & 1
        ok = wait_stage(c + 2) && wait_stage(c + 3);
        if (!ok || *sAbort) {
          fail();
          break;
        }
        tc_fence_after();
        mma_gram(tmem2, c + 2);
        mma_commit(bar_gram);
      }
      if (next) {
        // W_{s,c+1} in bf16, then [P_{c+2} | Q0_{c+1}] = W_{s,c+1} [K_{c+2}; Q_{c+1}]^T
        ok = mbar_wait_bounded(bar_wb, (uint32_t)(c & 1), lim) && wait_stage(c + 2);
        if (!ok || *sAbort) {
          fail();
          break;
        }
        tc_fence_after();
        mma_ws(tmem + col_p((c + 2) & 1), tKQ(c + 2), 32);
      }
    }
  }

  // =========================== teardown ===========================
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*sAbort) {
    if (issuer) {
      // all MMAs this thread issued (one commit tracks them all)
      mma_commit(bar_w);
      if (w_issued > 0) mbar_wait_bounded(bar_w, (uint32_t)((w_issued - 1) & 1), drain_lim);
      mbar_wait_bounded(bar_w, (uint32_t)(w_issued & 1), drain_lim);
    } else if (tma_thread) {
      // every TMA stage that may still be loading
      for (int x = (tma_issued > NST ? tma_issued - NST : 0); x < tma_issued; ++x)
        mbar_wait_bounded(&bar_tma[x % NST], tma_parity(x), drain_lim);
    }
  } else if (is_bulk && wq < 2) {
    const int row = wq * 32 + lane;  // W_T from the rows of copy 0
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

}  // namespace tcm
}  // namespace ttt
