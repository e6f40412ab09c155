// Tensor-core (tcgen05) mini-batch scan: d = 64, b = 16, bf16 q/k/v/logits,
// fp32 state W in TMEM, bf16 or fp32 outputs.
//
// Chunk step (PonderTTT, "Technical Architecture": dual-form updates; every
// gradient of a chunk taken at the chunk-start state W_s):
//     z_i = W_s k_i,  G_i = LayerNorm gradient ("Error Correction in Trained
//     TTT Layers", Abstract),  o_i = W_s q_i - sum_{j<=i} eta_j (k_j.q_i) G_j,
//     W_e = W_s - sum_j eta_j G_j k_j^T.
//
// Two-chunk look-ahead. With Aneg_c[f][j] = -eta_j G_j[f] (bf16, written by the
// chain) and W_{s,c+1} = W_{s,c} + Aneg_c K_c,
//     Z_x^T  = W_{s,x-2} K_x^T + Aneg_{x-2} (K_x K_{x-2}^T)^T + Aneg_{x-1} (K_x K_{x-1}^T)^T
//     O_x^T  = W_{s,x-1} Q_x^T + Aneg_{x-1} (Q_x K_{x-1}^T)^T + Aneg_x tril(Q_x K_x^T)^T
// The W_s products (MMA1) run two chunks early on an older W, and only the
// small corrections (MMAc, K = 16) follow the chain. Per chunk c the chain's
// Aneg_c feeds three MMAs:
//     MMAc_a  B(c+1) (+)= Aneg_c [Xg_{c+1}; M_c]^T    (Xg_{c+1} = K_{c+1} K_c^T, M_c = tril(Q_c K_c^T))
//     MMAc_b  B(c+2)  = Aneg_c [Y_{c+2}; N_{c+1}]^T   (Y_{c+2} = K_{c+2} K_c^T, N_{c+1} = Q_{c+1} K_c^T)
//     MMA3    W += Aneg_c K_c                          (fp32 state in TMEM)
// and MMA1 A(c+2) = W_{s,c} [K_{c+2}; Q_{c+1}]^T. The chain reads Z_x = A(x) +
// B(x) (P halves) and the bulk reads O_x = A(x+1) + B(x+1) (Q halves).
// The Grams [Xg; M; Y; N] (64 rows x 16, all against K_c) are formed one or two
// chunks ahead by a warp of their own with mma.sync, so no Gram MMA or TMEM
// round trip sits on any loop. The loops per chunk:
//     chain:  Z_c -> LayerNorm -> Aneg_c -> MMAc_a -> Z_{c+1}
//     state:  MMA3_c -> W_{s,c+1} fp32 -> bf16 (bulk) -> MMA3_{c+1}
// (W_s in bf16 is double-buffered, so MMA1 reading one copy overlaps the refresh
// of the other).
//
// Warps (352 threads with one CTA per SM, 320 with two):
//   chain 0-3   read Z_k (TMEM, feature-major), transpose through shared
//               memory, token-major LayerNorm + gradient (8 lanes per token,
//               one shuffle round of shifted moments), write Aneg_k (bf16).
//   bulk 4-7    W (fp32 TMEM) -> bf16 W_s; outputs o_c = gate * O_c^T into a
//               token-major shared-memory tile (two, alternating), written to
//               global memory by one TMA store per chunk (one thread issues
//               every output store); per-chunk scalars; SiLU variant: the
//               in-place SiLU of a stage.
//   issuer 8    (one thread) every tcgen05.mma and commit.
//   gram 9      the Gram operand of chunk c (mma.sync, 64 x 16 x 64), as soon
//               as its buffer is free (two chunks ahead of its use).
//   producer 10 (one thread; one CTA per SM) every TMA load of chunk x =
//               {K_x, Q_{x-1}, V_x} (only Q_{x-1} for a SKIP chunk x), NST
//               chunks ahead, once the bulk has freed the stage; with two CTAs
//               per SM the bulk's store thread issues them instead.
// M = 128 everywhere: A operands stack two copies of their 64 rows, so TMEM
// lanes 0-63 and 64-127 hold identical d-row results and every warp quarter
// reads its own lanes.
//
// SKIP chunks (PonderTTT, "Core Idea"): no K/V load, no LayerNorm, no MMAc, no
// MMA3, no W refresh (the bf16 copy of W_s stays valid); only the outputs
// W_s q, which MMA1 computes anyway.
//
// Every wait is bounded: on expiry the CTA records the timeout status, all
// warps leave their loops, the issuer drains its MMAs and the TMA thread its
// copies (each with a bound of its own) and TMEM is freed.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace ttt {

// Set to a nonzero code by a kernel whose bounded wait gave up; read and
// cleared by ttt_check_device_status(). One word per device, allocated with
// the module of the one translation unit that includes this header.
__device__ int g_ttt_status;

struct TcMaps {
  CUtensorMap q, k, v;  // [B*H][T][64] bf16 as {64, T, B*H}, box {64, 16, 1}
  CUtensorMap o;        // [B*H][T][64] of the output type, the same view and box
};

namespace tc {

constexpr int D = 64;
constexpr int CB = 16;              // chunk (b)
// threads: 4 chain + 4 bulk + 1 issuer + 1 Gram warps, and with one CTA per SM
// a producer warp for the TMA loads (two CTAs per SM issue them from a bulk
// thread: a further warp would cap the registers below what that build needs)
__host__ __device__ constexpr int nt_for(int minb) { return minb == 1 ? 352 : 320; }
constexpr int kMinbMany = 2;        // CTAs per SM of the build for more heads than SMs
constexpr int kSR = 32;             // scalar ring (chunks)
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColW = 0;       // W accumulator (64 columns)
// A(x): MMA1 results [P | Q0] (16 + 16 columns), three slots; B(x): the
// corrections, two slots
__device__ __forceinline__ uint32_t col_a(int x) { return 64u + 32u * (uint32_t)(x % 3); }
__device__ __forceinline__ uint32_t col_b(int x) { return 160u + 32u * (uint32_t)(x & 1); }
constexpr int kTile = CB * D * 2;   // 2048 bytes
constexpr int kZS = 72;             // row stride (floats) of the token-major Z tile

// TMA stages: the Gram operand of chunk c needs the keys of chunk c+2 about
// two chunk periods before MMA3 of chunk c, and a load issued once stage c
// frees takes a few microseconds here, so the stages run deep. The per-chunk
// scalars are stored up to 11 chunks ahead of every TMA issue (16 ahead, in
// blocks of 8), which bounds NST at 11.
__host__ __device__ constexpr int nst_for(int minb) { return minb == 1 ? 10 : 6; }

// shared memory (bytes from a 1024-aligned base)
// GCH: the build for a per-feature gate (room for its logit tiles).
template <int NST, bool GCH>
struct TcLayout {
  static_assert(NST <= 11, "the scalar ring must run ahead of every TMA issue");
  static constexpr int oKQ = 0;                             // [NST][K_x | Q_{x-1}] 128B-swizzled
  static constexpr int oV = oKQ + NST * 2 * kTile;          // [NST] V_x, row-major
  static constexpr int oWb = oV + NST * kTile;              // [2] W_s bf16, 128 rows x 128 B, 128B-swizzled
  static constexpr int oAneg = oWb + 2 * 128 * 128;         // [2] 128 rows x 16 bf16 (core matrices)
  static constexpr int oXM = oAneg + 2 * 128 * 32;          // [3] {[Xg; M], [Y; N]}: 2 x 32 x 16 bf16
  static constexpr int oOut = oXM + 3 * 2048;               // [2][16][64] outputs (<= f32), TMA-stored
  static constexpr int oGch = oOut + 2 * CB * D * 4;        // [3][16][64] bf16 per-feature gate logits
  static constexpr int oZ = oGch + (GCH ? 3 * CB * D * 2 : 0);  // [2][16][kZS] f32
  static constexpr int oEta = oZ + 2 * CB * kZS * 4;        // [kSR][16] f32 (mask folded in)
  static constexpr int oGate = oEta + kSR * CB * 4;         // [kSR][16] f32
  static constexpr int oFlag = oGate + kSR * CB * 4;        // [kSR] int
  static constexpr int oGam = oFlag + kSR * 4;              // gamma, beta [2][64] f32, sum gamma^2, sum gamma*beta
  static constexpr int oBar = oGam + 2 * D * 4 + 16;        // mbarriers
  // tma[NST], rdy[NST], free[NST], g[2], z[2], w, wb, pro
  static constexpr int kBars = 3 * NST + 2 + 2 + 3;
  static constexpr int oTmem = oBar + kBars * 8;            // TMEM base address
  static constexpr int oAbort = oTmem + 8;
  static constexpr int kSmemUsed = oAbort + 4;
  static constexpr int kSmemBytes = kSmemUsed + 1024;       // + alignment slack
  static_assert(oWb % 1024 == 0, "128B-swizzled operands are 1024-aligned");
  static_assert(oOut % 128 == 0 && oGch % 16 == 0, "TMA store source on 128 bytes; cp.async on 16");
};
template <int MINB, bool GCH>
constexpr int smem_bytes() { return TcLayout<nst_for(MINB), GCH>::kSmemBytes; }
static_assert(smem_bytes<1, true>() <= 227 * 1024, "one CTA per SM must fit in shared memory");
static_assert(2 * smem_bytes<kMinbMany, true>() <= 227 * 1024,
              "two CTAs per SM must fit in shared memory");
static_assert(2 * kTmemCols <= 512, "two CTAs per SM must fit in TMEM");

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
// Named barrier over `count` threads.
__device__ __forceinline__ void bar_sync(int bar_id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(sm100::smem_u32(bar))
               : "memory");
}
// One arrival for the whole warp: the lanes converge, which orders their
// earlier shared-memory writes before lane 0's arrival (a release). A barrier
// fed this way counts warps, not threads; one arrival per thread would put 32
// atomic updates of the same word in line.
__device__ __forceinline__ void mbar_arrive_warp(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}
// Four 8x8 b16 matrices from shared memory (one row address per lane).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// D (16x8 f32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
constexpr int kBarChain = 2;  // named barriers (0 is __syncthreads)
constexpr int kBarBulk = 3;

}  // namespace tc

// MINB = 2: two CTAs share an SM (heads above the SM count);
// MINB = 1: one CTA per SM, for up to one head per SM (more registers).
// GCH: a per-feature gate (p.gate_channel); the build without it has none of
// its shared memory or code.
template <typename OutT, int GM, int MINB, bool GCH>
__global__ void __launch_bounds__(tc::nt_for(MINB), MINB)
    scan_tc_kernel(const ScanParams p, const __grid_constant__ TcMaps maps) {
  using namespace tc;
  using namespace sm100;
  constexpr int NST = nst_for(MINB);
  constexpr bool kProducer = MINB == 1;  // a warp of its own issues the TMA loads
  using Lt = TcLayout<NST, GCH>;
  constexpr int oKQ = Lt::oKQ, oV = Lt::oV, oWb = Lt::oWb, oAneg = Lt::oAneg, oXM = Lt::oXM,
                oOut = Lt::oOut, oGch = Lt::oGch,
                oZ = Lt::oZ, oEta = Lt::oEta, oGate = Lt::oGate, oFlag = Lt::oFlag,
                oGam = Lt::oGam, oBar = Lt::oBar, oTmem = Lt::oTmem, oAbort = Lt::oAbort;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* sZ = reinterpret_cast<float*>(smem + oZ);
  float* sEta = reinterpret_cast<float*>(smem + oEta);
  float* sGate = reinterpret_cast<float*>(smem + oGate);
  int* sFlag = reinterpret_cast<int*>(smem + oFlag);
  float* sGam = reinterpret_cast<float*>(smem + oGam);
  float* sBet = sGam + D;
  float* sGamSums = sGam + 2 * D;  // [0] sum gamma^2, [1] sum gamma*beta
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(smem + oBar);  // [NST] chunk x -> x % NST
  // [NST] stage x ready for its readers: with the SiLU variant K_x and Q_{x-1}
  // transformed in place (bulk, one arrival per warp); otherwise the TMA
  // barrier is used
  uint64_t* bar_rdy = bar_tma + NST;
  // [NST] stage x % NST no longer read: every reader of chunk x's stage
  // completed before bar_w of chunk x (bulk, one arrival once it saw bar_w)
  uint64_t* bar_free = bar_rdy + NST;
  // [2] chunk k ready for the issuer: Aneg_k written (chain, one arrival per
  // warp) and the Gram operand of chunk k written, stage k+2 landed (Gram
  // warp, one arrival): five arrivals
  uint64_t* bar_g = bar_free + NST;
  uint64_t* bar_z = bar_g + 2;       // [2] Z_k complete in TMEM (commit)
  uint64_t* bar_w = bar_z + 2;       // a chunk's MMAs complete (commit)
  uint64_t* bar_wb = bar_w + 1;      // W read from TMEM and W_s bf16 refreshed (bulk, 4 warps)
  uint64_t* bar_pro = bar_wb + 1;    // prologue MMAs complete (commit)
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + oTmem);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + oAbort);
  auto tKQ = [&](int x) { return smem + oKQ + (x % NST) * 2 * kTile; };  // K_x, then Q_{x-1}
  auto tV = [&](int x) { return smem + oV + (x % NST) * kTile; };
  auto sWb = [&](int i) { return smem + oWb + i * 128 * 128; };
  auto aneg = [&](int c) { return smem + oAneg + (c & 1) * 4096; };
  auto xm = [&](int x) { return smem + oXM + (x % 3) * 2048; };  // [Xg_{x+1}; M_x], then [Y_{x+2}; N_{x+1}]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const bool is_chain = warp < 4;
  const bool is_bulk = warp >= 4 && warp < 8;
  const bool issuer = (tid == 256);
  const bool is_gram = warp == 9;
  const bool tma_thread = (tid == 224);        // bulk warp 7, lane 0: the output stores
  // every TMA load: warp 10, lane 0 (one CTA per SM) or the store thread
  const bool producer = kProducer ? (tid == 320) : tma_thread;
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
  // the gate: one logit per token (through the scalar ring) or, with a
  // per-feature gate, one per token and feature (a [16][64] tile per chunk)
  const __nv_bfloat16* ggl = (p.gate_logit && !GCH)
                                 ? static_cast<const __nv_bfloat16*>(p.gate_logit) + tok0
                                 : nullptr;
  const __nv_bfloat16* gch = (GCH && p.gate_logit)
                                 ? static_cast<const __nv_bfloat16*>(p.gate_logit) + tok0 * D
                                 : nullptr;
  float* Wc = p.W_chunks ? p.W_chunks + (size_t)bh * (p.n_mask_chunks + 1) * D * D : nullptr;
  const long long lim = p.wait_limit;
  const long long drain_lim = 1LL << 24;
  // tokens of chunk x (0 outside the sequence)
  auto chunk_len = [&](int x) { return (x >= 0 && x < nc) ? min(CB, T - x * CB) : 0; };
  auto upd_of = [&](int x) { return x >= 0 && x < nc && sFlag[x & (kSR - 1)] != 0; };
  // B(x) holds corrections iff chunk x-2 or x-1 updated
  auto b_valid = [&](int x) { return upd_of(x - 2) || upd_of(x - 1); };
  auto fail = [&]() {
    *sAbort = 1;
    atomicExch(&g_ttt_status, (int)kStatusTimeout);
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

  // ---- TMA ----
  int tma_issued = 0;  // TMA loads [0, tma_issued) issued (chunk x = {K_x, Q_{x-1}, V_x})
  int w_issued = 0;    // commits to bar_w
  // A SKIP chunk's keys and values are never read by anything whose result is
  // used (its z, gradient and update are not formed; the Gram rows against its
  // keys are zeroed), so only its queries are loaded.
  auto issue_tma = [&](int x) {
    uint64_t* bar = &bar_tma[x % NST];
    const bool kv = upd_of(x);
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
  // stage x ready for the MMAs and the Grams (see bar_rdy)
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

  // ---- issuer helpers ----
  const uint32_t idescN32 = idesc_bf16_f32(128, 32, false, false);
  const uint32_t idescW = idesc_bf16_f32(128, 64, false, true);
  // D = W_s (bf16 copy `wb`) . [32 rows of stage x]^T (N = 32)
  auto mma_ws = [&](uint32_t d, int wb, int x) {
    const uint32_t aw = smem_u32(sWb(wb)), ar = smem_u32(tKQ(x));
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16_ss(d, smem_desc(aw + kk * 32, 16, 1024, kLayoutSw128),
                  smem_desc(ar + kk * 32, 16, 1024, kLayoutSw128), idescN32, kk > 0 ? 1u : 0u);
  };

  // ---- Gram warp: the operand of chunk c (c < nc, c updates), rows
  // [Xg_{c+1}; M_c] and [Y_{c+2}; N_{c+1}] against the keys of chunk c: row
  // block w = 0..3 holds stage c+1 rows 0-15 / 16-31, stage c+2 rows 0-15 /
  // 16-31 (16 rows x 16 keys each, by mma.sync); zero wherever a factor is
  // outside a chunk or belongs to a SKIP chunk (whose stage holds stale keys) ----
  auto gram_operand = [&](int c) {
    const uint32_t right = smem_u32(tKQ(c));  // K_c, rows 0-15
    const int ra = lane & 15, ha = lane >> 4;                            // A: row, 8-column half
    const int rb = (lane & 7) + 8 * (lane >> 4), hb = (lane >> 3) & 1;  // B: key row, half
    // all four row blocks and both key halves at once: eight independent
    // accumulator chains of four k-steps each, so the latency of one mma.sync
    // overlaps the others
    float acc[4][2][4];
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[w][nt][i] = 0.f;
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) {
      uint32_t bq[4], a[4][4];
      ldsm_x4(right + (uint32_t)rb * 128u + (uint32_t)(((2 * kb + hb) ^ (rb & 7)) << 4), bq);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t left = smem_u32(tKQ(c + 1 + (w >> 1))) + (uint32_t)((w & 1) * 16) * 128u;
        const int rla = (w & 1) * 16 + ra;  // row within the stage
        ldsm_x4(left + (uint32_t)ra * 128u + (uint32_t)(((2 * kb + ha) ^ (rla & 7)) << 4), a[w]);
      }
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        mma_16816(acc[w][0], a[w], bq[0], bq[1]);
        mma_16816(acc[w][1], a[w], bq[2], bq[3]);
      }
    }
    const int n0 = chunk_len(c);
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      int nrow;  // rows of this block in a chunk whose keys / queries are used
      if (w == 0) nrow = upd_of(c + 1) ? chunk_len(c + 1) : 0;       // Xg_{c+1}
      else if (w == 1) nrow = n0;                                    // M_c
      else if (w == 2) nrow = upd_of(c + 2) ? chunk_len(c + 2) : 0;  // Y_{c+2}
      else nrow = chunk_len(c + 1);                                  // N_{c+1}
      unsigned char* dst = xm(c) + (w >> 1) * 1024;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int r = g + 8 * hr, j = 8 * nt + 2 * t4;
          const bool okr = r < nrow;
          float v0 = (okr && j < n0) ? acc[w][nt][2 * hr] : 0.f;
          float v1 = (okr && j + 1 < n0) ? acc[w][nt][2 * hr + 1] : 0.f;
          if (w == 1) {  // causal: key j <= query r
            v0 = (j <= r) ? v0 : 0.f;
            v1 = (j + 1 <= r) ? v1 : 0.f;
          }
          *reinterpret_cast<uint32_t*>(dst + core_off((w & 1) * 16 + r, j)) = pack_bf16(v0, v1);
        }
      }
    }
    fence_proxy_async_smem();
  };

  // =========================== prologue ===========================
  if (warp == 0) {
    tmem_alloc(sTmem, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bar_tma[s], 1);
      mbar_init(&bar_rdy[s], 4);
      mbar_init(&bar_free[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_g[s], 5);
      mbar_init(&bar_z[s], 1);
    }
    mbar_init(bar_w, 1);
    mbar_init(bar_wb, 4);
    mbar_init(bar_pro, 1);
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
  if (producer) {
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
    // W0 -> TMEM (both row copies) and the bf16 operand W_{s,0} (copy 0)
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
        *reinterpret_cast<uint4*>(sWb(0) + sw128_off(row, 4 * hf + ch)) = u;
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
  // stages 0, 1, 2 (read by the prologue MMAs and the first Gram operand)
  bool bad = false;
  for (int x = 0; x < 3 && x <= nc; ++x)
    if (!mbar_wait_bounded(&bar_tma[x], 0, lim)) bad = true;
  if (p.kq_silu && is_bulk) {
    // stages 0 .. min(3, nc), each marked ready
    for (int x = 0; x <= nc && x < 4; ++x) {
      if (x == 3 && !mbar_wait_bounded(&bar_tma[3], 0, lim)) bad = true;
      bad = __any_sync(0xffffffffu, bad);
      if (bad) break;
      silu_stage(x);
      mbar_arrive_warp(&bar_rdy[x]);
    }
  }
  tc_fence_before();
  const bool pro_bad = __syncthreads_or(bad);
  tc_fence_after();
  if (pro_bad && tid == 0) fail();
  if (issuer && !pro_bad) {
    mma_ws(tmem + col_a(0), 0, 0);  // A(0) = W0 [K_0; -]^T
    mma_ws(tmem + col_a(1), 0, 1);  // A(1) = W0 [K_1; Q_0]^T (stage 1 holds only Q_0 if nc = 1)
    mma_commit(bar_pro);
  }
  if (is_gram && !pro_bad) {
    if (upd_of(0)) gram_operand(0);
    mbar_arrive_warp(&bar_g[0]);  // (stages 0 .. 2 were waited above)
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
    (void)sgb;
    for (int k = 0; k < nc; ++k) {
      const int n = chunk_len(k);
      const bool upd = upd_of(k);
      // per-feature coefficients that do not depend on Z_k, formed before
      // waiting for it: LNJAC a = gamma^2, c = gamma (beta - v); simplified
      // a = gamma, c = beta - v; no LayerNorm c = -v; ablation (GM 3, and GM 4
      // next to the full Jacobian form) a = 0, c = -gamma v
      float a8[8], c8[8], cb8[8];
      bool vok = true;
      if (upd) vok = mbar_wait_bounded(&bar_tma[k % NST], tma_parity(k), lim);  // V_k landed
      if (upd && vok) {
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
      ok = ok && vok;
      if (upd && ok) {
        // Z_k^T = A(k) + B(k) (feature-major) -> token-major tile
        tc_fence_after();
        float z[8], zb[8];
        tmem_ld8(tmem + tlane + col_a(k) + 8 * half, z);
        const bool bv = b_valid(k);
        if (bv) tmem_ld8(tmem + tlane + col_b(k) + 8 * half, zb);
        tmem_wait_ld();
        float* Zk = sZ + (k & 1) * CB * kZS + 8 * half * kZS + fm;
#pragma unroll
        for (int u = 0; u < 8; ++u) Zk[u * kZS] = bv ? z[u] + zb[u] : z[u];
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
      mbar_arrive_warp(&bar_g[k & 1]);
    }
  } else if (is_gram && run) {
    // =========================== Gram ===========================
    // the operand of chunk c goes to buffer c % 3, last read by the MMAs of
    // chunk c-3, all complete once Z_{c-1} is (its commit follows them). It
    // reads stages c .. c+2; a stage this warp has seen land (seen > x) needs
    // no second wait (each wait costs a few hundred cycles even when the phase
    // is long complete). Every chunk, SKIP or not, waits through stage c+2
    // before its arrival, so the issuer's wait for chunk c also covers the
    // stage its MMA1 reads (a stage is reloaded only after bar_w of its chunk,
    // which needs this warp's arrival for that chunk, so no phase is missed)
    int seen = 3;  // stages 0 .. 2: waited by every thread in the prologue
    for (int c = 1; c < nc; ++c) {
      bool ok = (c == 1) ? mbar_wait_bounded(bar_pro, 0, lim)
                         : mbar_wait_bounded(&bar_z[(c - 1) & 1], (uint32_t)(((c - 2) >> 1) & 1),
                                             lim);
      if (ok) {
        const int top = min(c + 2, nc);
        for (int x = max(seen, c); x <= top; ++x) ok = ok && wait_stage(x);
        seen = max(seen, top + 1);
      }
      if (ok && upd_of(c)) {
        ok = __all_sync(0xffffffffu, ok);
        if (ok) gram_operand(c);
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) fail();
        break;
      }
      if (__any_sync(0xffffffffu, *sAbort != 0)) break;
      mbar_arrive_warp(&bar_g[c & 1]);
    }
  } else if (is_bulk && run) {
    // =========================== bulk ===========================
    // Per-feature gate: chunk x's [16][64] bf16 logits, one 16-byte piece per
    // bulk thread, copied into tile x % 3 two chunks ahead (rows past the
    // sequence zero-filled). One cp.async group per chunk, committed whether or
    // not it copies anything, so the group count matches the chunk count. A
    // call without that gate runs none of it: a cp.async wait would also wait
    // for this warp's other loads in flight (the scalar ring's, which are
    // meant to take four chunks).
    auto load_gch = [&](int x) {
      if (!gch) return;
      if (x < nc) {
        const int row = gt >> 3, piece = gt & 7;
        const bool ok = x * CB + row < T;
        const __nv_bfloat16* src = gch + (ok ? (size_t)(x * CB + row) * D + piece * 8 : 0);
        cp_async16_zfill(smem + oGch + (x % 3) * CB * D * 2 + row * D * 2 + piece * 16, src,
                         ok ? 16 : 0);
      }
      cp_async_commit_group();
    };
    load_gch(0);
    load_gch(1);
    Raw pre{};
    int wbuf = 0;  // the bf16 copy holding W_{s,c}
    for (int c = 0; c < nc; ++c) {
      const bool upd = upd_of(c);
      if ((c & 7) == 0) pre = fetch_block(c + 16);
      if (gch) cp_async_wait_group<1>();  // this thread's piece of chunk c's gate tile (the barrier below shares it)
      // ---- the MMAs of chunk c complete ----
      if (tma_thread) bulk_wait_group_read<1>();  // the store of chunk c-2 has read its tile
      bool ok = mbar_wait_bounded(bar_w, (uint32_t)(c & 1), lim);
      if (bar_any(kBarBulk, 128, !ok || *sAbort)) {
        if (gt == 0) fail();
        break;
      }
      tc_fence_after();
      // stage c may be refilled: every reader of its tiles (MMA1 of chunk c-2,
      // the Gram operands of chunks c-2 .. c, MMA3 of chunk c, the chain's V_c)
      // completed before bar_w of this chunk
      if (kProducer && gt == 0) mbar_arrive(&bar_free[c % NST]);
      // ---- outputs O_c = A(c+1) + B(c+1) (query halves) ----
      float ov[8];
      {
        float ob[8];
        tmem_ld8(tmem + tlane + col_a(c + 1) + 16 + 8 * half, ov);
        const bool bv = b_valid(c + 1);
        if (bv) tmem_ld8(tmem + tlane + col_b(c + 1) + 16 + 8 * half, ob);
        tmem_wait_ld();
        if (bv) {
#pragma unroll
          for (int u = 0; u < 8; ++u) ov[u] += ob[u];
        }
      }
      // ---- W_{s,c+1} (fp32 TMEM) -> the other bf16 copy; snapshot ----
      const int row = wq * 32 + lane;
      if (upd) {
        wbuf ^= 1;
        unsigned char* dstw = sWb(wbuf);
        float w[32];
        uint4 packed[4];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          tmem_ld32(tmem + tlane + kColW + 32 * hf, w);
          if (hf == 1) {
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
              *reinterpret_cast<uint4*>(dstw + sw128_off(row, ch)) = packed[ch];
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
          *reinterpret_cast<uint4*>(dstw + sw128_off(row, 4 + ch)) = packed[ch];
        fence_proxy_async_smem();
      } else if (Wc && row < 64) {
        const float* srcw = Wc + ((size_t)c * D + row) * D;  // W unchanged: repeat the snapshot
        float* dst = Wc + ((size_t)(c + 1) * D + row) * D;
        for (int k = 0; k < 64; k += 4)
          *reinterpret_cast<float4*>(dst + k) = *reinterpret_cast<const float4*>(srcw + k);
      }
      tc_fence_before();
      mbar_arrive_warp(bar_wb);
      if (!kProducer && tma_thread && c + NST <= nc) {  // refill stage c (see above)
        fence_proxy_async_smem();
        issue_tma(c + NST);
      }
      // SiLU variant: stage c+4, read first by the chain after chunk c+1
      if (p.kq_silu && c + 4 <= nc) {
        if (__all_sync(0xffffffffu,
                       mbar_wait_bounded(&bar_tma[(c + 4) % NST], tma_parity(c + 4), lim))) {
          silu_stage(c + 4);
          mbar_arrive_warp(&bar_rdy[(c + 4) % NST]);
        } else if (lane == 0) {
          fail();
        }
      }
      // ---- outputs o_c = gate * O_c^T: into a token-major tile, then one TMA
      // store of the tile (rows past the sequence are outside the tensor map
      // and are not written). The tile of chunk c-2 was last read by its store,
      // which the storing thread waited for before this chunk's first barrier.
      {
        const float* gte = sGate + (c & (kSR - 1)) * CB + 8 * half;
        const __nv_bfloat16* gtile =
            reinterpret_cast<const __nv_bfloat16*>(smem + oGch) + (c % 3) * CB * D;
        OutT* tile = reinterpret_cast<OutT*>(smem + oOut) + (c & 1) * CB * D;
        if (gch) {  // (one branch per chunk: a per-element select would evaluate both sides)
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int t = 8 * half + u;
            const float g = sigmoidf_(__bfloat162float(gtile[t * D + fm]));
            tile[t * D + fm] = from_f32<OutT>(g * ov[u]);
          }
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) tile[(8 * half + u) * D + fm] = from_f32<OutT>(gte[u] * ov[u]);
        }
        fence_proxy_async_smem();
        bar_sync(kBarBulk, 128);
        if (tma_thread) {
          tma_store_3d(&maps.o, tile, 0, c * CB, (int)bh);
          bulk_commit_group();
        }
      }
      if ((c & 7) == 4) store_block(c + 12, pre);
      // tile (c+2) % 3 was last read by the outputs of chunk c-1, before this
      // chunk's first barrier
      load_gch(c + 2);
    }
    if (gch) cp_async_wait_group<0>();     // no gate copy in flight when the CTA ends
    if (tma_thread) bulk_wait_group<0>();  // every output store complete before the CTA ends
  } else if (kProducer && producer && run) {
    // =========================== producer ===========================
    // load x goes into stage x % NST once the bulk has seen bar_w of chunk
    // x - NST. Phase x - NST of that stage's barrier cannot be overtaken: its
    // next phase needs chunk x's MMAs, which need load x.
    for (int x = NST; x <= nc; ++x) {
      const int y = x - NST;
      if (!mbar_wait_bounded(&bar_free[y % NST], (uint32_t)((y / NST) & 1), lim) || *sAbort) {
        fail();
        break;
      }
      fence_proxy_async_smem();
      issue_tma(x);
    }
  } else if (issuer && run) {
    // =========================== issuer ===========================
    int wbuf = 0;  // the bf16 copy holding W_{s,c}
    for (int c = 0; c < nc; ++c) {
      const bool upd = upd_of(c);
      // the Gram operand of chunk c, Aneg_c and stage c+2
      // (one barrier for the three)
      bool ok = mbar_wait_bounded(&bar_g[c & 1], (uint32_t)((c >> 1) & 1), lim);
      if (!ok || *sAbort) {
        fail();
        break;
      }
      tc_fence_after();
      const uint64_t da = smem_desc(smem_u32(aneg(c)), 128, 256, kLayoutNone);
      if (upd)  // B(c+1) (+)= Aneg_c [Xg_{c+1}; M_c]^T
        mma_bf16_ss(tmem + col_b(c + 1), da, smem_desc(smem_u32(xm(c)), 128, 256, kLayoutNone),
                    idescN32, upd_of(c - 1) ? 1u : 0u);
      if (c + 1 < nc) mma_commit(&bar_z[(c + 1) & 1]);
      // the bulk has read O_{c-1} (from A(c), B(c)) and W_{s,c} from TMEM, and
      // written the bf16 copy of W_{s,c}
      if (c > 0) {
        ok = mbar_wait_bounded(bar_wb, (uint32_t)((c - 1) & 1), lim);
        if (!ok || *sAbort) {
          fail();
          break;
        }
        tc_fence_after();
      }
      if (upd && c + 1 < nc)  // B(c+2) = Aneg_c [Y_{c+2}; N_{c+1}]^T (slot of B(c), read)
        mma_bf16_ss(tmem + col_b(c + 2), da,
                    smem_desc(smem_u32(xm(c) + 1024), 128, 256, kLayoutNone), idescN32, 0u);
      if (upd)  // W += Aneg_c K_c (K as an MN-major operand)
        mma_bf16_ss(tmem + kColW, da, smem_desc(smem_u32(tKQ(c)), 2048, 1024, kLayoutSw128),
                    idescW, 1u);
      mma_commit(bar_w);
      ++w_issued;
      if (c + 1 < nc) {
        // A(c+2) = W_{s,c} [K_{c+2}; Q_{c+1}]^T from the bf16 copy of W_{s,c}.
        // Stage c+2 has landed: the Gram warp saw it before its arrival for
        // chunk c, waited for above
        mma_ws(tmem + col_a(c + 2), wbuf, c + 2);
      }
      if (upd) wbuf ^= 1;
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
    } else if (producer) {
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
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace ttt
