// Tensor-core (tcgen05) mini-batch scan: d = 64, b = 16, bf16 q/k/v/logits,
// fp32 state W in TMEM, bf16 or fp32 outputs.
//
// Per chunk of b tokens (PonderTTT, "Technical Architecture": dual-form
// updates; the gradients of the chunk all taken at the chunk-start W_s):
//
//   MMA1   [Z^T | Q0^T] (d x 2b) = W_s (d x d) . [K_c ; Q_c]^T         (bf16 -> fp32 TMEM)
//   CUDA   per token: LayerNorm of z_i = W_s k_i over the d features and the
//          inner gradient G_i ("Error Correction in Trained TTT Layers",
//          Abstract); Aneg[f][j] = -eta_j G_j[f];  M[i][j] = q_i . k_j (j <= i)
//   MMA2   O^T += Aneg . M^T           -> o_i = W_s q_i - sum_{j<=i} eta_j (k_j.q_i) G_j
//   MMA3   W   += Aneg . K_c           -> W_e = W_s - sum_j eta_j G_j k_j^T   (fp32 in TMEM)
//   CUDA   o_i * sigmoid(gate_i) -> HBM; W (fp32 TMEM) -> bf16 W_s for the next MMA1.
//
// M = 128 everywhere: the A operands stack two identical copies of their 64
// rows, so the accumulator holds two identical copies of every d-row result
// (TMEM lanes 0-63 and 64-127) and all four warps read TMEM: warps 0/1 handle
// tokens 0-7 (features 0-31 / 32-63), warps 2/3 tokens 8-15.
//
// SKIP chunks (eta = 0) run only MMA1 and emit o_i = sigmoid(gate_i) W_s q_i;
// W is not touched. Every mbarrier wait is bounded: on expiry the CTA records
// TTT timeout status, drains the copies and MMAs it has in flight (with their
// own bound), frees its TMEM and returns.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace ttt {

struct TcMaps {
  CUtensorMap q, k, v;  // [B*H][T][64] bf16, box {64, 16, 1}; q, k 128B-swizzled
};

namespace tc {

constexpr int D = 64;
constexpr int CB = 16;             // chunk (b)
constexpr int NT = 128;            // threads
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kColW = 0;      // W accumulator, 64 columns
constexpr uint32_t kColZ = 64;     // Z^T, 16 columns
constexpr uint32_t kColO = 80;     // Q0^T then O^T, 16 columns
constexpr int kTileBytes = CB * D * 2;  // 2048

// shared-memory carve-up (bytes from a 1024-aligned base)
constexpr int oKQ = 0;                       // [2 stages][K rows 0-15 | Q rows 16-31] SW128
constexpr int oWb = oKQ + 2 * 2 * kTileBytes;  // W_s bf16, 128 rows x 128 B, SW128
constexpr int oV = oWb + 128 * 128;          // [2 stages][16][64] bf16, row-major
constexpr int oAneg = oV + 2 * kTileBytes;   // 128 rows x 16 bf16, core-matrix layout
constexpr int oM = oAneg + 128 * 32;         // 16 x 16 bf16, core-matrix layout
constexpr int oRed = oM + 16 * 16 * 2;       // [4 warps][3 rounds][16] f32
constexpr int oEta = oRed + 4 * 3 * 16 * 4;  // [2][16] f32
constexpr int oGate = oEta + 2 * 16 * 4;     // [2][16] f32
constexpr int oFlag = oGate + 2 * 16 * 4;    // [2] int
constexpr int oBar = oFlag + 16;             // 3 mbarriers (8-byte aligned)
constexpr int oTmem = oBar + 3 * 8;          // TMEM base address
constexpr int oAbort = oTmem + 4;
constexpr int kSmemUsed = oAbort + 4;
// 48 KB + alignment slack: at most four CTAs share an SM, matching the
// 4 x 128 TMEM columns an SM has.
constexpr int kSmemBytes = 48 * 1024 + 1024;
static_assert(kSmemUsed + 1024 <= kSmemBytes, "shared memory layout overflow");

// byte offset of element (row, k) of a K-major no-swizzle operand with
// 8x16B core matrices: LBO = 128 B between the two K halves, SBO = 256 B
// between 8-row groups (16 elements of K per row).
__device__ __forceinline__ int core_off(int row, int k) {
  return (row >> 3) * 256 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}
// byte offset of the 16-byte piece `chunk` of row `row` in a 128B-swizzled tile
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

// Sum N values over the 64 threads of a warp pair (warps 2p, 2p+1).
template <int N>
__device__ __forceinline__ void pair_reduce(float (&s)[N], float* red, int warp, int lane,
                                            int slot) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) s[i] += __shfl_xor_sync(0xffffffffu, s[i], off);
  }
  float* mine = red + (warp * 3 + slot) * 16;
  if (lane < N) {
    float val = 0.f;
#pragma unroll
    for (int i = 0; i < N; ++i)
      if (i == lane) val = s[i];
    mine[lane] = val;
  }
  asm volatile("bar.sync %0, 64;" ::"r"(2 + (warp >> 1)) : "memory");
  const float* other = red + ((warp ^ 1) * 3 + slot) * 16;
#pragma unroll
  for (int i = 0; i < N; ++i) s[i] += other[i];
}

}  // namespace tc

template <typename OutT, int GM>
__global__ void __launch_bounds__(tc::NT, 4)
    scan_tc_kernel(const ScanParams p, const __grid_constant__ TcMaps maps) {
  using namespace tc;
  using namespace sm100;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sKQ = smem + oKQ;
  unsigned char* sWb = smem + oWb;
  unsigned char* sV = smem + oV;
  unsigned char* sAneg = smem + oAneg;
  unsigned char* sM = smem + oM;
  float* sRed = reinterpret_cast<float*>(smem + oRed);
  float* sEta = reinterpret_cast<float*>(smem + oEta);
  float* sGate = reinterpret_cast<float*>(smem + oGate);
  int* sFlag = reinterpret_cast<int*>(smem + oFlag);
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(smem + oBar);  // [2]
  uint64_t* bar_mma = bar_tma + 2;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + oTmem);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int half = warp >> 1;                 // token half of the chunk
  const int f = (warp & 1) * 32 + lane;       // feature (row of W) this thread owns
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

  // ---------------- setup ----------------
  if (warp == 0) {
    tmem_alloc(sTmem, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_tma[0], 1);
    mbar_init(&bar_tma[1], 1);
    mbar_init(bar_mma, 1);
    mbar_init_fence();
    prefetch_tensormap(&maps.q);
    prefetch_tensormap(&maps.k);
    prefetch_tensormap(&maps.v);
    *reinterpret_cast<int*>(smem + oAbort) = 0;
  }
  // eta / gate / update flag of a chunk: raw loads issued early, stored later
  auto fetch_scalars = [&](int c, float& e, float& g, int& m) {
    e = 0.f; g = 0.f; m = 1;
    if (tid < CB && c < nc) {
      const int t0 = c * CB;
      if (p.mask) m = p.mask[(size_t)bi * p.n_mask_chunks + c];
      if (t0 + tid < T) {
        e = __bfloat162float(gel[t0 + tid]);
        if (ggl) g = __bfloat162float(ggl[t0 + tid]);
      }
    }
  };
  auto store_scalars = [&](int c, float e, float g, int m) {
    if (tid < CB && c < nc) {
      const bool ok = c * CB + tid < T;
      sEta[(c & 1) * CB + tid] = (ok && m) ? sigmoidf_(e) * (1.0f / D) : 0.f;
      sGate[(c & 1) * CB + tid] = ggl ? sigmoidf_(g) : 1.f;
      if (tid == 0) sFlag[c & 1] = m ? 1 : 0;
    }
  };
  {
    float e, g;
    int m;
    fetch_scalars(0, e, g, m);
    store_scalars(0, e, g, m);
  }
  // W0 -> both TMEM copies (fp32) and W_s bf16 (A operand of MMA1)
  float wrow[64];
  {
    const float* src = p.W0 + ((size_t)bh * D + f) * D;  // may alias W_T
#pragma unroll
    for (int k = 0; k < 64; k += 4) {
      const float4 w4 = *reinterpret_cast<const float4*>(src + k);
      wrow[k] = w4.x; wrow[k + 1] = w4.y; wrow[k + 2] = w4.z; wrow[k + 3] = w4.w;
    }
  }
  float gam = 1.f, bet = 0.f;
  if (!p.no_ln) {
    gam = p.gamma[(size_t)h * D + f];
    bet = p.beta[(size_t)h * D + f];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t tlane = (uint32_t)(warp * 32) << 16;  // this warp's TMEM lane quarter
  {
    float a[32], b2[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) { a[k] = wrow[k]; b2[k] = wrow[32 + k]; }
    tmem_st32(tmem + tlane + kColW, a);
    tmem_st32(tmem + tlane + kColW + 32, b2);
    const int row = warp * 32 + lane;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      uint4 u;
      u.x = pack_bf16(wrow[8 * ch + 0], wrow[8 * ch + 1]);
      u.y = pack_bf16(wrow[8 * ch + 2], wrow[8 * ch + 3]);
      u.z = pack_bf16(wrow[8 * ch + 4], wrow[8 * ch + 5]);
      u.w = pack_bf16(wrow[8 * ch + 6], wrow[8 * ch + 7]);
      *reinterpret_cast<uint4*>(sWb + sw128_off(row, ch)) = u;
    }
    tmem_wait_st();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // TMA issue (thread 0): K, Q, V tiles of chunk c into stage c & 1
  auto issue_tma = [&](int c) {
    const int s = c & 1;
    mbar_arrive_expect_tx(&bar_tma[s], 3 * kTileBytes);
    unsigned char* kq = sKQ + s * 2 * kTileBytes;
    tma_load_3d(kq, &maps.k, &bar_tma[s], 0, c * CB, (int)bh);
    tma_load_3d(kq + kTileBytes, &maps.q, &bar_tma[s], 0, c * CB, (int)bh);
    tma_load_3d(sV + s * kTileBytes, &maps.v, &bar_tma[s], 0, c * CB, (int)bh);
  };
  // bookkeeping kept identically by every thread (all branches are uniform)
  int tma_pending = 0;            // bit s: stage s has a load in flight
  int last_issued[2] = {-1, -1};  // latest chunk loaded into each stage
  int mma_pending = 0;            // commits not yet waited for
  uint32_t mma_phase = 0;
  if (tid == 0 && nc > 0) issue_tma(0);
  if (nc > 0) {
    tma_pending |= 1;
    last_issued[0] = 0;
  }

  const uint32_t idesc1 = idesc_bf16_f32(128, 32, false, false);
  const uint32_t idesc2 = idesc_bf16_f32(128, 16, false, false);
  const uint32_t idesc3 = idesc_bf16_f32(128, 64, false, true);
  const uint32_t aWb = smem_u32(sWb);
  const uint32_t aAneg = smem_u32(sAneg);
  const uint32_t aM = smem_u32(sM);
  bool aborted = false;

  for (int c = 0; c < nc; ++c) {
    const int s = c & 1;
    const int n = min(CB, T - c * CB);
    // prefetch the next chunk (its stage was released at the end of chunk c-1)
    if (c + 1 < nc) {
      if (tid == 0) {
        fence_proxy_async_smem();
        issue_tma(c + 1);
      }
      tma_pending |= 1 << ((c + 1) & 1);
      last_issued[(c + 1) & 1] = c + 1;
    }
    float pe, pg;
    int pm;
    fetch_scalars(c + 1, pe, pg, pm);

    // wait for this chunk's tiles
    {
      const bool ok = mbar_wait_bounded(&bar_tma[s], (uint32_t)((c >> 1) & 1), lim);
      if (__syncthreads_or(!ok)) { aborted = true; break; }
      tma_pending &= ~(1 << s);
    }
    const bool upd = sFlag[s] != 0;
    const unsigned char* tK = sKQ + s * 2 * kTileBytes;
    const unsigned char* tQ = tK + kTileBytes;
    const unsigned char* tV = sV + s * kTileBytes;

    // ---- MMA1: [Z^T | Q0^T] = W_s . [K ; Q]^T ----
    if (tid == 0) {
      tc_fence_after();
      const uint32_t aKQ = smem_u32(tK);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = smem_desc(aWb + kk * 32, 16, 1024, kLayoutSw128);
        const uint64_t db = smem_desc(aKQ + kk * 32, 16, 1024, kLayoutSw128);
        mma_bf16_ss(tmem + kColZ, da, db, idesc1, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar_mma);
    }
    mma_pending += 1;

    // ---- meanwhile: M[i][j] = q_i . k_j (j <= i) ----
    if (upd) {
      const int i = tid >> 3;
      const int j0 = (tid & 7) * 2;
      float acc0 = 0.f, acc1 = 0.f;
      if (j0 <= i && i < n) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          float qx[8], k0[8], k1[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(tQ + sw128_off(i, ch)), qx);
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(tK + sw128_off(j0, ch)), k0);
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(tK + sw128_off(j0 + 1, ch)), k1);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            acc0 = fmaf(qx[u], k0[u], acc0);
            acc1 = fmaf(qx[u], k1[u], acc1);
          }
        }
        if (j0 + 1 > i) acc1 = 0.f;
      }
      *reinterpret_cast<uint32_t*>(sM + core_off(i, j0)) = pack_bf16(acc0, acc1);
    }

    // ---- wait MMA1 ----
    {
      const bool ok = mbar_wait_bounded(bar_mma, mma_phase, lim);
      if (__syncthreads_or(!ok)) { aborted = true; break; }
      mma_phase ^= 1;
      mma_pending -= 1;
      tc_fence_after();
    }

    if (upd) {
      // ---- LayerNorm + inner gradient of tokens 8*half .. +8, feature f ----
      float z[8], v[8], G[8];
      tmem_ld8(tmem + tlane + kColZ + 8 * half, z);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int t = 8 * half + u;
        v[u] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tV + (t * D + f) * 2));
      }
      tmem_wait_ld();
      if (GM == 2) {
#pragma unroll
        for (int u = 0; u < 8; ++u) G[u] = z[u] - v[u];
      } else {
        float s1[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) s1[u] = z[u];
        pair_reduce<8>(s1, sRed, warp, lane, 0);
        float y[8], s2[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          y[u] = z[u] - s1[u] * (1.0f / D);
          s2[u] = y[u] * y[u];
        }
        pair_reduce<8>(s2, sRed, warp, lane, 1);
        float rs[8], xh[8], err[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          rs[u] = rsqrtf(fmaf(s2[u], 1.0f / D, p.eps));
          xh[u] = y[u] * rs[u];
          err[u] = fmaf(gam, xh[u], bet) - v[u];
        }
        if (GM == 1) {
          float s3[16];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float g = gam * err[u];
            s3[2 * u] = g;
            s3[2 * u + 1] = g * xh[u];
          }
          pair_reduce<16>(s3, sRed, warp, lane, 2);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float g = gam * err[u];
            G[u] = (g - s3[2 * u] * (1.0f / D) - xh[u] * s3[2 * u + 1] * (1.0f / D)) * rs[u];
          }
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) G[u] = err[u];
        }
      }
      // Aneg[f][t] = -eta_t G_t[f], in both row copies f and f + 64
      const float* et = sEta + s * CB + 8 * half;
      uint4 u4;
      u4.x = pack_bf16(-et[0] * G[0], -et[1] * G[1]);
      u4.y = pack_bf16(-et[2] * G[2], -et[3] * G[3]);
      u4.z = pack_bf16(-et[4] * G[4], -et[5] * G[5]);
      u4.w = pack_bf16(-et[6] * G[6], -et[7] * G[7]);
      *reinterpret_cast<uint4*>(sAneg + core_off(f, 8 * half)) = u4;
      *reinterpret_cast<uint4*>(sAneg + core_off(f + 64, 8 * half)) = u4;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      // ---- MMA2 (outputs) and MMA3 (W update) ----
      if (tid == 0) {
        tc_fence_after();
        const uint64_t da = smem_desc(aAneg, 128, 256, kLayoutNone);
        const uint64_t dm = smem_desc(aM, 128, 256, kLayoutNone);
        mma_bf16_ss(tmem + kColO, da, dm, idesc2, 1u);
        const uint64_t dk = smem_desc(smem_u32(tK), 2048, 1024, kLayoutSw128);
        mma_bf16_ss(tmem + kColW, da, dk, idesc3, 1u);
        mma_commit(bar_mma);
      }
      mma_pending += 1;
      const bool ok = mbar_wait_bounded(bar_mma, mma_phase, lim);
      if (__syncthreads_or(!ok)) { aborted = true; break; }
      mma_phase ^= 1;
      mma_pending -= 1;
      tc_fence_after();
    }

    // ---- outputs: o_t = sigmoid(gate_t) * O^T[f][t] ----
    {
      float ov[8];
      tmem_ld8(tmem + tlane + kColO + 8 * half, ov);
      tmem_wait_ld();
      const float* gt = sGate + s * CB + 8 * half;
      OutT* dst = go + (size_t)c * CB * D;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int t = 8 * half + u;
        if (t < n) dst[(size_t)t * D + f] = from_f32<OutT>(gt[u] * ov[u]);
      }
    }
    // ---- snapshot of W_s before this chunk's update, W_e -> bf16 W_s ----
    if (Wc && warp < 2) {
      float* dst = Wc + ((size_t)c * D + f) * D;
#pragma unroll
      for (int k = 0; k < 64; k += 4)
        *reinterpret_cast<float4*>(dst + k) =
            make_float4(wrow[k], wrow[k + 1], wrow[k + 2], wrow[k + 3]);
    }
    if (upd) {
      float a[32], b2[32];
      tmem_ld32(tmem + tlane + kColW, a);
      tmem_ld32(tmem + tlane + kColW + 32, b2);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 32; ++k) { wrow[k] = a[k]; wrow[32 + k] = b2[k]; }
      const int row = warp * 32 + lane;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint4 u;
        u.x = pack_bf16(wrow[8 * ch + 0], wrow[8 * ch + 1]);
        u.y = pack_bf16(wrow[8 * ch + 2], wrow[8 * ch + 3]);
        u.z = pack_bf16(wrow[8 * ch + 4], wrow[8 * ch + 5]);
        u.w = pack_bf16(wrow[8 * ch + 6], wrow[8 * ch + 7]);
        *reinterpret_cast<uint4*>(sWb + sw128_off(row, ch)) = u;
      }
      fence_proxy_async_smem();
    }
    store_scalars(c + 1, pe, pg, pm);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  if (aborted) {
    // record the timeout, then drain what this CTA still has in flight (with
    // a bound of its own) before its TMEM is freed
    if (tid == 0) {
      atomicExch(&g_ttt_status, (int)kStatusTimeout);
      for (int st = 0; st < 2; ++st)
        if (tma_pending & (1 << st))
          mbar_wait_bounded(&bar_tma[st], (uint32_t)((last_issued[st] >> 1) & 1), drain_lim);
      if (mma_pending > 0) mbar_wait_bounded(bar_mma, mma_phase, drain_lim);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  } else if (warp < 2) {
    if (Wc) {
      float* dst = Wc + ((size_t)p.n_mask_chunks * D + f) * D;
#pragma unroll
      for (int k = 0; k < 64; k += 4)
        *reinterpret_cast<float4*>(dst + k) =
            make_float4(wrow[k], wrow[k + 1], wrow[k + 2], wrow[k + 3]);
    }
    float* WT = p.W_T + ((size_t)bh * D + f) * D;
#pragma unroll
    for (int k = 0; k < 64; k += 4)
      *reinterpret_cast<float4*>(WT + k) =
          make_float4(wrow[k], wrow[k + 1], wrow[k + 2], wrow[k + 3]);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace ttt
