// Shared device helpers of the TTT-Linear scan kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ttt {

// Launch parameters shared by all scan kernels. Pointers are device pointers;
// element counts follow the layouts of include/ttt_scan.h.
struct ScanParams {
  const void* q;
  const void* k;
  const void* v;
  const void* eta_logit;
  const void* gate_logit;  // may be null
  const float* W0;
  const float* gamma;      // may be null with no_ln
  const float* beta;
  const unsigned char* mask;  // may be null
  void* o;
  float* W_T;
  float* W_chunks;         // may be null
  int* status;             // device status word (bounded waits)
  long long wait_limit;    // polls per bounded wait
  int B, H, T;
  int b;                   // mask / W_chunks granularity; mini-batch chunk
  int C;                   // internal chunk of the CUDA-core kernel (divides b when required)
  int n_mask_chunks;       // ceil(T / b)
  float eps;
  int lnjac;
  int no_ln;
  int minibatch;
  int gate_channel;        // gate_logit holds one logit per feature ([B, H, T, d])
  int ablate;              // ablation gradient (prediction removed, Jacobian kept)
  int norm_match;          // ... rescaled per token to the full gradient's norm
  float* grad_norms;       // [B, H, T, 2] per-token gradient norms (ablation), may be null
  int kq_silu;             // the `:mlp` variant: SiLU on every key and query as it is loaded
};

// Gradient variant of the CUDA-core chain: 0 simplified, 1 LN Jacobian, 2 no
// LayerNorm, 3 ablation, 4 ablation that also forms the full gradient's norm
// (per-token norm matching, or the gradient norms asked for).
inline int grad_variant(const ScanParams& p) {
  if (p.no_ln) return 2;
  if (p.ablate) return (p.norm_match || p.grad_norms) ? 4 : 3;
  return p.lnjac ? 1 : 0;
}

enum : int { kStatusOk = 0, kStatusTimeout = 1 };

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

// SiLU(x) = x sigmoid(x), the activation of the `:mlp` variant ("Edifice.Recurrent.TTT",
// `build` options, `:variant`) on keys and queries.
__device__ __forceinline__ float siluf_(float x) { return x * sigmoidf_(x); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Load 16 bytes of InT from global memory and widen to fp32.
template <typename InT>
struct Vec16;
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float* out) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(p));
    out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
  }
};
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* out) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

}  // namespace ttt
