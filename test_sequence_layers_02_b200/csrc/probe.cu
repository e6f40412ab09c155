// FP32 FFMA throughput probe (see include/ttt_probe.h).

#include <cuda_runtime.h>

#include "ttt_probe.h"

namespace {

constexpr int kChains = 8;
constexpr int kUnroll = 16;

__global__ void ffma_probe_kernel(float* sink, int iters) {
  float a[kChains];
#pragma unroll
  for (int i = 0; i < kChains; ++i) a[i] = 1.0f + 1e-7f * (float)(threadIdx.x + i);
  const float m = 0.99999f, c = 1e-6f;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
#pragma unroll
      for (int i = 0; i < kChains; ++i) a[i] = fmaf(a[i], m, c);
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kChains; ++i) s += a[i];
  sink[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

}  // namespace

extern "C" int ttt_probe_ffma(int blocks, int threads, int iters, float* sink,
                              double* flops_out, void* cuda_stream) {
  if (blocks <= 0 || threads <= 0 || threads > 1024 || (threads & 31) || iters <= 0 ||
      !sink || !flops_out)
    return -1;
  ffma_probe_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(cuda_stream)>>>(sink, iters);
  if (cudaGetLastError() != cudaSuccess) return -3;
  *flops_out = 2.0 * kChains * kUnroll * (double)iters * (double)threads * (double)blocks;
  return 0;
}
