// Launchers of the CUDA-core per-token kernel that spreads each head over a
// cluster of CTAs (scan_cluster.cuh).
#include "ttt_scan.h"
#include "launch.h"
#include "scan_cluster.cuh"

namespace {

constexpr int kClusterSize = 4;

template <typename InT, typename OutT, int GM>
struct ClusterLaunch {
  using L = ttt::ClusterLayout<InT, kClusterSize>;
  static cudaLaunchConfig_t config(long long heads, cudaStream_t stream,
                                   cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(heads * kClusterSize), 1, 1);
    cfg.blockDim = dim3(L::NT, 1, 1);
    cfg.dynamicSmemBytes = L::launch_bytes;
    cfg.stream = stream;
    attr->id = cudaLaunchAttributeClusterDimension;
    attr->val.clusterDim.x = kClusterSize;
    attr->val.clusterDim.y = 1;
    attr->val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
  }
  // Clusters of this kernel that can be resident at once on the current
  // device (0 if the query fails); cached per device.
  static int capacity() {
    static int cache[64] = {};  // value + 1; 0 = not queried yet
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cache[dev] == 0) {
      auto kernel = ttt::scan_cluster_kernel<InT, OutT, GM, kClusterSize>;
      int n = 0;
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               L::launch_bytes) == cudaSuccess) {
        cudaLaunchAttribute attr;
        const cudaLaunchConfig_t cfg = config(1, nullptr, &attr);
        if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) n = 0;
      }
      cudaGetLastError();  // a failed query must not leave a sticky launch error
      cache[dev] = n + 1;
    }
    return cache[dev] - 1;
  }
  static int launch(const ttt::ScanParams& p, cudaStream_t stream) {
    auto kernel = ttt::scan_cluster_kernel<InT, OutT, GM, kClusterSize>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::launch_bytes) != cudaSuccess)
      return TTT_ERR_CUDA;
    cudaLaunchAttribute attr;
    const cudaLaunchConfig_t cfg = config((long long)p.B * p.H, stream, &attr);
    if (cudaLaunchKernelEx(&cfg, kernel, p) != cudaSuccess) return TTT_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
  }
};

template <typename InT, typename OutT, int GM>
int cluster_one(const ttt::ScanParams* p, cudaStream_t s, int* capacity) {
  if (capacity) {
    *capacity = ClusterLaunch<InT, OutT, GM>::capacity();
    return TTT_OK;
  }
  return ClusterLaunch<InT, OutT, GM>::launch(*p, s);
}

// gm: 0 simplified, 1 LN Jacobian, 2 no LayerNorm, 3 ablation, 4 ablation with
// per-token norm matching (the gradient norms are written by the one-CTA kernel).
template <typename InT, typename OutT>
int cluster_dispatch(const ttt::ScanParams* p, int gm, cudaStream_t s, int* capacity) {
  switch (gm) {
    case 0: return cluster_one<InT, OutT, 0>(p, s, capacity);
    case 1: return cluster_one<InT, OutT, 1>(p, s, capacity);
    case 3: return cluster_one<InT, OutT, 3>(p, s, capacity);
    case 4: return cluster_one<InT, OutT, 4>(p, s, capacity);
    default: return cluster_one<InT, OutT, 2>(p, s, capacity);
  }
}

int call(const ttt::ScanParams* p, unsigned mode, int gm, cudaStream_t s, int* capacity) {
  const bool in_bf16 = mode & TTT_IN_BF16, out_bf16 = mode & TTT_OUT_BF16;
  if (in_bf16 && out_bf16) return cluster_dispatch<__nv_bfloat16, __nv_bfloat16>(p, gm, s, capacity);
  if (in_bf16) return cluster_dispatch<__nv_bfloat16, float>(p, gm, s, capacity);
  if (out_bf16) return cluster_dispatch<float, __nv_bfloat16>(p, gm, s, capacity);
  return cluster_dispatch<float, float>(p, gm, s, capacity);
}

}  // namespace

namespace ttt {

int launch_cluster(const ScanParams& p, unsigned mode, int gm, cudaStream_t stream) {
  return call(&p, mode, gm, stream, nullptr);
}

int cluster_status_take() {
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, g_cluster_status, sizeof(int)) != cudaSuccess) return -1;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_cluster_status, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return h;
}

int cluster_capacity(unsigned mode, int gm) {
  int cap = 0;
  call(nullptr, mode, gm, nullptr, &cap);
  return cap;
}

}  // namespace ttt
