// Launcher of the tensor-core kernel built for three CTAs per SM
// (scan_tc_many.cuh). Arguments are already checked and the q / k / v tensor
// maps encoded by the C-ABI entry point.
#include "ttt_scan.h"
#include "launch.h"
#include "scan_tc_many.cuh"

namespace {

template <typename OutT, int GM>
int launch(const ttt::ScanParams& p, const ttt::tcm::TcMaps& maps, cudaStream_t stream) {
  constexpr int kMinb = ttt::tcm::tc::kMinbMany;
  auto kernel = ttt::tcm::scan_tc_kernel<OutT, GM, kMinb>;
  const int smem = ttt::tcm::tc::smem_bytes<kMinb>();
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return TTT_ERR_CUDA;
  kernel<<<(unsigned)((long long)p.B * p.H), ttt::tcm::tc::NT, smem, stream>>>(p, maps);
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

template <typename OutT>
int by_gm(const ttt::ScanParams& p, const ttt::tcm::TcMaps& maps, int gm, cudaStream_t s) {
  switch (gm) {
    case 0: return launch<OutT, 0>(p, maps, s);
    case 1: return launch<OutT, 1>(p, maps, s);
    case 3: return launch<OutT, 3>(p, maps, s);
    case 4: return launch<OutT, 4>(p, maps, s);
    default: return launch<OutT, 2>(p, maps, s);
  }
}

}  // namespace

namespace ttt {

int launch_tc_many(const ScanParams& p, const CUtensorMap* q, const CUtensorMap* k,
                   const CUtensorMap* v, const CUtensorMap* o, bool out_bf16, int gm,
                   cudaStream_t stream) {
  tcm::TcMaps maps;
  maps.q = *q;
  maps.k = *k;
  maps.v = *v;
  maps.o = *o;
  return out_bf16 ? by_gm<__nv_bfloat16>(p, maps, gm, stream) : by_gm<float>(p, maps, gm, stream);
}

int tc_many_status_take() {
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, tcm::g_tcm_status, sizeof(int)) != cudaSuccess) return -1;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(tcm::g_tcm_status, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return h;
}

}  // namespace ttt
