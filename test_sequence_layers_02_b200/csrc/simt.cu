// Launchers of the one-CTA-per-head CUDA-core kernel (scan_simt.cuh).
//
// This one source is compiled into four objects, one per input dtype and mode
// (build.py defines TTT_SIMT_BF16 and TTT_SIMT_MINIBATCH), so the many
// instantiations of the kernel build in parallel. Each object defines one
// entry of launch.h. Arguments are already checked by the C-ABI entry points.
#include "ttt_scan.h"
#include "launch.h"
#include "scan_simt.cuh"

#if !defined(TTT_SIMT_BF16) || !defined(TTT_SIMT_MINIBATCH)
#error "simt.cu is compiled with -DTTT_SIMT_BF16=0|1 -DTTT_SIMT_MINIBATCH=0|1"
#endif

namespace {

#if TTT_SIMT_BF16
using InT = __nv_bfloat16;
#else
using InT = float;
#endif
constexpr bool kMiniBatch = TTT_SIMT_MINIBATCH != 0;

template <int D, typename OutT, int GM, int IH>
int launch_ih(const ttt::ScanParams& p, cudaStream_t stream) {
  using L = ttt::PipeLayout<D, InT, IH>;
  auto kernel = ttt::scan_simt_kernel<D, InT, OutT, kMiniBatch, GM, IH>;
  if (L::bytes > 48 * 1024) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)L::bytes) != cudaSuccess)
      return TTT_ERR_CUDA;
  }
  kernel<<<(unsigned)(p.B * p.H), L::NT, L::bytes, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

// Up to one head per SM of this device: 8 bulk warps per CTA (one CTA per
// SM); more heads: 4 bulk warps, so that three CTAs share an SM.
template <int D, typename OutT, int GM>
int launch(const ttt::ScanParams& p, cudaStream_t stream) {
  if constexpr (D == 64) {
    const int sms = ttt::device_sm_count();
    if (sms > 0 && (long long)p.B * p.H <= sms) return launch_ih<D, OutT, GM, 2>(p, stream);
  }
  return launch_ih<D, OutT, GM, 1>(p, stream);
}

template <int D, typename OutT>
int dispatch_gm(const ttt::ScanParams& p, cudaStream_t s) {
  switch (ttt::grad_variant(p)) {
    case 0: return launch<D, OutT, 0>(p, s);
    case 1: return launch<D, OutT, 1>(p, s);
    case 3: return launch<D, OutT, 3>(p, s);
    case 4: return launch<D, OutT, 4>(p, s);
    default: return launch<D, OutT, 2>(p, s);
  }
}

}  // namespace

namespace ttt {

#if TTT_SIMT_BF16 && TTT_SIMT_MINIBATCH
int launch_simt_bf16_minibatch(const ScanParams& p, unsigned mode, int d, cudaStream_t s)
#elif TTT_SIMT_BF16
int launch_simt_bf16_pertoken(const ScanParams& p, unsigned mode, int d, cudaStream_t s)
#elif TTT_SIMT_MINIBATCH
int launch_simt_f32_minibatch(const ScanParams& p, unsigned mode, int d, cudaStream_t s)
#else
int launch_simt_f32_pertoken(const ScanParams& p, unsigned mode, int d, cudaStream_t s)
#endif
{
  const bool out_bf16 = mode & TTT_OUT_BF16;
  if (d == 64) return out_bf16 ? dispatch_gm<64, __nv_bfloat16>(p, s) : dispatch_gm<64, float>(p, s);
  return out_bf16 ? dispatch_gm<16, __nv_bfloat16>(p, s) : dispatch_gm<16, float>(p, s);
}

}  // namespace ttt
