// Launchers of the one-CTA-per-head CUDA-core kernel for bf16 inputs.
#include "ttt_scan.h"
#include "launch.h"
#include "scan_simt.cuh"

namespace {

template <int D, typename InT, typename OutT, bool MINIB, int GM, int IH>
int launch_simt_ih(const ttt::ScanParams& p, cudaStream_t stream) {
  using L = ttt::PipeLayout<D, InT, IH>;
  auto kernel = ttt::scan_simt_kernel<D, InT, OutT, MINIB, GM, IH>;
  if (L::bytes > 48 * 1024) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)L::bytes) != cudaSuccess)
      return TTT_ERR_CUDA;
  }
  kernel<<<(unsigned)(p.B * p.H), L::NT, L::bytes, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

// Few heads (at most one CTA per SM): 8 bulk warps per CTA; otherwise 4, so
// that several CTAs share an SM.
template <int D, typename InT, typename OutT, bool MINIB, int GM>
int launch_simt(const ttt::ScanParams& p, cudaStream_t stream) {
  if constexpr (D == 64) {
    if ((long long)p.B * p.H <= 148) return launch_simt_ih<D, InT, OutT, MINIB, GM, 2>(p, stream);
  }
  return launch_simt_ih<D, InT, OutT, MINIB, GM, 1>(p, stream);
}

template <int D, typename InT, typename OutT>
int dispatch_simt_mode(const ttt::ScanParams& p, cudaStream_t s) {
  const int gm = ttt::grad_variant(p);
  if (p.minibatch) {
    if (gm == 0) return launch_simt<D, InT, OutT, true, 0>(p, s);
    if (gm == 1) return launch_simt<D, InT, OutT, true, 1>(p, s);
    return launch_simt<D, InT, OutT, true, 2>(p, s);
  }
  if (gm == 0) return launch_simt<D, InT, OutT, false, 0>(p, s);
  if (gm == 1) return launch_simt<D, InT, OutT, false, 1>(p, s);
  if (gm == 3) return launch_simt<D, InT, OutT, false, 3>(p, s);
  if (gm == 4) return launch_simt<D, InT, OutT, false, 4>(p, s);
  return launch_simt<D, InT, OutT, false, 2>(p, s);
}

template <int D>
int dispatch_out(const ttt::ScanParams& p, unsigned mode, cudaStream_t s) {
  if (mode & TTT_OUT_BF16) return dispatch_simt_mode<D, __nv_bfloat16, __nv_bfloat16>(p, s);
  return dispatch_simt_mode<D, __nv_bfloat16, float>(p, s);
}

}  // namespace

namespace ttt {

int launch_simt_bf16in(const ScanParams& p, unsigned mode, int d, cudaStream_t stream) {
  return d == 64 ? dispatch_out<64>(p, mode, stream) : dispatch_out<16>(p, mode, stream);
}

}  // namespace ttt
