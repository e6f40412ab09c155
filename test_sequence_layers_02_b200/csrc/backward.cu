// C-ABI entry points of the scan's backward pass: argument checks, workspace
// size, launch of the per-head kernel and of the gamma / beta reduction over
// batch rows. See include/ttt_scan.h for the contract.
#include <cmath>

#include "ttt_scan.h"
#include "abi_util.h"
#include "scan_bwd.cuh"

namespace {

using ttt::abi::misaligned;
using ttt::abi::overlaps;
using ttt::abi::Span;

constexpr unsigned kKnownModes = TTT_MODE_MINIBATCH | TTT_GRAD_LNJAC | TTT_NO_LN |
                                 TTT_IN_BF16 | TTT_OUT_BF16 | TTT_KERNEL_SIMT |
                                 TTT_GATE_CHANNEL | TTT_KERNEL_SINGLE_CTA | TTT_GRAD_ABLATE |
                                 TTT_GRAD_NORM_MATCH | TTT_KQ_SILU;

template <int D, typename InT, bool MINIB, int GM>
int launch_bwd(const ttt::BwdParams& p, cudaStream_t s) {
  using L = ttt::BwdLayout<D>;
  auto kernel = ttt::scan_bwd_kernel<D, InT, MINIB, GM>;
  if (L::bytes > 48 * 1024 &&
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::bytes) !=
          cudaSuccess)
    return TTT_ERR_CUDA;
  kernel<<<(unsigned)((long long)p.B * p.H), L::NT, L::bytes, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

template <int D, typename InT, bool MINIB>
int dispatch_gm(const ttt::BwdParams& p, unsigned mode, cudaStream_t s) {
  if (mode & TTT_NO_LN) return launch_bwd<D, InT, MINIB, 2>(p, s);
  if (mode & TTT_GRAD_ABLATE) return launch_bwd<D, InT, MINIB, 3>(p, s);
  if (mode & TTT_GRAD_LNJAC) return launch_bwd<D, InT, MINIB, 1>(p, s);
  return launch_bwd<D, InT, MINIB, 0>(p, s);
}

template <int D, typename InT>
int dispatch_mode(const ttt::BwdParams& p, unsigned mode, cudaStream_t s) {
  return (mode & TTT_MODE_MINIBATCH) ? dispatch_gm<D, InT, true>(p, mode, s)
                                     : dispatch_gm<D, InT, false>(p, mode, s);
}

template <int D>
int dispatch_in(const ttt::BwdParams& p, unsigned mode, cudaStream_t s) {
  return (mode & TTT_IN_BF16) ? dispatch_mode<D, __nv_bfloat16>(p, mode, s)
                              : dispatch_mode<D, float>(p, mode, s);
}

size_t workspace_bytes_for(int B, int H, int d, unsigned mode) {
  if ((mode & TTT_NO_LN) || B <= 0 || H <= 0 || d <= 0) return 0;
  return (size_t)B * H * 2 * d * sizeof(float);
}

}  // namespace

extern "C" {

size_t ttt_scan_backward_workspace_bytes(int B, int H, int d, unsigned mode) {
  return workspace_bytes_for(B, H, d, mode);
}

int ttt_scan_backward(const void* q, const void* k, const void* v, const void* eta_logit,
                      const void* gate_logit, const float* gamma, const float* beta, int B, int H,
                      int T, int d, float eps, unsigned mode, int b, const unsigned char* mask,
                      const float* W_chunks, const float* dO, const float* dW_T, float* dq,
                      float* dk, float* dv, float* d_eta_logit, float* d_gate_logit, float* dW0,
                      float* dgamma, float* dbeta, void* workspace, size_t workspace_bytes,
                      void* cuda_stream) {
  // ---- argument checks (nothing is launched on failure) ----
  if (mode & ~kKnownModes) return TTT_ERR_INVALID_ARG;
  if ((mode & TTT_GRAD_ABLATE) && (mode & TTT_NO_LN)) return TTT_ERR_INVALID_ARG;
  if ((mode & TTT_GRAD_NORM_MATCH) && !(mode & TTT_GRAD_ABLATE)) return TTT_ERR_INVALID_ARG;
  if (B < 0 || H < 0 || T < 0 || b < 1 || d <= 0) return TTT_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return TTT_ERR_INVALID_ARG;
  const bool no_ln = mode & TTT_NO_LN;
  const bool heads = (long long)B * H > 0;
  const bool toks = heads && T > 0;
  if (toks && (!q || !k || !v || !eta_logit || !dO || !dq || !dk || !dv || !d_eta_logit))
    return TTT_ERR_INVALID_ARG;
  if (heads && (!W_chunks || !dW0)) return TTT_ERR_INVALID_ARG;
  if (toks && gate_logit && !d_gate_logit) return TTT_ERR_INVALID_ARG;
  if (heads && !no_ln && (!gamma || !beta || !dgamma || !dbeta)) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, eta_logit, gate_logit, gamma, beta, mask, W_chunks, dO, dW_T,
                        dq, dk, dv, d_eta_logit, d_gate_logit, dW0, dgamma, dbeta, workspace};
  for (const void* p : ptrs)
    if (misaligned(p)) return TTT_ERR_INVALID_ARG;
  const size_t need = workspace_bytes_for(B, H, d, mode);
  if (need > 0 && (!workspace || workspace_bytes < need)) return TTT_ERR_INVALID_ARG;
  if (d != 16 && d != 64) return TTT_ERR_UNSUPPORTED;
  if (b > ttt::kC) return TTT_ERR_UNSUPPORTED;
  if (mode & TTT_GRAD_NORM_MATCH) return TTT_ERR_UNSUPPORTED;
  if ((long long)B * H > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;

  const size_t nh = (size_t)B * H;
  const int nc = (T + b - 1) / b;
  const size_t ie = (mode & TTT_IN_BF16) ? 2 : 4;
  const size_t tok_in = nh * T * d * ie, scal_in = nh * T * ie;
  const size_t gate_in = (mode & TTT_GATE_CHANNEL) ? tok_in : scal_in;
  const size_t tok_f = nh * T * d * 4, scal_f = nh * T * 4;
  const size_t gate_f = (mode & TTT_GATE_CHANNEL) ? tok_f : scal_f;
  const size_t w_f = nh * d * d * 4, gb_f = (size_t)H * d * 4;
  const Span inputs[] = {{q, tok_in}, {k, tok_in}, {v, tok_in}, {eta_logit, scal_in},
                         {gate_logit, gate_in}, {gamma, no_ln ? 0 : gb_f},
                         {beta, no_ln ? 0 : gb_f}, {mask, mask ? (size_t)B * nc : 0},
                         {W_chunks, nh * (nc + 1) * d * d * 4}, {dO, tok_f},
                         {dW_T, dW_T ? w_f : 0}};
  const Span outputs[] = {{dq, tok_f}, {dk, tok_f}, {dv, tok_f}, {d_eta_logit, scal_f},
                          {d_gate_logit, gate_logit ? gate_f : 0}, {dW0, w_f},
                          {dgamma, no_ln ? 0 : gb_f}, {dbeta, no_ln ? 0 : gb_f},
                          {workspace, need}};
  for (const Span& o : outputs) {
    for (const Span& in : inputs)
      if (overlaps(o.p, o.n, in.p, in.n)) return TTT_ERR_INVALID_ARG;
    for (const Span& o2 : outputs)
      if (&o2 != &o && overlaps(o.p, o.n, o2.p, o2.n)) return TTT_ERR_INVALID_ARG;
  }
  if (!heads) {
    // no heads: only the gamma / beta gradients (zero) have elements
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    if (!no_ln && H > 0) {
      if (cudaMemsetAsync(dgamma, 0, gb_f, s) != cudaSuccess ||
          cudaMemsetAsync(dbeta, 0, gb_f, s) != cudaSuccess)
        return TTT_ERR_CUDA;
    }
    return TTT_OK;
  }

  ttt::BwdParams p{};
  p.q = q; p.k = k; p.v = v; p.eta_logit = eta_logit; p.gate_logit = gate_logit;
  p.gamma = no_ln ? nullptr : gamma;
  p.beta = no_ln ? nullptr : beta;
  p.mask = mask; p.W_chunks = W_chunks; p.dO = dO; p.dW_T = dW_T;
  p.dq = dq; p.dk = dk; p.dv = dv; p.deta = d_eta_logit; p.dgate = d_gate_logit; p.dW0 = dW0;
  p.gb_part = no_ln ? nullptr : static_cast<float*>(workspace);
  p.B = B; p.H = H; p.T = T; p.b = b; p.n_chunks = nc;
  p.eps = eps;
  p.gate_channel = (mode & TTT_GATE_CHANNEL) ? 1 : 0;
  p.kq_silu = (mode & TTT_KQ_SILU) ? 1 : 0;

  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const int rc = d == 64 ? dispatch_in<64>(p, mode, s) : dispatch_in<16>(p, mode, s);
  if (rc != TTT_OK || no_ln) return rc;
  const int n = H * d;
  ttt::bwd_reduce_gb_kernel<<<(n + 255) / 256, 256, 0, s>>>(p.gb_part, B, H, d, dgamma, dbeta);
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

}  // extern "C"

// ---- The no-allocation variant: the same backward with its scratch in a fixed
// device array, for callers that cannot call cudaMalloc. ----
namespace {

// The per-head dgamma / dbeta partial sums of ttt_scan_backward_noalloc: room
// for 2^20 floats (4 MiB), i.e. B * H * 2 * d <= 2^20 (8192 heads at d = 64,
// 32768 at d = 16). A file-scope device array: every GPU that loads the
// library holds it until the process exits.
constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;
static __device__ __align__(256) float g_bwd_scratch[kNoAllocScratchFloats];

// Device address of g_bwd_scratch on the current device. In host code the
// array's name stands for a host-side shadow, not for device memory, so the
// address is looked up (once per device, with that device current) and cached.
float* noalloc_scratch_current_device() {
  static float* cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (cache[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_bwd_scratch) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<float*>(ptr);
  }
  return cache[dev];
}

}  // namespace

extern "C" int ttt_scan_backward_noalloc(
    const void* q, const void* k, const void* v, const void* eta_logit, const void* gate_logit,
    const float* gamma, const float* beta, int B, int H, int T, int d, float eps, unsigned mode,
    int b, const unsigned char* mask, const float* W_chunks, const float* dO, const float* dW_T,
    float* dq, float* dk, float* dv, float* d_eta_logit, float* d_gate_logit, float* dW0,
    float* dgamma, float* dbeta, void* cuda_stream) {
  const size_t need = workspace_bytes_for(B, H, d, mode);
  if (need > sizeof(g_bwd_scratch)) return TTT_ERR_UNSUPPORTED;
  float* scratch = nullptr;
  if (need > 0) {
    scratch = noalloc_scratch_current_device();
    if (scratch == nullptr) return TTT_ERR_CUDA;
  }
  return ttt_scan_backward(q, k, v, eta_logit, gate_logit, gamma, beta, B, H, T, d, eps, mode, b,
                           mask, W_chunks, dO, dW_T, dq, dk, dv, d_eta_logit, d_gate_logit, dW0,
                           dgamma, dbeta, scratch, need, cuda_stream);
}
