// C-ABI entry points of the TTT-Linear scan: argument checks, kernel choice,
// launch, and the device status word. See include/ttt_scan.h for the contract.

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <type_traits>

#include "ttt_scan.h"
#include "common.cuh"
#include "scan_simt.cuh"  // chunk limit kC (the kernels themselves are instantiated elsewhere)
#include "scan_tc.cuh"
#include "decode.cuh"
#include "launch.h"
#include "abi_util.h"

#include <cudaTypedefs.h>

namespace {

long long g_wait_limit = 1LL << 20;

constexpr unsigned kKnownModes = TTT_MODE_MINIBATCH | TTT_GRAD_LNJAC | TTT_NO_LN |
                                 TTT_IN_BF16 | TTT_OUT_BF16 | TTT_KERNEL_SIMT |
                                 TTT_GATE_CHANNEL | TTT_KERNEL_SINGLE_CTA | TTT_GRAD_ABLATE |
                                 TTT_GRAD_NORM_MATCH | TTT_KQ_SILU;

// Gradient-mode combinations that make no sense, whatever the kernel.
bool bad_grad_mode(unsigned mode) {
  if ((mode & TTT_GRAD_ABLATE) && (mode & TTT_NO_LN)) return true;
  if ((mode & TTT_GRAD_NORM_MATCH) && !(mode & TTT_GRAD_ABLATE)) return true;
  return false;
}

using ttt::abi::misaligned;
using ttt::abi::overlaps;

// Largest divisor of b that is <= cap.
int largest_divisor_upto(int b, int cap) {
  for (int c = cap < b ? cap : b; c > 1; --c)
    if (b % c == 0) return c;
  return 1;
}

// Gradient variant of a call (as ttt::grad_variant): 0 simplified, 1 LN
// Jacobian, 2 no LayerNorm, 3 ablation, 4 ablation with norm matching or with
// the gradient norms written.
int grad_variant_of(unsigned mode, bool norms) {
  if (mode & TTT_NO_LN) return 2;
  if (mode & TTT_GRAD_ABLATE) return ((mode & TTT_GRAD_NORM_MATCH) || norms) ? 4 : 3;
  return (mode & TTT_GRAD_LNJAC) ? 1 : 0;
}

// Which kernel a valid call runs (see ttt_scan_kernel_choice in the header).
// `norms`: the gradient norms are asked for (ttt_scan_forward_grad_norms).
int choose_kernel(long long heads, int T, int d, unsigned mode, int b, bool norms) {
  if (heads == 0) return TTT_KERNEL_NONE;
  const bool minibatch = mode & TTT_MODE_MINIBATCH;
  if (minibatch && (mode & TTT_IN_BF16) && d == 64 && b == ttt::tc::CB &&
      !(mode & TTT_KERNEL_SIMT) && T > 0)
    return TTT_KERNEL_ID_TENSOR_CORE;
  if (!minibatch && d == 64 && !(mode & TTT_KERNEL_SINGLE_CTA) && !norms && T > 0) {
    if (heads <= ttt::cluster_capacity(mode, grad_variant_of(mode, norms)))
      return TTT_KERNEL_ID_CUDA_CORE_CLUSTER;
  }
  return TTT_KERNEL_ID_CUDA_CORE;
}

// The CUDA-core kernels apply the SiLU variant to fp32 tiles only (a bf16
// tile would round SiLU(k) back to bf16); the tensor-core kernel reads bf16
// operands anyway.
bool silu_unsupported(int kernel, unsigned mode) {
  return (mode & TTT_KQ_SILU) && (mode & TTT_IN_BF16) && kernel != TTT_KERNEL_ID_TENSOR_CORE &&
         kernel != TTT_KERNEL_NONE;
}

// ---- tensor-core kernel: tensor maps and launch ----
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// [B*H][T][64] bf16 viewed as a 3-D tensor {64, T, B*H}; box {64, 16, 1}.
bool encode_qkv_map(CUtensorMap* map, const void* base, int T, long long heads, bool swizzle) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {64, (cuuint64_t)T, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {64 * 2, (cuuint64_t)T * 64 * 2};
  const cuuint32_t box[3] = {64, 16, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The output [B*H][T][64] (bf16 or fp32) in the same view and box, no swizzle:
// the kernel stores a token-major tile of 16 rows per chunk.
bool encode_out_map(CUtensorMap* map, void* base, int T, long long heads, bool bf16) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t elt = bf16 ? 2 : 4;
  const cuuint64_t dims[3] = {64, (cuuint64_t)T, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {64 * elt, (cuuint64_t)T * 64 * elt};
  const cuuint32_t box[3] = {64, 16, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                        3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <typename OutT, int GM>
int launch_tc(const ttt::ScanParams& p, cudaStream_t stream) {
  ttt::TcMaps maps;
  const long long heads = (long long)p.B * p.H;
  if (!encode_qkv_map(&maps.q, p.q, p.T, heads, true) ||
      !encode_qkv_map(&maps.k, p.k, p.T, heads, true) ||
      !encode_qkv_map(&maps.v, p.v, p.T, heads, false) ||
      !encode_out_map(&maps.o, p.o, p.T, heads, std::is_same<OutT, __nv_bfloat16>::value))
    return TTT_ERR_CUDA;
  // Up to one head per SM: the one-CTA-per-SM build (more registers per
  // thread, deeper staging); beyond that two CTAs share an SM. The kernel of
  // scan_tc_many.cuh fits three per SM, with a chunk loop about 1.5 times as
  // long: it goes where it saves a wave, (waves at three per SM) * 1.5 <
  // (waves at two per SM), i.e. for 2 to 3 heads per SM.
  const long long sms = ttt::device_sm_count();
  const bool one = heads <= sms;
  if (sms > 0 && !p.gate_channel) {  // (the three-per-SM kernel has no per-feature gate)
    const long long waves2 = (heads + 2 * sms - 1) / (2 * sms);
    const long long waves3 = (heads + 3 * sms - 1) / (3 * sms);
    if (3 * waves3 < 2 * waves2)
      return ttt::launch_tc_many(p, &maps.q, &maps.k, &maps.v, &maps.o,
                                 std::is_same<OutT, __nv_bfloat16>::value, GM, stream);
  }
  constexpr int kMany = ttt::tc::kMinbMany;
  const bool g = p.gate_channel != 0;
  auto kernel = one ? (g ? ttt::scan_tc_kernel<OutT, GM, 1, true>
                         : ttt::scan_tc_kernel<OutT, GM, 1, false>)
                    : (g ? ttt::scan_tc_kernel<OutT, GM, kMany, true>
                         : ttt::scan_tc_kernel<OutT, GM, kMany, false>);
  const int smem = one ? (g ? ttt::tc::smem_bytes<1, true>() : ttt::tc::smem_bytes<1, false>())
                       : (g ? ttt::tc::smem_bytes<kMany, true>()
                            : ttt::tc::smem_bytes<kMany, false>());
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return TTT_ERR_CUDA;
  kernel<<<(unsigned)heads, ttt::tc::nt_for(one ? 1 : kMany), smem, stream>>>(p, maps);
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

template <typename OutT>
int dispatch_tc_gm(const ttt::ScanParams& p, cudaStream_t s) {
  switch (ttt::grad_variant(p)) {
    case 0: return launch_tc<OutT, 0>(p, s);
    case 1: return launch_tc<OutT, 1>(p, s);
    case 3: return launch_tc<OutT, 3>(p, s);
    case 4: return launch_tc<OutT, 4>(p, s);
    default: return launch_tc<OutT, 2>(p, s);
  }
}

int dispatch_tc(const ttt::ScanParams& p, unsigned mode, cudaStream_t s) {
  return (mode & TTT_OUT_BF16) ? dispatch_tc_gm<__nv_bfloat16>(p, s) : dispatch_tc_gm<float>(p, s);
}

template <int D, typename InT, typename OutT>
int launch_decode(const ttt::DecodeParams& p, cudaStream_t stream) {
  using S = ttt::DecodeShape<D>;
  const long long blocks = (p.heads + S::HPB - 1) / S::HPB;
  ttt::decode_step_kernel<D, InT, OutT><<<(unsigned)blocks, S::NT, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

template <int D>
int dispatch_decode(const ttt::DecodeParams& p, unsigned mode, cudaStream_t s) {
  const bool in_bf16 = mode & TTT_IN_BF16, out_bf16 = mode & TTT_OUT_BF16;
  if (in_bf16 && out_bf16) return launch_decode<D, __nv_bfloat16, __nv_bfloat16>(p, s);
  if (in_bf16) return launch_decode<D, __nv_bfloat16, float>(p, s);
  if (out_bf16) return launch_decode<D, float, __nv_bfloat16>(p, s);
  return launch_decode<D, float, float>(p, s);
}

}  // namespace

namespace ttt {

int device_sm_count() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

}  // namespace ttt

extern "C" {

const char* ttt_status_string(int status) {
  switch (status) {
    case TTT_OK: return "TTT_OK";
    case TTT_ERR_INVALID_ARG: return "TTT_ERR_INVALID_ARG";
    case TTT_ERR_UNSUPPORTED: return "TTT_ERR_UNSUPPORTED";
    case TTT_ERR_CUDA: return "TTT_ERR_CUDA";
    case TTT_ERR_DEVICE_TIMEOUT: return "TTT_ERR_DEVICE_TIMEOUT";
    default: return "TTT_UNKNOWN_STATUS";
  }
}

int ttt_set_wait_limit(long long polls) {
  if (polls < 0) return TTT_ERR_INVALID_ARG;
  g_wait_limit = polls;
  return TTT_OK;
}

int ttt_check_device_status(void* cuda_stream) {
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return TTT_ERR_CUDA;
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, ttt::g_ttt_status, sizeof(int)) != cudaSuccess) return TTT_ERR_CUDA;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(ttt::g_ttt_status, &zero, sizeof(int)) != cudaSuccess) return TTT_ERR_CUDA;
  }
  const int hc = ttt::cluster_status_take();
  const int hm = ttt::tc_many_status_take();
  if (hc < 0 || hm < 0) return TTT_ERR_CUDA;
  return (h != 0 || hc != 0 || hm != 0) ? TTT_ERR_DEVICE_TIMEOUT : TTT_OK;
}

static int scan_forward(const void* q, const void* k, const void* v, const void* eta_logit,
                        const void* gate_logit, const float* W0, const float* gamma,
                        const float* beta, int B, int H, int T, int d, float eps, unsigned mode,
                        int b, const unsigned char* mask, void* o, float* W_T, float* W_chunks,
                        float* grad_norms, void* cuda_stream) {
  // ---- argument checks (nothing is launched on failure) ----
  if ((mode & ~kKnownModes) || bad_grad_mode(mode)) return TTT_ERR_INVALID_ARG;
  if (grad_norms && !(mode & TTT_GRAD_ABLATE)) return TTT_ERR_INVALID_ARG;
  if (B < 0 || H < 0 || T < 0 || b < 1 || d <= 0) return TTT_ERR_INVALID_ARG;
  const bool no_ln = mode & TTT_NO_LN;
  // a pointer may be null only where the tensor it names is empty
  const bool has_heads = (long long)B * H > 0;
  if (has_heads && T > 0 && (!q || !k || !v || !eta_logit || !o)) return TTT_ERR_INVALID_ARG;
  if (has_heads && (!W0 || !W_T)) return TTT_ERR_INVALID_ARG;
  if (has_heads && !no_ln && (!gamma || !beta)) return TTT_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, eta_logit, gate_logit, W0, gamma, beta, mask, o, W_T, W_chunks,
                        grad_norms};
  for (const void* p : ptrs)
    if (misaligned(p)) return TTT_ERR_INVALID_ARG;
  if (d != 16 && d != 64) return TTT_ERR_UNSUPPORTED;
  if ((long long)B * H > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
  const int which = choose_kernel((long long)B * H, T, d, mode, b, grad_norms != nullptr);
  if (silu_unsupported(which, mode)) return TTT_ERR_UNSUPPORTED;
  if (which == TTT_KERNEL_ID_CUDA_CORE && (mode & TTT_MODE_MINIBATCH) && b > ttt::kC)
    return TTT_ERR_UNSUPPORTED;

  const size_t heads = (size_t)B * H;
  const int n_mask_chunks = (T + b - 1) / b;
  const size_t in_elt = (mode & TTT_IN_BF16) ? 2 : 4;
  const size_t out_elt = (mode & TTT_OUT_BF16) ? 2 : 4;
  const size_t tok_bytes = heads * (size_t)T * d * in_elt;
  const size_t scal_bytes = heads * (size_t)T * in_elt;
  const size_t o_bytes = heads * (size_t)T * d * out_elt;
  const size_t w_bytes = heads * (size_t)d * d * sizeof(float);
  const size_t gb_bytes = (size_t)H * d * sizeof(float);
  const size_t mask_bytes = (size_t)B * n_mask_chunks;
  const size_t wc_bytes = heads * (size_t)(n_mask_chunks + 1) * d * d * sizeof(float);
  struct Span { const void* p; size_t n; };
  const size_t gate_bytes = (mode & TTT_GATE_CHANNEL) ? tok_bytes : scal_bytes;
  const Span inputs[] = {{q, tok_bytes}, {k, tok_bytes}, {v, tok_bytes},
                         {eta_logit, scal_bytes}, {gate_logit, gate_bytes},
                         {W0, w_bytes}, {gamma, no_ln ? 0 : gb_bytes},
                         {beta, no_ln ? 0 : gb_bytes}, {mask, mask ? mask_bytes : 0}};
  for (const Span& in : inputs) {
    if (overlaps(o, o_bytes, in.p, in.n)) return TTT_ERR_INVALID_ARG;
    if (in.p != W0 && overlaps(W_T, w_bytes, in.p, in.n)) return TTT_ERR_INVALID_ARG;
    if (W_chunks && overlaps(W_chunks, wc_bytes, in.p, in.n)) return TTT_ERR_INVALID_ARG;
  }
  if (W_T != W0 && overlaps(W_T, w_bytes, W0, w_bytes)) return TTT_ERR_INVALID_ARG;
  if (overlaps(o, o_bytes, W_T, w_bytes)) return TTT_ERR_INVALID_ARG;
  if (W_chunks && (overlaps(W_chunks, wc_bytes, o, o_bytes) ||
                   overlaps(W_chunks, wc_bytes, W_T, w_bytes)))
    return TTT_ERR_INVALID_ARG;
  if (grad_norms) {
    const size_t gn_bytes = heads * (size_t)T * 2 * sizeof(float);
    for (const Span& in : inputs)
      if (overlaps(grad_norms, gn_bytes, in.p, in.n)) return TTT_ERR_INVALID_ARG;
    if (overlaps(grad_norms, gn_bytes, o, o_bytes) || overlaps(grad_norms, gn_bytes, W_T, w_bytes) ||
        (W_chunks && overlaps(grad_norms, gn_bytes, W_chunks, wc_bytes)))
      return TTT_ERR_INVALID_ARG;
  }
  if (heads == 0) return TTT_OK;

  ttt::ScanParams p{};
  p.q = q; p.k = k; p.v = v; p.eta_logit = eta_logit; p.gate_logit = gate_logit;
  p.W0 = W0; p.gamma = gamma; p.beta = beta; p.mask = mask;
  p.o = o; p.W_T = W_T; p.W_chunks = W_chunks;
  p.status = nullptr;
  p.wait_limit = g_wait_limit;
  p.B = B; p.H = H; p.T = T; p.b = b; p.n_mask_chunks = n_mask_chunks;
  p.eps = eps;
  p.lnjac = (mode & TTT_GRAD_LNJAC) ? 1 : 0;
  p.no_ln = no_ln ? 1 : 0;
  p.minibatch = (mode & TTT_MODE_MINIBATCH) ? 1 : 0;
  p.ablate = (mode & TTT_GRAD_ABLATE) ? 1 : 0;
  p.norm_match = (mode & TTT_GRAD_NORM_MATCH) ? 1 : 0;
  p.gate_channel = (mode & TTT_GATE_CHANNEL) ? 1 : 0;
  p.grad_norms = grad_norms;
  p.kq_silu = (mode & TTT_KQ_SILU) ? 1 : 0;

  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  if (which == TTT_KERNEL_ID_TENSOR_CORE) return dispatch_tc(p, mode, stream);
  if (p.minibatch) {
    p.C = b;
  } else {
    // chunks must not straddle a mask / snapshot boundary when either is asked for
    p.C = (mask || W_chunks) ? largest_divisor_upto(b, ttt::kC) : ttt::kC;
  }
  if (which == TTT_KERNEL_ID_CUDA_CORE_CLUSTER)
    return ttt::launch_cluster(p, mode, ttt::grad_variant(p), stream);
  if (mode & TTT_IN_BF16)
    return p.minibatch ? ttt::launch_simt_bf16_minibatch(p, mode, d, stream)
                       : ttt::launch_simt_bf16_pertoken(p, mode, d, stream);
  return p.minibatch ? ttt::launch_simt_f32_minibatch(p, mode, d, stream)
                     : ttt::launch_simt_f32_pertoken(p, mode, d, stream);
}

int ttt_scan_forward(const void* q, const void* k, const void* v, const void* eta_logit,
                     const void* gate_logit, const float* W0, const float* gamma,
                     const float* beta, int B, int H, int T, int d, float eps, unsigned mode,
                     int b, const unsigned char* mask, void* o, float* W_T, float* W_chunks,
                     void* cuda_stream) {
  return scan_forward(q, k, v, eta_logit, gate_logit, W0, gamma, beta, B, H, T, d, eps, mode, b,
                      mask, o, W_T, W_chunks, nullptr, cuda_stream);
}

int ttt_scan_forward_grad_norms(const void* q, const void* k, const void* v,
                                const void* eta_logit, const void* gate_logit, const float* W0,
                                const float* gamma, const float* beta, int B, int H, int T,
                                int d, float eps, unsigned mode, int b,
                                const unsigned char* mask, void* o, float* W_T, float* W_chunks,
                                float* grad_norms, void* cuda_stream) {
  if (!grad_norms && (long long)B * H * T > 0) return TTT_ERR_INVALID_ARG;
  return scan_forward(q, k, v, eta_logit, gate_logit, W0, gamma, beta, B, H, T, d, eps, mode, b,
                      mask, o, W_T, W_chunks, grad_norms, cuda_stream);
}

int ttt_scan_kernel_choice(int B, int H, int T, int d, unsigned mode, int b) {
  if ((mode & ~kKnownModes) || bad_grad_mode(mode)) return TTT_ERR_INVALID_ARG;
  if (B < 0 || H < 0 || T < 0 || b < 1 || d <= 0) return TTT_ERR_INVALID_ARG;
  if (d != 16 && d != 64) return TTT_ERR_UNSUPPORTED;
  if ((long long)B * H > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
  const int which = choose_kernel((long long)B * H, T, d, mode, b, false);
  if (silu_unsupported(which, mode)) return TTT_ERR_UNSUPPORTED;
  if (which == TTT_KERNEL_ID_CUDA_CORE && (mode & TTT_MODE_MINIBATCH) && b > ttt::kC)
    return TTT_ERR_UNSUPPORTED;
  return which;
}

int ttt_decode_step(const void* q, const void* k, const void* v, const void* eta_logit,
                    const void* gate_logit, float* W, const float* gamma, const float* beta,
                    int B, int H, int d, float eps, unsigned mode, const unsigned char* update,
                    void* o, void* cuda_stream) {
  if ((mode & ~kKnownModes) || bad_grad_mode(mode)) return TTT_ERR_INVALID_ARG;
  if (B < 0 || H < 0 || d <= 0) return TTT_ERR_INVALID_ARG;
  const bool no_ln = mode & TTT_NO_LN;
  const bool has_heads = (long long)B * H > 0;
  if (has_heads && (!q || !k || !v || !eta_logit || !W || !o)) return TTT_ERR_INVALID_ARG;
  if (has_heads && !no_ln && (!gamma || !beta)) return TTT_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, eta_logit, gate_logit, W, gamma, beta, update, o};
  for (const void* p : ptrs)
    if (misaligned(p)) return TTT_ERR_INVALID_ARG;
  if (d != 16 && d != 64) return TTT_ERR_UNSUPPORTED;
  if (mode & TTT_MODE_MINIBATCH) return TTT_ERR_UNSUPPORTED;
  if ((long long)B * H > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;

  const size_t heads = (size_t)B * H;
  const size_t in_elt = (mode & TTT_IN_BF16) ? 2 : 4;
  const size_t out_elt = (mode & TTT_OUT_BF16) ? 2 : 4;
  const size_t vec_bytes = heads * d * in_elt;
  const size_t scal_bytes = heads * in_elt;
  const size_t gate_bytes = (mode & TTT_GATE_CHANNEL) ? vec_bytes : scal_bytes;
  const size_t o_bytes = heads * d * out_elt;
  const size_t w_bytes = heads * (size_t)d * d * sizeof(float);
  const size_t gb_bytes = (size_t)H * d * sizeof(float);
  struct Span { const void* p; size_t n; };
  const Span inputs[] = {{q, vec_bytes}, {k, vec_bytes}, {v, vec_bytes},
                         {eta_logit, scal_bytes}, {gate_logit, gate_bytes},
                         {gamma, no_ln ? 0 : gb_bytes}, {beta, no_ln ? 0 : gb_bytes},
                         {update, update ? (size_t)B : 0}};
  for (const Span& in : inputs) {
    if (overlaps(o, o_bytes, in.p, in.n)) return TTT_ERR_INVALID_ARG;
    if (overlaps(W, w_bytes, in.p, in.n)) return TTT_ERR_INVALID_ARG;
  }
  if (overlaps(o, o_bytes, W, w_bytes)) return TTT_ERR_INVALID_ARG;
  if (heads == 0) return TTT_OK;

  ttt::DecodeParams p{};
  p.q = q; p.k = k; p.v = v; p.eta_logit = eta_logit; p.gate_logit = gate_logit;
  p.W = W; p.gamma = gamma; p.beta = beta; p.update = update; p.o = o;
  p.heads = (long long)heads;
  p.H = H;
  p.eps = eps;
  p.lnjac = (mode & TTT_GRAD_LNJAC) ? 1 : 0;
  p.no_ln = no_ln ? 1 : 0;
  p.gate_channel = (mode & TTT_GATE_CHANNEL) ? 1 : 0;
  p.ablate = (mode & TTT_GRAD_ABLATE) ? 1 : 0;
  p.norm_match = (mode & TTT_GRAD_NORM_MATCH) ? 1 : 0;
  p.kq_silu = (mode & TTT_KQ_SILU) ? 1 : 0;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  return d == 64 ? dispatch_decode<64>(p, mode, stream) : dispatch_decode<16>(p, mode, stream);
}

}  // extern "C"
