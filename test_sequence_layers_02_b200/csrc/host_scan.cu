// ttt_scan_forward_host: the scan with its inputs and outputs in host memory,
// the sequence cut into segments whose host<->device copies overlap the scans
// of their neighbours. See include/ttt_scan.h for the contract.
//
// Per segment i (buffers in set i % 2 of the caller's device workspace):
//   copy-in stream : wait for the scan of segment i-2 (it read this set's
//                    inputs), copy segment i's inputs in, record `in[i%2]`
//   caller's stream: wait `in[i%2]` and the copy-out of segment i-2 (it read
//                    this set's o), scan segment i from the state W the scan
//                    of segment i-1 left (in place), record `kdone[i%2]`
//   copy-out stream: wait `kdone[i%2]`, copy segment i's o out, record `out[i%2]`
// then W_T is copied out and the caller's stream waits for the copy-out
// stream. Every segment but the last is a multiple of b tokens long, so each
// chunk (and each mask byte) falls in one segment and the scans take the same
// chunks as one scan of the whole sequence would.
#include <cmath>
#include <mutex>

#include "ttt_scan.h"
#include "abi_util.h"

#include <cuda_runtime.h>

namespace {

constexpr int kMaxDevices = 64;

struct Lanes {
  bool ready = false;
  cudaStream_t copy_in = nullptr, copy_out = nullptr;
  cudaEvent_t start = nullptr, fin = nullptr;
  cudaEvent_t in[2] = {}, kdone[2] = {}, out[2] = {};
};
Lanes g_lanes[kMaxDevices];
std::mutex g_mutex;  // one call enqueues at a time (the lanes and events are shared)

// The library's copy streams and events of the current device, created once.
Lanes* lanes_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  Lanes& L = g_lanes[dev];
  if (L.ready) return &L;
  const unsigned sf = cudaStreamNonBlocking;
  const unsigned ef = cudaEventDisableTiming;
  if (cudaStreamCreateWithFlags(&L.copy_in, sf) != cudaSuccess ||
      cudaStreamCreateWithFlags(&L.copy_out, sf) != cudaSuccess ||
      cudaEventCreateWithFlags(&L.start, ef) != cudaSuccess ||
      cudaEventCreateWithFlags(&L.fin, ef) != cudaSuccess)
    return nullptr;
  for (int s = 0; s < 2; ++s)
    if (cudaEventCreateWithFlags(&L.in[s], ef) != cudaSuccess ||
        cudaEventCreateWithFlags(&L.kdone[s], ef) != cudaSuccess ||
        cudaEventCreateWithFlags(&L.out[s], ef) != cudaSuccess)
      return nullptr;
  L.ready = true;
  return &L;
}

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

// Byte offsets in the device workspace.
struct Layout {
  size_t gam = 0, bet = 0, w = 0;
  size_t q[2], k[2], v[2], eta[2], gate[2], mask[2], o[2];
  size_t total = 0;
};

// The default segment: about an eighth of the sequence (measured at workload 5
// against a sixteenth, a quarter and whole: the fastest), at least 256 tokens,
// a multiple of b and of 16 (the per-token kernels' own chunk of up to 16
// tokens then never straddles a segment boundary either).
int segment_tokens(int T, int b, int seg_tokens) {
  if (seg_tokens > 0) return seg_tokens;
  int g = 16, r = b;  // gcd(b, 16)
  while (r != 0) {
    const int t = g % r;
    g = r;
    r = t;
  }
  const long long unit = (long long)b / g * 16;
  const long long part = ((long long)T + 7) / 8;
  const long long want = part > 256 ? part : 256;
  const long long s = (want + unit - 1) / unit * unit;
  return s > 0x40000000LL ? 0x40000000 : (int)s;
}

Layout layout_for(int B, int H, int T, int d, unsigned mode, int b, int S) {
  Layout L{};
  const size_t heads = (size_t)B * H;
  const size_t seg = (size_t)(S < T ? S : T);
  const size_t ie = (mode & TTT_IN_BF16) ? 2 : 4;
  const size_t oe = (mode & TTT_OUT_BF16) ? 2 : 4;
  const bool no_ln = mode & TTT_NO_LN;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align_up(bytes);
    return at;
  };
  L.gam = take(no_ln ? 0 : (size_t)H * d * 4);
  L.bet = take(no_ln ? 0 : (size_t)H * d * 4);
  L.w = take(heads * d * d * 4);
  for (int s = 0; s < 2; ++s) {
    L.q[s] = take(heads * seg * d * ie);
    L.k[s] = take(heads * seg * d * ie);
    L.v[s] = take(heads * seg * d * ie);
    L.eta[s] = take(heads * seg * ie);
    L.gate[s] = take(heads * seg * ((mode & TTT_GATE_CHANNEL) ? d : 1) * ie);
    L.mask[s] = take((size_t)B * ((seg + b - 1) / b));
    L.o[s] = take(heads * seg * d * oe);
  }
  L.total = off;
  return L;
}

// `height` rows of `width` bytes, `src_pitch` bytes apart -> packed rows.
cudaError_t copy2d(void* dst, const void* src, size_t src_pitch, size_t width, size_t height,
                   cudaMemcpyKind kind, cudaStream_t s) {
  if (width == 0 || height == 0) return cudaSuccess;
  return cudaMemcpy2DAsync(dst, width, src, src_pitch, width, height, kind, s);
}

}  // namespace

extern "C" {

size_t ttt_scan_forward_host_workspace_bytes(int B, int H, int T, int d, unsigned mode, int b,
                                             int seg_tokens) {
  if (B < 0 || H < 0 || T < 0 || d <= 0 || b < 1 || seg_tokens < 0) return 0;
  if (seg_tokens > 0 && seg_tokens % b != 0) return 0;
  return layout_for(B, H, T, d, mode, b, segment_tokens(T, b, seg_tokens)).total;
}

int ttt_scan_forward_host(const void* q, const void* k, const void* v, const void* eta_logit,
                          const void* gate_logit, const float* W0, const float* gamma,
                          const float* beta, int B, int H, int T, int d, float eps,
                          unsigned mode, int b, const unsigned char* mask, void* o, float* W_T,
                          int seg_tokens, void* workspace, size_t workspace_bytes,
                          void* cuda_stream) {
  // ---- argument checks (nothing is enqueued on failure) ----
  if (B < 0 || H < 0 || T < 0 || b < 1 || d <= 0 || seg_tokens < 0) return TTT_ERR_INVALID_ARG;
  if (seg_tokens > 0 && seg_tokens % b != 0) return TTT_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return TTT_ERR_INVALID_ARG;
  const int choice = ttt_scan_kernel_choice(B, H, T, d, mode, b);
  if (choice < 0) return choice;
  const long long heads = (long long)B * H;
  if (heads == 0) return TTT_OK;
  const bool no_ln = mode & TTT_NO_LN;
  if (T > 0 && (!q || !k || !v || !eta_logit || !o)) return TTT_ERR_INVALID_ARG;
  if (!W0 || !W_T) return TTT_ERR_INVALID_ARG;
  if (!no_ln && (!gamma || !beta)) return TTT_ERR_INVALID_ARG;
  {
    // the host buffers: o and W_T must not overlap the inputs (W_T may be W0)
    const size_t ie = (mode & TTT_IN_BF16) ? 2 : 4, oe = (mode & TTT_OUT_BF16) ? 2 : 4;
    const size_t tok = (size_t)heads * T * d * ie, scal = (size_t)heads * T * ie;
    const size_t gate = (mode & TTT_GATE_CHANNEL) ? tok : scal;
    const size_t wb = (size_t)heads * d * d * 4, gb = no_ln ? 0 : (size_t)H * d * 4;
    const size_t ob = (size_t)heads * T * d * oe, mb = mask ? (size_t)B * ((T + b - 1) / b) : 0;
    const ttt::abi::Span ins[] = {{q, tok}, {k, tok}, {v, tok}, {eta_logit, scal},
                                  {gate_logit, gate_logit ? gate : 0}, {W0, wb}, {gamma, gb},
                                  {beta, gb}, {mask, mb}};
    for (const auto& in : ins) {
      if (ttt::abi::overlaps(o, ob, in.p, in.n)) return TTT_ERR_INVALID_ARG;
      if (in.p != W0 && ttt::abi::overlaps(W_T, wb, in.p, in.n)) return TTT_ERR_INVALID_ARG;
    }
    if (W_T != W0 && ttt::abi::overlaps(W_T, wb, W0, wb)) return TTT_ERR_INVALID_ARG;
    if (ttt::abi::overlaps(o, ob, W_T, wb)) return TTT_ERR_INVALID_ARG;
  }
  const int S = segment_tokens(T, b, seg_tokens);
  const Layout Lw = layout_for(B, H, T, d, mode, b, S);
  if (!workspace || ttt::abi::misaligned(workspace) || workspace_bytes < Lw.total)
    return TTT_ERR_INVALID_ARG;

  std::lock_guard<std::mutex> lock(g_mutex);
  Lanes* L = lanes_current_device();
  if (!L) return TTT_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  const size_t ie = (mode & TTT_IN_BF16) ? 2 : 4;
  const size_t oe = (mode & TTT_OUT_BF16) ? 2 : 4;
  const size_t w_bytes = (size_t)heads * d * d * 4;
  const size_t gate_w = (mode & TTT_GATE_CHANNEL) ? (size_t)d : 1;
  const int nch = (T + b - 1) / b;
  float* Wd = reinterpret_cast<float*>(ws + Lw.w);
  const float* gd = no_ln ? nullptr : reinterpret_cast<const float*>(ws + Lw.gam);
  const float* bd = no_ln ? nullptr : reinterpret_cast<const float*>(ws + Lw.bet);

#define TTT_TRY(x)                                       \
  do {                                                   \
    if ((x) != cudaSuccess) return TTT_ERR_CUDA;         \
  } while (0)
  // everything earlier on the caller's stream (a previous user of the
  // workspace, the producer of the host inputs) before the first copy
  TTT_TRY(cudaEventRecord(L->start, s));
  TTT_TRY(cudaStreamWaitEvent(L->copy_in, L->start, 0));
  TTT_TRY(cudaStreamWaitEvent(L->copy_out, L->start, 0));
  TTT_TRY(cudaMemcpyAsync(Wd, W0, w_bytes, cudaMemcpyHostToDevice, L->copy_in));
  if (!no_ln) {
    TTT_TRY(cudaMemcpyAsync(ws + Lw.gam, gamma, (size_t)H * d * 4, cudaMemcpyHostToDevice,
                            L->copy_in));
    TTT_TRY(cudaMemcpyAsync(ws + Lw.bet, beta, (size_t)H * d * 4, cudaMemcpyHostToDevice,
                            L->copy_in));
  }
  if (T == 0) {  // W_T = W0 through the device copy
    TTT_TRY(cudaEventRecord(L->in[0], L->copy_in));
    TTT_TRY(cudaStreamWaitEvent(L->copy_out, L->in[0], 0));
    TTT_TRY(cudaMemcpyAsync(W_T, Wd, w_bytes, cudaMemcpyDeviceToHost, L->copy_out));
    TTT_TRY(cudaEventRecord(L->fin, L->copy_out));
    TTT_TRY(cudaStreamWaitEvent(s, L->fin, 0));
    return TTT_OK;
  }

  const int nseg = (T + S - 1) / S;
  const size_t rows = (size_t)heads;
  for (int i = 0; i < nseg; ++i) {
    const int set = i & 1;
    const int t0 = i * S;
    const int n = (T - t0 < S) ? T - t0 : S;  // tokens of this segment
    const int c0 = t0 / b, nc = (n + b - 1) / b;
    unsigned char* dq = ws + Lw.q[set];
    unsigned char* dk = ws + Lw.k[set];
    unsigned char* dv = ws + Lw.v[set];
    unsigned char* de = ws + Lw.eta[set];
    unsigned char* dg = ws + Lw.gate[set];
    unsigned char* dm = ws + Lw.mask[set];
    unsigned char* dout = ws + Lw.o[set];
    // ---- copy in (set reuse: the scan of segment i-2 has read it) ----
    if (i >= 2) TTT_TRY(cudaStreamWaitEvent(L->copy_in, L->kdone[set], 0));
    const size_t tok_w = (size_t)n * d * ie, tok_p = (size_t)T * d * ie;
    const unsigned char* hq = static_cast<const unsigned char*>(q) + (size_t)t0 * d * ie;
    const unsigned char* hk = static_cast<const unsigned char*>(k) + (size_t)t0 * d * ie;
    const unsigned char* hv = static_cast<const unsigned char*>(v) + (size_t)t0 * d * ie;
    TTT_TRY(copy2d(dq, hq, tok_p, tok_w, rows, cudaMemcpyHostToDevice, L->copy_in));
    TTT_TRY(copy2d(dk, hk, tok_p, tok_w, rows, cudaMemcpyHostToDevice, L->copy_in));
    TTT_TRY(copy2d(dv, hv, tok_p, tok_w, rows, cudaMemcpyHostToDevice, L->copy_in));
    TTT_TRY(copy2d(de, static_cast<const unsigned char*>(eta_logit) + (size_t)t0 * ie,
                   (size_t)T * ie, (size_t)n * ie, rows, cudaMemcpyHostToDevice, L->copy_in));
    if (gate_logit)
      TTT_TRY(copy2d(dg, static_cast<const unsigned char*>(gate_logit) + (size_t)t0 * gate_w * ie,
                     (size_t)T * gate_w * ie, (size_t)n * gate_w * ie, rows,
                     cudaMemcpyHostToDevice, L->copy_in));
    if (mask)
      TTT_TRY(copy2d(dm, mask + c0, (size_t)nch, (size_t)nc, (size_t)B, cudaMemcpyHostToDevice,
                     L->copy_in));
    TTT_TRY(cudaEventRecord(L->in[set], L->copy_in));
    // ---- scan (o of this set: the copy-out of segment i-2 has read it) ----
    TTT_TRY(cudaStreamWaitEvent(s, L->in[set], 0));
    if (i >= 2) TTT_TRY(cudaStreamWaitEvent(s, L->out[set], 0));
    const int rc = ttt_scan_forward(dq, dk, dv, de, gate_logit ? dg : nullptr, Wd, gd, bd, B, H,
                                    n, d, eps, mode, b, mask ? dm : nullptr, dout, Wd, nullptr,
                                    cuda_stream);
    if (rc != TTT_OK) return rc;
    TTT_TRY(cudaEventRecord(L->kdone[set], s));
    // ---- copy out ----
    TTT_TRY(cudaStreamWaitEvent(L->copy_out, L->kdone[set], 0));
    const size_t o_w = (size_t)n * d * oe, o_p = (size_t)T * d * oe;
    TTT_TRY(cudaMemcpy2DAsync(static_cast<unsigned char*>(o) + (size_t)t0 * d * oe, o_p, dout,
                              o_w, o_w, rows, cudaMemcpyDeviceToHost, L->copy_out));
    TTT_TRY(cudaEventRecord(L->out[set], L->copy_out));
  }
  // W_T after the last scan (the copy-out stream waited for it above)
  TTT_TRY(cudaMemcpyAsync(W_T, Wd, w_bytes, cudaMemcpyDeviceToHost, L->copy_out));
  TTT_TRY(cudaEventRecord(L->fin, L->copy_out));
  TTT_TRY(cudaStreamWaitEvent(s, L->fin, 0));
#undef TTT_TRY
  return TTT_OK;
}

}  // extern "C"
