/*
 * ttt_scan.h -- C ABI of the B200 (sm_100a) TTT-Linear inner-loop scan.
 *
 * The scan is the per-(batch row, head) recurrence of "Edifice.Recurrent.TTT",
 * section "Equations (TTT-Linear)": the hidden state is a d x d fast-weight
 * matrix W (z = W k, stored row-major as W[out][in]); for every token t
 *
 *     eta_t  = sigmoid(eta_logit_t) / d
 *     pred_t = LayerNorm_{gamma,beta}(W_{t-1} k_t),   err_t = pred_t - v_t
 *     W_t    = W_{t-1} - eta_t * G_t k_t^T
 *     o_t    = (W_t q_t) * sigmoid(gate_logit_t)
 *
 * where G_t is the simplified gradient err_t (the Equations section) or the full
 * squared-error gradient through the LayerNorm Jacobian, g = gamma*err,
 * G = (g - mean(g) - xhat*mean(g*xhat)) / sqrt(var + eps) ("Error Correction in
 * Trained TTT Layers", Abstract). LayerNorm is over the d features of one head
 * with biased variance and eps inside the square root.
 *
 * Mini-batch mode is the dual form of PonderTTT ("Technical Architecture",
 * dual-form updates): in each chunk of b tokens every gradient is taken at the
 * chunk-start state W_s, o_i = sigmoid(gate_i)*(W_s q_i - sum_{j<=i} eta_j
 * (k_j.q_i) G_j) and W advances once by - sum_j eta_j G_j k_j^T. The last chunk
 * may be partial (cortex_rust src/layers/ttt.rs, forward_chunkwise).
 *
 * The optional mask holds one SKIP/UPDATE byte per chunk of b tokens and per
 * batch row (PonderTTT, "Core Idea: Binary Gating via Gumbel-Softmax"); a SKIP
 * chunk has eta = 0 for all its tokens, leaves W bit-for-bit unchanged and still
 * produces outputs. The granularity is b in both modes.
 */
#ifndef TTT_SCAN_H
#define TTT_SCAN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. Argument errors are reported before anything is launched. */
typedef enum {
  TTT_OK = 0,
  TTT_ERR_INVALID_ARG = -1,    /* null/misaligned pointer, bad size, aliasing, unknown mode bit */
  TTT_ERR_UNSUPPORTED = -2,    /* valid arguments this build does not implement (d, b, dtype mix) */
  TTT_ERR_CUDA = -3,           /* a CUDA runtime call or a launch failed */
  TTT_ERR_DEVICE_TIMEOUT = -4  /* a bounded in-kernel wait gave up; outputs are not valid */
} ttt_status;

/* Mode bit flags. */
enum {
  TTT_MODE_MINIBATCH = 1u << 0, /* dual-form chunk update; else the exact per-token recurrence */
  TTT_GRAD_LNJAC = 1u << 1,     /* gradient through the LayerNorm Jacobian; else G = err */
  TTT_NO_LN = 1u << 2,          /* no LayerNorm: pred = z, G = z - v (delta rule); gamma/beta unused */
  TTT_IN_BF16 = 1u << 3,        /* q, k, v, eta_logit, gate_logit are bf16; else fp32 */
  TTT_OUT_BF16 = 1u << 4,       /* o is bf16; else fp32 */
  TTT_KERNEL_SIMT = 1u << 5,    /* run the CUDA-core kernel even where the tensor-core kernel applies */
  TTT_GATE_CHANNEL = 1u << 6,   /* gate_logit holds one logit per feature (d per token), applied
                                   elementwise; else one per token */
  TTT_KERNEL_SINGLE_CTA = 1u << 7, /* per-token mode: keep every head on one CTA even when the
                                      heads are few enough to spread each over a cluster */
  TTT_GRAD_ABLATE = 1u << 8,      /* ablation gradient: the LayerNorm Jacobian applied to
                                     -gamma*v, i.e. the prediction's contribution removed
                                     ("Error Correction in Trained TTT Layers", Abstract);
                                     both modes; invalid with TTT_NO_LN */
  TTT_GRAD_NORM_MATCH = 1u << 9,  /* with TTT_GRAD_ABLATE: rescale each token's gradient to the
                                     L2 norm of its full LN-Jacobian gradient (0 where the
                                     ablated gradient is 0); invalid without TTT_GRAD_ABLATE */
  TTT_KQ_SILU = 1u << 10          /* the `:mlp` variant ("Edifice.Recurrent.TTT", `build`
                                     options, `:variant`): k <- SiLU(k), q <- SiLU(q)
                                     (SiLU(x) = x sigmoid(x)) before the inner model, every
                                     other step unchanged. The CUDA-core scan kernels take it
                                     with fp32 inputs only (TTT_ERR_UNSUPPORTED with bf16
                                     inputs there); the tensor-core kernel applies it to its
                                     bf16 operands; the decode step takes both dtypes */
};

/* Kernel identifiers returned by ttt_scan_kernel_choice(). */
enum {
  TTT_KERNEL_NONE = 0,                  /* nothing to launch (B*H == 0) */
  TTT_KERNEL_ID_CUDA_CORE = 1,          /* CUDA cores, one CTA per head */
  TTT_KERNEL_ID_CUDA_CORE_CLUSTER = 2,  /* CUDA cores, each head's rows of W split over a
                                           cluster of 4 CTAs (per-token, d = 64, few heads) */
  TTT_KERNEL_ID_TENSOR_CORE = 3         /* tcgen05 mini-batch kernel */
};

/*
 * Run the scan on `cuda_stream` (a cudaStream_t; 0 = legacy default stream).
 * Enqueue-only: returns once the kernel is launched. Device-side failures are
 * read with ttt_check_device_status().
 *
 * All pointers are DEVICE pointers owned by the caller, 16-byte aligned,
 * contiguous row-major (a pointer may be NULL when the tensor it names has no
 * elements, e.g. q..o when T == 0, everything when B*H == 0):
 *   q, k, v      [B, H, T, d]   fp32, or bf16 with TTT_IN_BF16
 *   eta_logit    [B, H, T]      same dtype as q
 *   gate_logit   [B, H, T], or [B, H, T, d] with TTT_GATE_CHANNEL (o[r] = sigmoid(gate[r]) *
 *                (W q)[r]); same dtype as q; NULL = no output gate (factor 1)
 *   W0           [B, H, d, d]   fp32 initial fast weights, z = W k
 *   gamma, beta  [H, d]         fp32 inner-LayerNorm affine; may be NULL with TTT_NO_LN
 *   mask         [B, ceil(T/b)] bytes, nonzero = UPDATE, 0 = SKIP; NULL = all UPDATE
 *   o            [B, H, T, d]   out: fp32, or bf16 with TTT_OUT_BF16; must not overlap any input
 *   W_T          [B, H, d, d]   out: fp32 final fast weights; may equal W0 (in place), must not
 *                               otherwise overlap it
 *   W_chunks     NULL, or out [B, H, ceil(T/b) + 1, d, d] fp32: W before every chunk of b tokens
 *                and, in the last slot, W after the last token (a debugging aid)
 * Sizes: B, H, T >= 0 (B*H == 0 launches nothing; T == 0 copies W0 to W_T),
 *   d in {16, 64}, b >= 1, eps >= 0 (finite).
 * Kernels: per-token mode runs a CUDA-core kernel for any b: at d = 64, when
 *   the B*H heads fit on the device as clusters of 4 CTAs (one per SM), each
 *   head's rows of W are split over such a cluster; otherwise (or with
 *   TTT_KERNEL_SINGLE_CTA) one CTA runs each head. Mini-batch mode runs the
 *   tcgen05 tensor-core kernel for d = 64, b = 16 with bf16 inputs (either gate
 *   form), and otherwise (or with TTT_KERNEL_SIMT) the CUDA-core kernel, which
 *   takes b <= 16. Every gradient form (TTT_GRAD_LNJAC, TTT_NO_LN,
 *   TTT_GRAD_ABLATE, TTT_GRAD_NORM_MATCH) runs in both modes on every kernel.
 *   Other combinations return TTT_ERR_UNSUPPORTED.
 * The library allocates no device memory per call.
 */
int ttt_scan_forward(const void* q, const void* k, const void* v,
                     const void* eta_logit, const void* gate_logit,
                     const float* W0, const float* gamma, const float* beta,
                     int B, int H, int T, int d, float eps, unsigned mode, int b,
                     const unsigned char* mask, void* o, float* W_T,
                     float* W_chunks, void* cuda_stream);

/*
 * ttt_scan_forward, plus the per-token inner-gradient norms of the ablation
 * study ("Error Correction in Trained TTT Layers", Abstract: the mean ratio of
 * the ablated gradient's norm to the full gradient's norm). Needs
 * TTT_GRAD_ABLATE (else TTT_ERR_INVALID_ARG), in either mode (mini-batch: both
 * norms at the chunk-start state W_s); the outputs o, W_T and W_chunks are
 * those of ttt_scan_forward with the same arguments. Per-token calls run on
 * one CTA per head.
 *   grad_norms  device, [B, H, T, 2] fp32, written: per head-token the L2 norm
 *               of the full LayerNorm-Jacobian gradient J^T(gamma*(pred - v))
 *               and of the ablated gradient J^T(-gamma*v) before any norm
 *               matching, both at the state the token's gradient is taken at
 *               (W_{t-1} per token, W_s in mini-batch mode); zeros on the
 *               tokens of SKIP chunks, which take no gradient. Must not
 *               overlap any other argument; null only when B*H*T == 0.
 * The call costs one more warp reduction per token on the gradient chain.
 */
int ttt_scan_forward_grad_norms(const void* q, const void* k, const void* v,
                                const void* eta_logit, const void* gate_logit,
                                const float* W0, const float* gamma, const float* beta,
                                int B, int H, int T, int d, float eps, unsigned mode, int b,
                                const unsigned char* mask, void* o, float* W_T,
                                float* W_chunks, float* grad_norms, void* cuda_stream);

/*
 * The kernel ttt_scan_forward would run for these sizes and mode bits on the
 * current CUDA device: one of the TTT_KERNEL_* identifiers above, or a negative
 * status (TTT_ERR_INVALID_ARG / TTT_ERR_UNSUPPORTED for arguments the scan
 * rejects). Launches nothing.
 */
int ttt_scan_kernel_choice(int B, int H, int T, int d, unsigned mode, int b);

/*
 * ttt_scan_forward with its inputs and outputs in HOST memory: the end-to-end
 * call of a caller whose tensors live on the host. No page has this call; it
 * is plumbing around the same scan. The sequence is cut into segments of
 * `seg_tokens` tokens (0: the library's choice, about an eighth of T,
 * at least 256, a multiple of b and of 16); segment i+1's inputs are copied in while
 * segment i is scanned and segment i-1's outputs are copied out, and the
 * state W passes from one segment to the next on the device, exactly. o and
 * W_T are those of ttt_scan_forward on the whole sequence up to rounding (the
 * kernels' look-ahead products restart at a segment boundary, where the first
 * chunk's z comes straight from the state), and bit for bit when one segment
 * covers the sequence.
 *
 * Arguments as for ttt_scan_forward, except:
 *   q .. mask, o, W_T   HOST pointers (page-locked memory lets the copies run
 *                       asynchronously; pageable memory works, more slowly).
 *                       W_T may equal W0. They must stay valid, and o / W_T
 *                       unread, until `cuda_stream` has completed the call.
 *   seg_tokens          0, or a positive multiple of b.
 *   workspace           DEVICE memory of at least
 *                       ttt_scan_forward_host_workspace_bytes(B, H, T, d, mode, b,
 *                       seg_tokens) bytes, 16-byte aligned, owned by the caller and
 *                       not touched by anything else until the call completes on
 *                       `cuda_stream`.
 * There is no W_chunks output. Enqueue-only: the copies run on two streams of
 * the library's own (created on first use on each device, kept until exit) and
 * the scans on `cuda_stream`, which waits for the last copy, so synchronising
 * `cuda_stream` completes the call. Calls from several host threads are
 * enqueued one at a time. Errors: TTT_ERR_INVALID_ARG for arguments the scan
 * rejects, for seg_tokens that is negative or not a multiple of b, or for a
 * workspace that is too small or misaligned (nothing is enqueued);
 * TTT_ERR_CUDA if a copy or a stream operation fails to enqueue.
 */
size_t ttt_scan_forward_host_workspace_bytes(int B, int H, int T, int d, unsigned mode, int b,
                                             int seg_tokens);
int ttt_scan_forward_host(const void* q, const void* k, const void* v,
                          const void* eta_logit, const void* gate_logit,
                          const float* W0, const float* gamma, const float* beta,
                          int B, int H, int T, int d, float eps, unsigned mode, int b,
                          const unsigned char* mask, void* o, float* W_T, int seg_tokens,
                          void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * One streaming decode step: the per-token recurrence above for a single token
 * of every (batch row, head), with the fast weights carried between calls and
 * updated IN PLACE (the state-in, state-out step of cortex_rust
 * src/layers/ttt.rs, forward_update). For each head
 *
 *     eta = sigmoid(eta_logit) / d        (0 when update[b] == 0)
 *     G   = inner gradient at z = W k     (as selected by mode)
 *     W  <- W - eta * G k^T               (W is not written at all when eta == 0)
 *     o   = (W q) * sigmoid(gate_logit)   (with the updated W)
 *
 * so a chain of T calls equals ttt_scan_forward in per-token mode over those
 * T tokens (up to fp32 rounding order). Arithmetic is fp32.
 *
 * Enqueue-only on `cuda_stream`. All pointers are DEVICE pointers owned by the
 * caller, 16-byte aligned, contiguous row-major; NULL only where the tensor
 * has no elements (B*H == 0) or where noted:
 *   q, k, v      [B, H, d]      fp32, or bf16 with TTT_IN_BF16
 *   eta_logit    [B, H]         same dtype as q
 *   gate_logit   [B, H], or [B, H, d] with TTT_GATE_CHANNEL; same dtype as q;
 *                NULL = no output gate (factor 1)
 *   W            [B, H, d, d]   fp32 fast weights (z = W k), read and overwritten
 *   gamma, beta  [H, d]         fp32 inner-LayerNorm affine; may be NULL with TTT_NO_LN
 *   update       [B] bytes, nonzero = UPDATE, 0 = SKIP (W left bit for bit); NULL = all UPDATE
 *   o            [B, H, d]      out: fp32, or bf16 with TTT_OUT_BF16
 * No output may overlap an input, and W may overlap nothing else.
 * mode: TTT_GRAD_LNJAC, TTT_NO_LN, TTT_IN_BF16, TTT_OUT_BF16, TTT_GATE_CHANNEL,
 *   TTT_GRAD_ABLATE, TTT_GRAD_NORM_MATCH, TTT_KQ_SILU (as for the scan).
 *   TTT_MODE_MINIBATCH returns TTT_ERR_UNSUPPORTED (a one-token step has no
 *   chunk); TTT_KERNEL_SIMT and TTT_KERNEL_SINGLE_CTA are accepted and ignored.
 * Sizes: B, H >= 0, d in {16, 64}, eps >= 0 (finite). Returns TTT_OK or an error
 * code before launching anything. Allocates no device memory.
 */
int ttt_decode_step(const void* q, const void* k, const void* v,
                    const void* eta_logit, const void* gate_logit, float* W,
                    const float* gamma, const float* beta, int B, int H, int d,
                    float eps, unsigned mode, const unsigned char* update, void* o,
                    void* cuda_stream);

/*
 * Backward of the scan: the gradients of L = <dO, o> + <dW_T, W_T> with respect
 * to every input of a ttt_scan_forward call with the same arguments, by the
 * chain rule taken through the forward's steps in reverse (no page gives this
 * pass; it is the reverse of the recurrence in the comment at the top of this
 * file, for the training both "Edifice.Recurrent.TTT" (Architecture) and
 * PonderTTT (Technical Architecture) do). Per-token and mini-batch mode, the
 * SIMPLE, LN-Jacobian, no-LayerNorm and ablation gradients, scalar, per-feature
 * or no gate, the mask and the SiLU variant. Arithmetic is fp32.
 *
 * Enqueue-only on `cuda_stream`. All pointers are DEVICE pointers owned by the
 * caller, 16-byte aligned, contiguous row-major:
 *   q, k, v, eta_logit, gate_logit, gamma, beta, mask   as for ttt_scan_forward
 *   W_chunks     [B, H, ceil(T/b) + 1, d, d] fp32: the W_chunks snapshots written by
 *                ttt_scan_forward with the same arguments (the state before every chunk
 *                of b tokens; the backward recomputes each chunk from its snapshot)
 *   dO           [B, H, T, d] fp32, dL/do
 *   dW_T         [B, H, d, d] fp32, dL/dW_T; NULL = zero
 *   dq, dk, dv   [B, H, T, d] fp32 out
 *   d_eta_logit  [B, H, T] fp32 out (0 on SKIP chunks)
 *   d_gate_logit fp32 out, the shape of gate_logit; NULL only when gate_logit is NULL
 *   dW0          [B, H, d, d] fp32 out
 *   dgamma, dbeta [H, d] fp32 out, summed over the batch rows (in batch-row order, so
 *                the result is deterministic); unused (may be NULL) with TTT_NO_LN
 *   workspace    device scratch of at least ttt_scan_backward_workspace_bytes(B, H, d,
 *                mode) bytes (per-head partial sums of dgamma, dbeta); NULL when that
 *                is 0. Owned by the caller; calls that share one must not overlap.
 * No output may overlap an input, another output or the workspace.
 * Sizes: as for ttt_scan_forward, with b <= 16 (the chunk the backward recomputes
 *   from one snapshot) and d in {16, 64}. mode: the forward's bits; TTT_OUT_BF16,
 *   TTT_KERNEL_SIMT and TTT_KERNEL_SINGLE_CTA are ignored, TTT_GRAD_NORM_MATCH returns
 *   TTT_ERR_UNSUPPORTED. Returns TTT_OK or an error code before launching anything.
 * Allocates no device memory.
 */
size_t ttt_scan_backward_workspace_bytes(int B, int H, int d, unsigned mode);

int ttt_scan_backward(const void* q, const void* k, const void* v,
                      const void* eta_logit, const void* gate_logit,
                      const float* gamma, const float* beta,
                      int B, int H, int T, int d, float eps, unsigned mode, int b,
                      const unsigned char* mask, const float* W_chunks,
                      const float* dO, const float* dW_T,
                      float* dq, float* dk, float* dv, float* d_eta_logit,
                      float* d_gate_logit, float* dW0, float* dgamma, float* dbeta,
                      void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * ttt_scan_backward for callers that cannot allocate device memory. (The
 * pages have no counterpart; this is an interface of this library.) Some
 * callers cannot call cudaMalloc: code that runs inside a framework whose
 * allocator owns all of the device's memory, or a loop that cannot afford the
 * implicit device synchronisation of cudaMalloc. This entry point takes the
 * arguments of ttt_scan_backward without the workspace: the per-head
 * dgamma / dbeta partial sums live in a fixed array of 2^20 floats (4 MiB) of
 * device memory that the library defines, which every GPU that loads the
 * library holds until the process exits. It allocates nothing and calls no
 * allocating routine.
 *   - Limit: B * H * 2 * d <= 2^20 (8192 heads at d = 64, 32768 at d = 16);
 *     larger problems return TTT_ERR_UNSUPPORTED before anything is launched.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture.
 *   - Every call on a device shares the one array and leaves its partial sums
 *     there; nothing in it needs to start at zero (each call writes every
 *     partial sum it reads). Calls whose kernels overlap on the GPU (on
 *     different streams, with no ordering between them) race on the array;
 *     order them on one stream.
 * Everything else, including the results, is as for ttt_scan_backward.
 */
int ttt_scan_backward_noalloc(const void* q, const void* k, const void* v,
                              const void* eta_logit, const void* gate_logit,
                              const float* gamma, const float* beta,
                              int B, int H, int T, int d, float eps, unsigned mode, int b,
                              const unsigned char* mask, const float* W_chunks,
                              const float* dO, const float* dW_T,
                              float* dq, float* dk, float* dv, float* d_eta_logit,
                              float* d_gate_logit, float* dW0, float* dgamma, float* dbeta,
                              void* cuda_stream);

/*
 * Synchronise `cuda_stream`, then report and clear the device status word that
 * the kernels set when a bounded wait gives up. Returns TTT_OK,
 * TTT_ERR_DEVICE_TIMEOUT, or TTT_ERR_CUDA (a sticky or asynchronous CUDA error).
 */
int ttt_check_device_status(void* cuda_stream);

/* Static, human-readable name of a status code (never NULL). */
const char* ttt_status_string(int status);

/*
 * Upper bound on the number of polls of each bounded in-kernel wait, for all
 * later launches of this process (default 2^20). A value of 0 makes every such wait give up at
 * once, which exercises the timeout path without hanging; waits that only
 * drain work already in flight keep their own bound. Returns TTT_OK or
 * TTT_ERR_CUDA.
 */
int ttt_set_wait_limit(long long polls);

#ifdef __cplusplus
}
#endif

#endif /* TTT_SCAN_H */
