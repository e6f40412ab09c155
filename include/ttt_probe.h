/*
 * ttt_probe.h -- measurement helper shipped with the scan library.
 *
 * The per-token scan is bound by fp32 FMA throughput (6 d^2 flops per
 * head-token on CUDA cores); its roofline needs the FP32 peak of the device,
 * which this probe measures with a launch of independent FFMA chains.
 */
#ifndef TTT_PROBE_H
#define TTT_PROBE_H

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Enqueue one FFMA-throughput kernel on `cuda_stream`: `blocks` CTAs of
 * `threads` threads (a multiple of 32, <= 1024), each thread running 8
 * independent fused multiply-add chains for `iters` x 16 steps. `sink` is a
 * caller-owned DEVICE buffer of blocks*threads floats that receives one value
 * per thread (it keeps the work observable). On success *flops_out (host
 * pointer) holds the flop count of the launch (2 per FMA) and TTT_OK (0) is
 * returned; the caller times the launch with events on the same stream.
 * Returns -1 on an invalid argument, -3 if the launch fails.
 */
int ttt_probe_ffma(int blocks, int threads, int iters, float* sink, double* flops_out,
                   void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* TTT_PROBE_H */
