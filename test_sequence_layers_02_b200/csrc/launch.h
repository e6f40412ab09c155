// Host-side launchers of the CUDA-core kernels, each compiled in its own
// translation unit (four objects of simt.cu, cluster.cu, tc_many.cu) so the library
// builds in parallel. Arguments are already checked by the C-ABI entry points;
// every function returns a ttt_status code.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace ttt {

// SMs of the current device (0 if the query fails); cached per device.
int device_sm_count();

// One CTA per head, by input dtype and mode (output dtype, gradient form and d
// from the arguments).
int launch_simt_f32_pertoken(const ScanParams& p, unsigned mode, int d, cudaStream_t stream);
int launch_simt_f32_minibatch(const ScanParams& p, unsigned mode, int d, cudaStream_t stream);
int launch_simt_bf16_pertoken(const ScanParams& p, unsigned mode, int d, cudaStream_t stream);
int launch_simt_bf16_minibatch(const ScanParams& p, unsigned mode, int d, cudaStream_t stream);

// Per-token d = 64, each head over a cluster of CTAs. gm: 0 simplified,
// 1 LN-Jacobian, 2 no LayerNorm gradient, 3 ablation, 4 ablation with
// per-token norm matching.
int launch_cluster(const ScanParams& p, unsigned mode, int gm, cudaStream_t stream);
// Clusters of that kernel that fit on the current device at once (0 if unknown).
int cluster_capacity(unsigned mode, int gm);
// Read and clear that kernel's device status word: 0 clean, > 0 a bounded wait
// gave up, < 0 the copy failed.
int cluster_status_take();

// Mini-batch d = 64 on the tensor cores, the build for three CTAs per SM
// (scan_tc_many.cuh); q, k, v, o are the tensor maps of the three inputs and
// of the output. gm as for launch_cluster.
int launch_tc_many(const ScanParams& p, const CUtensorMap* q, const CUtensorMap* k,
                   const CUtensorMap* v, const CUtensorMap* o, bool out_bf16, int gm,
                   cudaStream_t stream);
// Read and clear that kernel's device status word (as cluster_status_take).
int tc_many_status_take();

}  // namespace ttt
