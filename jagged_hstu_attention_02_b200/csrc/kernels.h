// kernels.h -- launchers of the device kernels (host-callable, C++ linkage, internal).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace hstu {

template <typename T>
cudaError_t launch_simt_fwd(const DevParams &p, const void *q, const void *k, const void *v,
                            float *y, cudaStream_t st);
template <typename T>
cudaError_t launch_ln_gate(const DevParams &p, const float *y, const void *u, void *out,
                           float *mean, float *rstd, cudaStream_t st);
template <typename T>
cudaError_t launch_ln_gate_bwd(const DevParams &p, const void *dout, const void *u,
                               const float *y, const float *mean, const float *rstd, void *du,
                               float *dy, cudaStream_t st);
template <typename T>
cudaError_t launch_simt_bwd(const DevParams &p, const void *q, const void *k, const void *v,
                            const float *dy, float *dq_acc, void *dk, void *dv, float *d_rel,
                            float *d_tb, cudaStream_t st);
template <typename T>
cudaError_t launch_convert(const float *src, void *dst, int64_t n, cudaStream_t st);

// tcgen05 forward attention (bf16): Y = (1/N) sum_j A_ij V_j in fp32.
bool tc_fwd_supported(int dqk, int dv, int64_t T);
cudaError_t launch_tc_fwd(const DevParams &p, const void *q, const void *k, const void *v,
                          float *y, cudaStream_t st);

cudaError_t launch_debug_mask(const DevParams &p, int seq, int seq_len, uint32_t *bits,
                              cudaStream_t st);

}  // namespace hstu
