// kernels.h -- launchers of the device kernels (host-callable, C++ linkage, internal).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace hstu {

// Launches kern with programmatic stream serialisation: it may start while the kernel ahead
// of it on the stream finishes, and must call grid_dep_wait() before it touches anything that
// kernel writes or reads.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

template <typename T>
cudaError_t launch_simt_fwd(const DevParams &p, const void *q, const void *k, const void *v,
                            float *y, cudaStream_t st);
template <typename T>
cudaError_t launch_ln_gate(const DevParams &p, const float *y, const void *u, void *out,
                           float *mean, float *rstd, cudaStream_t st);
// Buffers the LayerNorm backward zeroes on the way, so that the attention backward that
// follows on the stream needs no separate memset launches: row_floats floats per token at
// rows (the dQ accumulator), and the two table-gradient arrays (by block 0).
struct BwdZero {
    float *rows;
    int64_t row_floats;
    float *a, *b;
    int na, nb;
};

__device__ __forceinline__ void bwd_zero_row(const BwdZero &z, int64_t row, int lane)
{
    if (z.rows) {
        float *r = z.rows + row * z.row_floats;
        if ((z.row_floats & 3) == 0) {
            float4 *r4 = reinterpret_cast<float4 *>(r);
            for (int64_t x = lane; x < z.row_floats / 4; x += 32) r4[x] = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
            for (int64_t x = lane; x < z.row_floats; x += 32) r[x] = 0.f;
        }
    }
}

__device__ __forceinline__ void bwd_zero_small(const BwdZero &z)
{
    if (blockIdx.x != 0) return;
    for (int x = threadIdx.x; x < z.na; x += blockDim.x) z.a[x] = 0.f;
    for (int x = threadIdx.x; x < z.nb; x += blockDim.x) z.b[x] = 0.f;
}

// dy receives fp32 values (dy_bf16 false) or bf16 hi parts at dy and lo parts at dy + T*D
// (dy_bf16 true).
template <typename T>
cudaError_t launch_ln_gate_bwd(const DevParams &p, const void *dout, const void *u,
                               const float *y, const float *mean, const float *rstd, void *du,
                               void *dy, bool dy_bf16, const BwdZero &zero, cudaStream_t st);
// Vectorised LayerNorm + gating (norm.cu) for rows of 128*k features (k <= 8 or 16).
bool ln_vec_supported(int D);
template <typename T>
cudaError_t launch_ln_gate_vec(const DevParams &p, const float *y, const void *u, void *out,
                               float *mean, float *rstd, cudaStream_t st);
template <typename T>
cudaError_t launch_ln_gate_bwd_vec(const DevParams &p, const void *dout, const void *u,
                                   const float *y, const float *mean, const float *rstd,
                                   void *du, void *dy, bool dy_bf16, const BwdZero &zero,
                                   cudaStream_t st);
template <typename T>
cudaError_t launch_simt_bwd(const DevParams &p, const void *q, const void *k, const void *v,
                            const float *dy, float *dq_acc, void *dk, void *dv, float *d_rel,
                            float *d_tb, cudaStream_t st);
template <typename T>
cudaError_t launch_convert(const float *src, void *dst, int64_t n, cudaStream_t st);

// tcgen05 forward attention (bf16): Y = (1/N) sum_j A_ij V_j in fp32.  `training` selects
// the variant whose Y carries ~16 significant bits (A split into bf16 hi + lo parts).
bool tc_fwd_supported(int dqk, int dv, int64_t T);
// unit_ctr: work-unit counter in device memory, zero at launch.
cudaError_t launch_tc_fwd(const DevParams &p, const void *q, const void *k, const void *v,
                          float *y, unsigned long long *unit_ctr, bool training,
                          cudaStream_t st);

// Multiprocessors of the current device (cached after the first query).
int num_sms();

// tcgen05 backward attention (bf16): dQ added into an fp32 accumulator (zeroed by the
// caller), dK/dV written, table gradients added into d_rel/d_tb (zeroed by the caller).
// tb_slots is scratch of kBwdMaxCtas * kMaxTimeBuckets floats (no initial contents).
constexpr int kBwdMaxCtas = 1024;
bool tc_bwd_supported(int dqk, int dv, int64_t T);
cudaError_t launch_tc_bwd(const DevParams &p, const void *q, const void *k, const void *v,
                          const void *dy_bf16 /* hi, then lo at + T*D */, float *dq_acc,
                          void *dk, void *dv, float *d_rel, float *d_tb, float *tb_slots,
                          unsigned long long *unit_ctr /* zeroed */, cudaStream_t st);

// [T, H, d] bf16 row-major as a 3-D TMA tensor (d, H, T): box 64 x 1 x 128, 128-byte swizzle.
bool encode_tmap_bf16(CUtensorMap *m, const void *base, int d, int H, int64_t T);

cudaError_t launch_debug_mask(const DevParams &p, int seq, int seq_len, uint32_t *bits,
                              cudaStream_t st);

// The layer around the attention (gemm.cu): C = A B (+ bias, SiLU, residual), bf16, with the
// columns [seg_lo[s], seg_lo[s+1]) of C written to outs[s]; and the input LayerNorm.
cudaError_t launch_gemm(const void *A, const void *B, int M, int N, int K, const float *bias,
                        bool silu, const void *resid, int nseg, const int *seg_lo,
                        void *const *outs, int32_t *status, long long wait_limit,
                        cudaStream_t st);
cudaError_t launch_ln_rows(const void *x, void *y, int64_t rows, int width, float eps,
                           cudaStream_t st);

// Jagged operations (jagged.cu).  p carries B, T, offsets, counts and the status word.
constexpr int kMaxConcatParts = 16;
cudaError_t launch_stochastic_length(const DevParams &p, const float *keys, int budget,
                                     int64_t *out_rows, int64_t *out_offsets, cudaStream_t st);
cudaError_t launch_gather_rows(const void *src, int64_t row_bytes, const int64_t *rows,
                               const int64_t *n_rows, int64_t max_rows, void *dst,
                               cudaStream_t st);
cudaError_t launch_jagged_concat(int n_parts, const void *const *values,
                                 const int64_t *const *offsets, int B, int64_t row_bytes,
                                 void *out, int64_t *out_offsets, cudaStream_t st);
// Mask of rows [row0, row0 + nrows) x keys [0, nkeys) (nkeys a multiple of 32) of sequence
// seq as the tensor-core forward (kernel 0) or backward (kernel 1) decides it.
cudaError_t launch_debug_kernel_mask(const DevParams &p, int seq, int kernel, int row0,
                                     int nrows, int nkeys, uint32_t *bits, cudaStream_t st);

}  // namespace hstu
