// norm.cu -- LayerNorm over the H*d_v features of a token and U gating, forward and backward,
// for rows whose width is a multiple of 128: one warp per token, 16-byte loads of the fp32
// attention output and 8-byte loads of the bf16 (or 16-byte fp32) gate and gradients, so a
// warp instruction moves whole 128-byte lines.  "HSTU tensor by tensor: SiLU aggregation,
// temporal bias and gating", "Trace four projections": O = U * LayerNorm(Y), biased
// variance, eps inside the square root, no affine.  Other widths use the general kernels
// in simt.cu.
#include "kernels.h"
#include "lnrow.cuh"

namespace hstu {

namespace {

constexpr int kRows = 8;                  // tokens (warps) per 256-thread block

// Forward: out = u * (y - mean) * rstd.  Lane l holds elements 128 c + 4 l .. +3.
template <typename T, int NV>
__global__ void __launch_bounds__(32 * kRows)
    ln_gate_vec_kernel(const __grid_constant__ DevParams p, const float *__restrict__ y,
                       const T *__restrict__ u, T *__restrict__ out, float *__restrict__ mean_out,
                       float *__restrict__ rstd_out)
{
    using V = Vec4<T>;
    grid_dep_wait();   // y comes from the attention kernel ahead on the stream
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kRows + (threadIdx.x >> 5);
    if (row >= p.T) return;
    constexpr int D = 128 * NV;
    const float4 *yr = reinterpret_cast<const float4 *>(y + row * D) + lane;
    const typename V::type *ur = reinterpret_cast<const typename V::type *>(u + row * D) + lane;
    float v[NV][4];
    float uu[NV][4];
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        const float4 t = __ldg(yr + 32 * c);
        v[c][0] = t.x; v[c][1] = t.y; v[c][2] = t.z; v[c][3] = t.w;
        V::unpack(ur[32 * c], uu[c]);
    }
    typename V::type *orow = reinterpret_cast<typename V::type *>(out + row * D) + lane;
    float mu, rs;
    ln_gate_regs<T, NV>(v, uu, p.eps, orow, &mu, &rs);
    if (lane == 0 && mean_out) {
        mean_out[row] = mu;
        rstd_out[row] = rs;
    }
}

// Backward of out = u * z, z = (y - mean) * rstd:
//   du = dout * z;  dz = dout * u;  dy = rstd * (dz - mean(dz) - z * mean(dz * z)).
// dy is written in fp32, or (DYT = bf16) as a hi part at dy and a lo part at dy + T*D.
template <typename T, typename DYT, int NV>
__global__ void __launch_bounds__(32 * kRows)
    ln_gate_bwd_vec_kernel(const __grid_constant__ DevParams p, const T *__restrict__ dout,
                           const T *__restrict__ u, const float *__restrict__ y,
                           const float *__restrict__ mean, const float *__restrict__ rstd,
                           T *__restrict__ du, DYT *__restrict__ dy, const BwdZero zj)
{
    using V = Vec4<T>;
    grid_dep_release();   // the attention backward may start its set-up
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kRows + (threadIdx.x >> 5);
    bwd_zero_small(zj);
    if (row >= p.T) return;
    bwd_zero_row(zj, row, lane);
    constexpr int D = 128 * NV;
    const float mu = mean[row], rs = rstd[row];
    const float4 *yr = reinterpret_cast<const float4 *>(y + row * D) + lane;
    const typename V::type *gr = reinterpret_cast<const typename V::type *>(dout + row * D) + lane;
    const typename V::type *ur = reinterpret_cast<const typename V::type *>(u + row * D) + lane;
    typename V::type *dur = reinterpret_cast<typename V::type *>(du + row * D) + lane;
    float z[NV][4], dz[NV][4];
    float m1 = 0.f, m2 = 0.f;
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        const float4 t = __ldg(yr + 32 * c);
        float g[4], uu[4], o[4];
        V::unpack(gr[32 * c], g);
        V::unpack(ur[32 * c], uu);
        z[c][0] = (t.x - mu) * rs;
        z[c][1] = (t.y - mu) * rs;
        z[c][2] = (t.z - mu) * rs;
        z[c][3] = (t.w - mu) * rs;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            dz[c][e] = g[e] * uu[e];
            o[e] = g[e] * z[c][e];
            m1 += dz[c][e];
            m2 = fmaf(dz[c][e], z[c][e], m2);
        }
        dur[32 * c] = V::pack(o);
    }
    m1 = warp_sum(m1) * (1.0f / D);
    m2 = warp_sum(m2) * (1.0f / D);
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        float gy[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) gy[e] = rs * (dz[c][e] - m1 - z[c][e] * m2);
        if constexpr (sizeof(DYT) == 4) {
            reinterpret_cast<float4 *>(dy + row * D)[lane + 32 * c] = make_float4(gy[0], gy[1], gy[2], gy[3]);
        } else {
            float lo[4];
            const uint2 hi = Vec4<__nv_bfloat16>::pack(gy);
            float hf[4];
            Vec4<__nv_bfloat16>::unpack(hi, hf);
#pragma unroll
            for (int e = 0; e < 4; ++e) lo[e] = gy[e] - hf[e];
            reinterpret_cast<uint2 *>(dy + row * D)[lane + 32 * c] = hi;
            reinterpret_cast<uint2 *>(dy + p.T * D + row * D)[lane + 32 * c] =
                Vec4<__nv_bfloat16>::pack(lo);
        }
    }
}

template <typename T, int NV>
cudaError_t fwd_nv(const DevParams &p, const float *y, const void *u, void *out, float *mean,
                   float *rstd, cudaStream_t st)
{
    const int64_t blocks = (p.T + kRows - 1) / kRows;
    return launch_pdl(ln_gate_vec_kernel<T, NV>, dim3((unsigned)blocks), dim3(32 * kRows), 0, st,
                      p, y, (const T *)u, (T *)out, mean, rstd);
}

template <typename T, int NV>
cudaError_t bwd_nv(const DevParams &p, const void *dout, const void *u, const float *y,
                   const float *mean, const float *rstd, void *du, void *dy, bool dy_bf16,
                   const BwdZero &zero, cudaStream_t st)
{
    const int64_t blocks = (p.T + kRows - 1) / kRows;
    if (dy_bf16)
        ln_gate_bwd_vec_kernel<T, __nv_bfloat16, NV><<<(unsigned)blocks, 32 * kRows, 0, st>>>(
            p, (const T *)dout, (const T *)u, y, mean, rstd, (T *)du, (__nv_bfloat16 *)dy, zero);
    else
        ln_gate_bwd_vec_kernel<T, float, NV><<<(unsigned)blocks, 32 * kRows, 0, st>>>(
            p, (const T *)dout, (const T *)u, y, mean, rstd, (T *)du, (float *)dy, zero);
    return cudaGetLastError();
}

}  // namespace

bool ln_vec_supported(int D) { return D % 128 == 0 && (D / 128 <= 8 || D / 128 == 16); }

template <typename T>
cudaError_t launch_ln_gate_vec(const DevParams &p, const float *y, const void *u, void *out,
                               float *mean, float *rstd, cudaStream_t st)
{
    switch (p.D / 128) {
    case 1: return fwd_nv<T, 1>(p, y, u, out, mean, rstd, st);
    case 2: return fwd_nv<T, 2>(p, y, u, out, mean, rstd, st);
    case 3: return fwd_nv<T, 3>(p, y, u, out, mean, rstd, st);
    case 4: return fwd_nv<T, 4>(p, y, u, out, mean, rstd, st);
    case 5: return fwd_nv<T, 5>(p, y, u, out, mean, rstd, st);
    case 6: return fwd_nv<T, 6>(p, y, u, out, mean, rstd, st);
    case 7: return fwd_nv<T, 7>(p, y, u, out, mean, rstd, st);
    case 8: return fwd_nv<T, 8>(p, y, u, out, mean, rstd, st);
    case 16: return fwd_nv<T, 16>(p, y, u, out, mean, rstd, st);
    default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_ln_gate_bwd_vec(const DevParams &p, const void *dout, const void *u,
                                   const float *y, const float *mean, const float *rstd,
                                   void *du, void *dy, bool dy_bf16, const BwdZero &zero,
                                   cudaStream_t st)
{
    switch (p.D / 128) {
    case 1: return bwd_nv<T, 1>(p, dout, u, y, mean, rstd, du, dy, dy_bf16, zero, st);
    case 2: return bwd_nv<T, 2>(p, dout, u, y, mean, rstd, du, dy, dy_bf16, zero, st);
    case 3: return bwd_nv<T, 3>(p, dout, u, y, mean, rstd, du, dy, dy_bf16, zero, st);
    case 4: return bwd_nv<T, 4>(p, dout, u, y, mean, rstd, du, dy, dy_bf16, zero, st);
    case 5: return bwd_nv<T, 5>(p, dout, u, y, mean, rstd, du, dy, dy_bf16, zero, st);
    case 6: return bwd_nv<T, 6>(p, dout, u, y, mean, rstd, du, dy, dy_bf16, zero, st);
    case 7: return bwd_nv<T, 7>(p, dout, u, y, mean, rstd, du, dy, dy_bf16, zero, st);
    case 8: return bwd_nv<T, 8>(p, dout, u, y, mean, rstd, du, dy, dy_bf16, zero, st);
    case 16: return bwd_nv<T, 16>(p, dout, u, y, mean, rstd, du, dy, dy_bf16, zero, st);
    default: return cudaErrorInvalidValue;
    }
}

template cudaError_t launch_ln_gate_vec<float>(const DevParams &, const float *, const void *,
                                               void *, float *, float *, cudaStream_t);
template cudaError_t launch_ln_gate_vec<__nv_bfloat16>(const DevParams &, const float *,
                                                       const void *, void *, float *, float *,
                                                       cudaStream_t);
template cudaError_t launch_ln_gate_bwd_vec<float>(const DevParams &, const void *,
                                                   const void *, const float *, const float *,
                                                   const float *, void *, void *, bool,
                                                   const BwdZero &, cudaStream_t);
template cudaError_t launch_ln_gate_bwd_vec<__nv_bfloat16>(const DevParams &, const void *,
                                                           const void *, const float *,
                                                           const float *, const float *,
                                                           void *, void *, bool,
                                                           const BwdZero &, cudaStream_t);

}  // namespace hstu
