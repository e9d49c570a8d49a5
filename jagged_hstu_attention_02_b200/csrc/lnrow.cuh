// lnrow.cuh -- LayerNorm over the H*d_v features of one token and U gating, one warp per
// token, for rows whose width is a multiple of 128 ("HSTU tensor by tensor: SiLU
// aggregation, temporal bias and gating", "Trace four projections": O = U * LayerNorm(Y),
// biased variance, eps inside the square root, no affine), kept in registers.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace hstu {

template <typename T> struct Vec4;
template <> struct Vec4<float> {
    using type = float4;
    static __device__ __forceinline__ void unpack(const float4 &v, float (&f)[4])
    {
        f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    }
    static __device__ __forceinline__ float4 pack(const float (&f)[4])
    {
        return make_float4(f[0], f[1], f[2], f[3]);
    }
};
template <> struct Vec4<__nv_bfloat16> {
    using type = uint2;
    static __device__ __forceinline__ void unpack(const uint2 &v, float (&f)[4])
    {
        f[0] = __uint_as_float(v.x << 16);
        f[1] = __uint_as_float(v.x & 0xFFFF0000u);
        f[2] = __uint_as_float(v.y << 16);
        f[3] = __uint_as_float(v.y & 0xFFFF0000u);
    }
    static __device__ __forceinline__ uint2 pack(const float (&f)[4])
    {
        const __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]);
        const __nv_bfloat162 b = __floats2bfloat162_rn(f[2], f[3]);
        return make_uint2(*reinterpret_cast<const uint32_t *>(&a),
                          *reinterpret_cast<const uint32_t *>(&b));
    }
};

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One token row of width 128 * nv, held in registers: lane l holds elements 128 c + 4 l .. +3.
// out = u * (y - mean) * rstd; returns mean and rstd (the same for every lane).
template <typename T, int NV>
__device__ __forceinline__ void ln_gate_regs(float (&v)[NV][4], const float (&uu)[NV][4],
                                            float eps, typename Vec4<T>::type *orow,
                                            float *mean_o, float *rstd_o)
{
    constexpr int D = 128 * NV;
    float sum = 0.f;
#pragma unroll
    for (int c = 0; c < NV; ++c) sum += (v[c][0] + v[c][1]) + (v[c][2] + v[c][3]);
    const float mu = warp_sum(sum) * (1.0f / D);
    float sq = 0.f;
#pragma unroll
    for (int c = 0; c < NV; ++c)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[c][e] -= mu;
            sq = fmaf(v[c][e], v[c][e], sq);
        }
    const float rs = rsqrtf(warp_sum(sq) * (1.0f / D) + eps);
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        float o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] = uu[c][e] * (v[c][e] * rs);
        orow[32 * c] = Vec4<T>::pack(o);
    }
    *mean_o = mu;
    *rstd_o = rs;
}

}  // namespace hstu
