// gemm.cu -- the dense steps of the HSTU layer around the attention, for B200 (sm_100a):
//   - the fused U/V/Q/K projection: one GEMM of the normalised tokens with the concatenated
//     weights, bias (and optionally SiLU) in the epilogue, which writes the four branches to
//     their own tensors ("HSTU tensor by tensor: SiLU aggregation, temporal bias and gating",
//     "Trace four projections": one larger projection, split to match the weight layout);
//   - the output projection W_o with bias and the residual added in the epilogue (same page,
//     "Similar shape, different aggregation": o_i = W_o[U_i (.) Norm(...)] + x_i);
//   - the LayerNorm of the input tokens (no affine) that precedes the projection.
//
// GEMM: C[M, N] = A[M, K] B[K, N], bf16 operands (A row-major: K-major; B row-major: N-major),
// fp32 accumulation in TMEM.  Persistent CTAs take 128 x BN output tiles (BN = 128) in a
// static order; warp 0 lane 0 streams 64-wide K slices of A and B through a four-stage ring
// with TMA (128-byte swizzle), warp 1 lane 0 issues tcgen05.mma into one of two TMEM
// accumulators, warps 2-9 read the other accumulator back (two warps per TMEM lane quarter,
// each half of the columns; thread = row = TMEM lane) and write bf16 outputs, so a tile's
// epilogue overlaps the next tile's MMAs.  Every wait is bounded.
#include <cudaTypedefs.h>

#include <cstring>

#include "kernels.h"
#include "sm100.cuh"
#include "units.cuh"

namespace hstu {

using namespace sm100;

namespace {

constexpr int GBM = 128;          // rows (tokens) per tile
constexpr int GBK = 64;           // K per stage: one 128-byte swizzle atom of bf16
constexpr int kGStages = 4;
constexpr int kGEpiWarps = 8;
constexpr int kGThreads = 32 * (2 + kGEpiWarps);   // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
                                                   // (warp 2 also owns TMEM)
constexpr int kMaxSegs = 4;

struct GemmArgs {
    CUtensorMap ta, tb;               // A (K, M) and B (N, K) as TMA tensors
    int M, N, K;
    const float *bias;                // [N] or null
    int silu;                         // apply x * sigmoid(x) after the bias
    const __nv_bfloat16 *resid;       // [M, N] added last, or null
    int nseg;                         // output segments: columns [lo[s], lo[s+1]) of C go to
    int lo[kMaxSegs + 1];             // out[s] (row stride lo[s+1] - lo[s])
    __nv_bfloat16 *out[kMaxSegs];
    int32_t *status;
    long long wait_limit;
};

template <int BN>
struct GLayout {
    static constexpr int AB = GBM * GBK * 2;      // 16 KB
    static constexpr int BB = GBK * BN * 2;       // BN/64 boxes of 64 x 64 (8 KB each)
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = kGStages * AB;
    static constexpr int BAR_OFF = B_OFF + kGStages * BB;
    static constexpr int TOTAL = BAR_OFF + 256;
    static constexpr int ALLOC = TOTAL + 1024;
};

enum GBar { G_FULL = 0, G_EMPTY = 4, ACC_FULL = 8, ACC_EMPTY = 10, G_DONE = 12, G_NBARS = 13 };

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void gemm_flag(const GemmArgs &a)
{
    if (a.status) atomicOr(a.status, HSTU_DEV_WAIT_TIMEOUT);
}

template <int BN>
__global__ void __launch_bounds__(kGThreads, 1) gemm_tc_kernel(const __grid_constant__ GemmArgs a)
{
    using L = GLayout<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR_OFF);
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::BAR_OFF + 8 * 16);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int x = 0; x < G_NBARS; ++x) mbar_init(&bars[x], 1);
        mbar_init(&bars[ACC_EMPTY], kGEpiWarps);
        mbar_init(&bars[ACC_EMPTY + 1], kGEpiWarps);
        fence_mbar_init();
    }
    if (warp == 2) tmem_alloc(slot, 2 * BN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    const uint32_t sm_base = smem_u32(sm);
    const int mt = (a.M + GBM - 1) / GBM, nt = (a.N + BN - 1) / BN;
    const int ntiles = mt * nt, kch = (a.K + GBK - 1) / GBK;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- TMA producer
            prefetch_tmap(&a.ta);
            prefetch_tmap(&a.tb);
            int g = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
                const int m0 = (tile / nt) * GBM, n0 = (tile % nt) * BN;
                for (int kc = 0; kc < kch; ++kc, ++g) {
                    const int s = g % kGStages;
                    if (g >= kGStages &&
                        !mbar_wait(&bars[G_EMPTY + s], ((g / kGStages) - 1) & 1, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars[G_FULL + s], L::AB + L::BB);
                    tma_load_2d(sm + L::A_OFF + s * L::AB, &a.ta, &bars[G_FULL + s], kc * GBK, m0);
                    for (int nb = 0; nb < BN / 64; ++nb)
                        tma_load_2d(sm + L::B_OFF + s * L::BB + nb * (64 * GBK * 2), &a.tb,
                                    &bars[G_FULL + s], n0 + nb * 64, kc * GBK);
                }
            }
            if (!ok) gemm_flag(a);
            // every copy issued has landed before the block may exit
            bool drained = true;
            for (int x = g - 1; x >= 0 && x >= g - kGStages; --x)
                drained &= mbar_wait(&bars[G_FULL + x % kGStages], (x / kGStages) & 1,
                                     kWaitLimitCycles);
            if (!drained) gemm_flag(a);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            constexpr uint32_t idesc = idesc_bf16(GBM, BN, false, true);
            int g = 0, t = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++t) {
                const int acc = t & 1;
                if (t >= 2 && !mbar_wait(&bars[ACC_EMPTY + acc], ((t >> 1) - 1) & 1, a.wait_limit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + acc * BN;
                for (int kc = 0; kc < kch; ++kc, ++g) {
                    const int s = g % kGStages;
                    if (!mbar_wait(&bars[G_FULL + s], (g / kGStages) & 1, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t aa = sm_base + L::A_OFF + s * L::AB;
                    const uint32_t bb = sm_base + L::B_OFF + s * L::BB;
#pragma unroll
                    for (int kk = 0; kk < GBK / 16; ++kk) {
                        // A: K-major rows of 128 bytes; B: N-major, 64-column blocks at 8 KB,
                        // 8-row K groups at 1 KB; 16 K rows per step
                        const uint64_t ad = sw128_desc(aa + kk * 32, 16, 1024);
                        const uint64_t bd = sw128_desc(bb + kk * 2048, 64 * GBK * 2, 1024);
                        umma_bf16_ss(d, ad, bd, idesc, (kc | kk) ? 1u : 0u);
                    }
                    umma_commit(&bars[G_EMPTY + s]);
                }
                if (!ok) break;
                umma_commit(&bars[ACC_FULL + acc]);
            }
            if (!ok) gemm_flag(a);
            umma_commit(&bars[G_DONE]);
            if (!mbar_wait(&bars[G_DONE], 0, kWaitLimitCycles)) gemm_flag(a);
        }
    } else {
        // -------------------------------------------------------------------- epilogue
        // 64 columns per step: a lane converts its row's 64 values into 8 chunks of 8 bf16,
        // then a transpose over groups of 8 lanes lets 8 lanes store one row's 128 bytes
        // side by side (segment boundaries and N are multiples of 64)
        const int q = warp & 3;                          // TMEM lane quarter: rows 32q ..
        const int half = (warp - 2) >> 2;                // columns [half BN/2, (half+1) BN/2)
        const int r = q * 32 + lane;                     // row of the tile == TMEM lane
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const int j = lane & 7;                          // chunk this lane stores
        int t = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++t) {
            const int acc = t & 1;
            const int m0 = (tile / nt) * GBM, n0 = (tile % nt) * BN;
            if (!warp_wait(&bars[ACC_FULL + acc], (t >> 1) & 1, a.wait_limit)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int m = m0 + r;
#pragma unroll 1
            for (int c0 = half * (BN / 2); c0 < (half + 1) * (BN / 2); c0 += 64) {
                __syncwarp();                             // the warp-wide TMEM loads below
                uint32_t v[32], w[32];
                tmem_ld32(tmem + lane_base + acc * BN + c0, v);
                tmem_ld32(tmem + lane_base + acc * BN + c0 + 32, w);
                tmem_wait_ld();
                reg_fence(v);
                reg_fence(w);
                const int nb = n0 + c0;
                if (nb >= a.N) continue;                  // (warp-uniform)
                int sg = 0;
                while (sg + 1 < a.nseg && nb >= a.lo[sg + 1]) ++sg;
                float4 o[8];                              // 8 chunks of 8 bf16 (as 16 bytes)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float f[32];
#pragma unroll
                    for (int x = 0; x < 32; ++x) f[x] = __uint_as_float(hh ? w[x] : v[x]);
                    const int nc = nb + 32 * hh;
                    if (a.bias) {
                        const float4 *bp = reinterpret_cast<const float4 *>(a.bias + nc);
#pragma unroll
                        for (int x = 0; x < 8; ++x) {
                            const float4 bv = __ldg(bp + x);
                            f[4 * x] += bv.x; f[4 * x + 1] += bv.y; f[4 * x + 2] += bv.z; f[4 * x + 3] += bv.w;
                        }
                    }
                    if (a.silu) {
#pragma unroll
                        for (int x = 0; x < 32; ++x) f[x] = f[x] * __fdividef(1.0f, 1.0f + __expf(-f[x]));
                    }
                    if (a.resid && m < a.M) {
                        const uint4 *rp = reinterpret_cast<const uint4 *>(a.resid + (int64_t)m * a.N + nc);
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            const uint4 rv = rp[x];
                            const uint32_t u4[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
                            for (int y = 0; y < 4; ++y) {
                                f[8 * x + 2 * y] += __uint_as_float(u4[y] << 16);
                                f[8 * x + 2 * y + 1] += __uint_as_float(u4[y] & 0xFFFF0000u);
                            }
                        }
                    }
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        o[4 * hh + x] = make_float4(__uint_as_float(pack_bf16x2(f[8 * x], f[8 * x + 1])),
                                                    __uint_as_float(pack_bf16x2(f[8 * x + 2], f[8 * x + 3])),
                                                    __uint_as_float(pack_bf16x2(f[8 * x + 4], f[8 * x + 5])),
                                                    __uint_as_float(pack_bf16x2(f[8 * x + 6], f[8 * x + 7])));
                }
                // lane l now stores chunk j = l % 8 of rows l - j .. l - j + 7 of this warp
                transpose_chunks<8>(o);
                const int width = a.lo[sg + 1] - a.lo[sg];
                const int mr = m0 + q * 32 + (lane - j);
                __nv_bfloat16 *ob = a.out[sg] + (int64_t)mr * width + (nb - a.lo[sg]) + 8 * j;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    if (mr + c < a.M)
                        *reinterpret_cast<float4 *>(ob + (int64_t)c * width) = o[c];
            }
            __syncwarp();
            tc_fence_before();
            warp_arrive(&bars[ACC_EMPTY + acc]);
        }
        if (!ok && lane == 0) gemm_flag(a);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * BN);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// A row-major [rows, cols] bf16 matrix as a 2-D TMA tensor (cols, rows), box (64, box_rows).
bool encode_2d(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int BN>
cudaError_t run_gemm(GemmArgs &a, cudaStream_t st)
{
    using L = GLayout<BN>;
    static_assert(L::ALLOC <= 232448, "shared memory");
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    const int tiles = ((a.M + GBM - 1) / GBM) * ((a.N + BN - 1) / BN);
    int grid = num_sms();
    if (tiles < grid) grid = tiles;
    if (grid <= 0) return cudaSuccess;
    gemm_tc_kernel<BN><<<grid, kGThreads, L::ALLOC, st>>>(a);
    return cudaGetLastError();
}

// Input normalisation: one warp per row of `width` (a multiple of 32, at most 1024) bf16
// values; LayerNorm without affine (biased variance, eps inside the square root).
__global__ void __launch_bounds__(256) ln_rows_kernel(const __nv_bfloat16 *__restrict__ x,
                                                      __nv_bfloat16 *__restrict__ y,
                                                      int64_t rows, int width, float eps)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int per = width / 32;
    float v[32];
    float sum = 0.f;
#pragma unroll
    for (int c = 0; c < 32; ++c)
        if (c < per) {
            v[c] = __bfloat162float(x[row * width + c * 32 + lane]);
            sum += v[c];
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float mu = sum / (float)width;
    float sq = 0.f;
#pragma unroll
    for (int c = 0; c < 32; ++c)
        if (c < per) {
            v[c] -= mu;
            sq = fmaf(v[c], v[c], sq);
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    const float rs = rsqrtf(sq / (float)width + eps);
#pragma unroll
    for (int c = 0; c < 32; ++c)
        if (c < per) y[row * width + c * 32 + lane] = __float2bfloat16_rn(v[c] * rs);
}

}  // namespace

cudaError_t launch_ln_rows(const void *x, void *y, int64_t rows, int width, float eps,
                           cudaStream_t st)
{
    if (rows <= 0) return cudaSuccess;
    const int64_t blocks = (rows + 7) / 8;
    ln_rows_kernel<<<(unsigned)blocks, 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16 *>(x), reinterpret_cast<__nv_bfloat16 *>(y), rows,
        width, eps);
    return cudaGetLastError();
}

cudaError_t launch_gemm(const void *A, const void *B, int M, int N, int K, const float *bias,
                        bool silu, const void *resid, int nseg, const int *seg_lo,
                        void *const *outs, int32_t *status, long long wait_limit,
                        cudaStream_t st)
{
    if (M <= 0) return cudaSuccess;
    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    // 128-wide tiles: twice the tiles of 256-wide ones, so the last wave of the persistent
    // grid is fuller (the U/V/Q/K projection of 10.9k tokens: 0.0256 against 0.0267 ms)
    constexpr int BN = 128;
    if (!encode_2d(&a.ta, A, M, K, GBM) || !encode_2d(&a.tb, B, K, N, GBK))
        return cudaErrorInvalidValue;
    a.M = M;
    a.N = N;
    a.K = K;
    a.bias = bias;
    a.silu = silu ? 1 : 0;
    a.resid = reinterpret_cast<const __nv_bfloat16 *>(resid);
    a.nseg = nseg;
    for (int s = 0; s <= nseg; ++s) a.lo[s] = seg_lo[s];
    for (int s = 0; s < nseg; ++s) a.out[s] = reinterpret_cast<__nv_bfloat16 *>(outs[s]);
    a.status = status;
    a.wait_limit = wait_limit;
    return run_gemm<BN>(a, st);
}

}  // namespace hstu
