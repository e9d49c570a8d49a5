// fwd_sm100.cu -- tensor-core (tcgen05) forward attention of jagged HSTU for B200.
//
// One CTA per (128-row query tile, sequence, head).  Per key tile of 128 that holds a valid
// pair:  S = Q K^T on tcgen05 (bf16 operands staged by TMA in 128-byte-swizzled shared
// memory, fp32 accumulator in TMEM), then the epilogue warps read S from TMEM and form
// A = mask ? SiLU(alpha*S + b) : 0 in fp32 (bias = relative-position + bucketed time table
// entries; the mask is applied after the nonlinearity, never as -inf before it, as "HSTU
// tensor by tensor: SiLU aggregation, temporal bias and gating", section "Do not copy softmax
// masking mechanically", requires), round it to bf16 into shared memory, and tcgen05 adds
// A V into the fp32 output accumulator in TMEM.  The 1/N scale ("HSTU-MUSA: HSTU for Moore
// Threads (MUSA)", "Accuracy Alignment": N = batch max_seqlen) is applied once to the
// accumulator, and Y goes to global memory in fp32 for the LayerNorm + gating kernel.
//
// Warp roles: warp 0 lane 0 issues TMA loads (Q once, K/V double-buffered), warp 1 lane 0
// issues the MMAs, warp 2 owns the TMEM allocation, warps 4-7 are the epilogue (one query
// row per thread, which is also the row's TMEM lane).  S is double-buffered in TMEM so
// QK^T of the next tile runs while the epilogue works on the current one.  Every wait is
// bounded; a timeout sets HSTU_DEV_WAIT_TIMEOUT and the CTA unwinds.
#include <cudaTypedefs.h>

#include <cstring>

#include "kernels.h"
#include "sm100.cuh"

namespace hstu {

using namespace sm100;

namespace {

constexpr int BM = 128, BN = 128;
constexpr int kTcThreads = 256;
constexpr int kRelSmemMax = 4096;
constexpr uint32_t kTmemCols = 512;
constexpr int kBlockBytes = 128 * 128;   // one 128-row x 64-element bf16 swizzle block

enum Bar { Q_FULL = 0, KV_FULL = 1, KV_EMPTY = 3, S_FULL = 5, S_FREE = 7, P_FULL = 9,
           P_FREE = 10, O_FULL = 11, MMA_DONE = 12, NUM_BARS = 13 };

template <int DQK, int DV>
struct FwdLayout {
    static constexpr int QB = BM * DQK * 2;
    static constexpr int KB = BN * DQK * 2;
    static constexpr int VB = BN * DV * 2;
    static constexpr int PB = BM * BN * 2;
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + QB;
    static constexpr int V_OFF = K_OFF + 2 * KB;
    static constexpr int P_OFF = V_OFF + 2 * VB;
    static constexpr int BAR_OFF = P_OFF + PB;
    static constexpr int SLOT_OFF = BAR_OFF + 8 * 16;
    static constexpr int THR_OFF = SLOT_OFF + 16;
    static constexpr int TB_OFF = THR_OFF + 8 * kMaxTimeBuckets;
    static constexpr int REL_OFF = TB_OFF + 4 * kMaxTimeBuckets;
    static constexpr int TOTAL = REL_OFF + 4 * kRelSmemMax;
    static constexpr int ALLOC = TOTAL + 1024;   // slack to align the base to 1024 bytes
};

struct FwdTcArgs {
    CUtensorMap tq, tk, tv;
    DevParams p;
    float *y;
};

// Visits the key tiles of query tile [i0, i0+BM) that hold a valid pair, in order.
struct TileIter {
    const SeqInfo &s;
    int i0, W, kt, nkt;
    __device__ TileIter(const SeqInfo &s_, int i0_, int W_)
        : s(s_), i0(i0_), W(W_), kt(-1), nkt((s_.L + BN - 1) / BN) {}
    __device__ bool next()
    {
        while (++kt < nkt)
            if (tile_any_valid(i0, i0 + BM - 1, kt * BN, kt * BN + BN - 1, s, W)) return true;
        return false;
    }
};

__device__ __forceinline__ void report_timeout(const DevParams &p) { flag_error(p, HSTU_DEV_WAIT_TIMEOUT); }

template <int DQK, int DV>
__global__ void __launch_bounds__(kTcThreads, 1) fwd_tc_kernel(const __grid_constant__ FwdTcArgs args)
{
    using L = FwdLayout<DQK, DV>;
    const DevParams &p = args.p;
    const int qt = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
    const SeqInfo s = load_seq(p, b, qt == 0 && h == 0 && threadIdx.x == 0);
    const int i0 = qt * BM;
    if (i0 >= s.L) return;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR_OFF);
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT_OFF);
    uint64_t *thr = reinterpret_cast<uint64_t *>(sm + L::THR_OFF);
    float *tbs = reinterpret_cast<float *>(sm + L::TB_OFF);
    float *rels = reinterpret_cast<float *>(sm + L::REL_OFF);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        mbar_init(&bars[Q_FULL], 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars[KV_FULL + x], 1);
            mbar_init(&bars[KV_EMPTY + x], 1);
            mbar_init(&bars[S_FULL + x], 1);
            mbar_init(&bars[S_FREE + x], 128);
        }
        mbar_init(&bars[P_FULL], 128);
        mbar_init(&bars[P_FREE], 1);
        mbar_init(&bars[O_FULL], 1);
        mbar_init(&bars[MMA_DONE], 1);
        fence_mbar_init();
    }
    if (warp == 2) tmem_alloc(slot, kTmemCols);
    for (int x = threadIdx.x; x < p.n_thr; x += kTcThreads) thr[x] = p.thr[x];
    for (int x = threadIdx.x; x < p.NB; x += kTcThreads) tbs[x] = p.tb[x];
    const bool rel_in_smem = p.R <= kRelSmemMax;
    if (rel_in_smem)
        for (int x = threadIdx.x; x < p.R; x += kTcThreads) rels[x] = p.rel[x];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    const uint32_t sm_base = smem_u32(sm);

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- TMA producer
            prefetch_tmap(&args.tq);
            prefetch_tmap(&args.tk);
            prefetch_tmap(&args.tv);
            const int row0 = (int)s.start;
            mbar_arrive_expect_tx(&bars[Q_FULL], L::QB);
            for (int kb = 0; kb < DQK / 64; ++kb)
                tma_load_3d(sm + L::Q_OFF + kb * kBlockBytes, &args.tq, &bars[Q_FULL], kb * 64, h,
                            row0 + i0);
            TileIter t(s, i0, p.W);
            int it = 0;
            bool ok = true;
            while (t.next()) {
                const int st = it & 1;
                if (it >= 2 && !mbar_wait(&bars[KV_EMPTY + st], ((it >> 1) - 1) & 1)) {
                    ok = false;
                    break;
                }
                const int j0 = t.kt * BN;
                mbar_arrive_expect_tx(&bars[KV_FULL + st], L::KB + L::VB);
                for (int kb = 0; kb < DQK / 64; ++kb)
                    tma_load_3d(sm + L::K_OFF + st * L::KB + kb * kBlockBytes, &args.tk,
                                &bars[KV_FULL + st], kb * 64, h, row0 + j0);
                for (int kb = 0; kb < DV / 64; ++kb)
                    tma_load_3d(sm + L::V_OFF + st * L::VB + kb * kBlockBytes, &args.tv,
                                &bars[KV_FULL + st], kb * 64, h, row0 + j0);
                ++it;
            }
            if (!ok) report_timeout(p);
            // Loads issued must land before the CTA can exit (bounded).
            bool drained = mbar_wait(&bars[Q_FULL], 0);
            for (int x = it - 1; x >= 0 && x >= it - 2; --x)
                drained &= mbar_wait(&bars[KV_FULL + (x & 1)], (x >> 1) & 1);
            if (!drained) report_timeout(p);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            constexpr uint32_t idesc_qk = idesc_bf16(BM, BN, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16(BM, DV, false, true);
            const uint32_t q_addr = sm_base + L::Q_OFF;
            const uint32_t p_addr = sm_base + L::P_OFF;
            const uint32_t o_tmem = tmem + 256;
            bool ok = mbar_wait(&bars[Q_FULL], 0);
            tc_fence_after();
            auto issue_pv = [&](int x) -> bool {
                if (!mbar_wait(&bars[P_FULL], x & 1)) return false;
                tc_fence_after();
                const uint32_t v_addr = sm_base + L::V_OFF + (x & 1) * L::VB;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t a = sw128_desc(p_addr + (kk >> 2) * kBlockBytes + (kk & 3) * 32,
                                                  16, 1024);
                    const uint64_t bd = sw128_desc(v_addr + kk * 2048, kBlockBytes, 1024);
                    umma_bf16_ss(o_tmem, a, bd, idesc_pv, (x > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&bars[P_FREE]);
                umma_commit(&bars[KV_EMPTY + (x & 1)]);
                return true;
            };
            TileIter t(s, i0, p.W);
            int it = 0;
            while (ok && t.next()) {
                const int st = it & 1;
                if (!mbar_wait(&bars[KV_FULL + st], (it >> 1) & 1)) { ok = false; break; }
                if (it >= 2 && !mbar_wait(&bars[S_FREE + st], ((it >> 1) - 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t k_addr = sm_base + L::K_OFF + st * L::KB;
                const uint32_t s_tmem = tmem + st * 128;
#pragma unroll
                for (int kb = 0; kb < DQK / 64; ++kb)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t a = sw128_desc(q_addr + kb * kBlockBytes + ks * 32, 16, 1024);
                        const uint64_t bd = sw128_desc(k_addr + kb * kBlockBytes + ks * 32, 16, 1024);
                        umma_bf16_ss(s_tmem, a, bd, idesc_qk, (kb | ks) ? 1u : 0u);
                    }
                umma_commit(&bars[S_FULL + st]);
                if (it >= 1 && !issue_pv(it - 1)) { ok = false; break; }
                ++it;
            }
            if (ok && it >= 1) ok = issue_pv(it - 1);
            umma_commit(&bars[O_FULL]);
            if (!ok) report_timeout(p);
            // every MMA issued must complete before TMEM is released (bounded)
            umma_commit(&bars[MMA_DONE]);
            if (!mbar_wait(&bars[MMA_DONE], 0)) report_timeout(p);
        }
    } else if (warp >= 4) {
        // -------------------------------------------------------------------- epilogue
        const int r = threadIdx.x - 128;            // query row in the tile == TMEM lane
        const int i = i0 + r;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const int pi = clamp_pos(i, s.E);
        const bool use_ts = p.NB > 0;
        const int64_t tsi = (use_ts && i < s.L) ? p.ts[s.start + pi] : 0;
        const int64_t *tsg = p.ts + s.start;
        const float *relp = rel_in_smem ? rels : p.rel;
        const float half_alpha = 0.5f * p.alpha;
        const uint32_t p_row = sm_base + L::P_OFF + r * 128;
        bool ok = true;
        TileIter t(s, i0, p.W);
        int it = 0;
        while (t.next()) {
            const int st = it & 1;
            const int j0 = t.kt * BN;
            const bool full = tile_all_valid(i0, i0 + BM - 1, j0, j0 + BN - 1, s, p.W);
            // warp-uniform outcome, so the .sync.aligned TMEM loads below never diverge
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[S_FULL + st], (it >> 1) & 1))) {
                ok = false;
                break;
            }
            if (it >= 1 && !__all_sync(0xffffffffu, mbar_wait(&bars[P_FREE], (it - 1) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t ra[32], rb[32];
                tmem_ld32(tmem + lane_base + st * 128 + half * 64, ra);
                tmem_ld32(tmem + lane_base + st * 128 + half * 64 + 32, rb);
                tmem_wait_ld();
                reg_fence(ra);
                reg_fence(rb);
                uint32_t pk[32];
#pragma unroll
                for (int c2 = 0; c2 < 32; ++c2) {
                    float av[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int c = 2 * c2 + e;                 // column within the half
                        const int j = j0 + half * 64 + c;
                        const uint32_t raw = c < 32 ? ra[c] : rb[c - 32];
                        const bool valid = full || (i < s.L && j < s.L && pair_valid(i, j, s, p.W));
                        float bias = 0.f;
                        const int pj = clamp_pos(j, s.E);
                        if (p.R > 0) {
                            int ri = pi - pj;
                            ri = ri < 0 ? 0 : (ri > p.R - 1 ? p.R - 1 : ri);
                            bias += relp[ri];
                        }
                        if (use_ts) {
                            const int64_t tsj = j < s.L ? __ldg(tsg + pj) : 0;
                            bias += tbs[bucket_search(thr, p.n_thr, abs_diff_u64(tsi, tsj))];
                        }
                        // SiLU(x) = x*sigmoid(x) = h + h*tanh(h) with h = x/2
                        const float hx = fmaf(half_alpha, __uint_as_float(raw), 0.5f * bias);
                        const float a = fmaf(hx, tanh_approx(hx), hx);
                        av[e] = valid ? a : 0.f;
                    }
                    pk[c2] = pack_bf16x2(av[0], av[1]);
                }
                // 128-byte-swizzled K-major A operand: 16-byte chunk ch of row r at (ch ^ (r&7))
                const uint32_t blk = p_row + half * kBlockBytes;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    st_shared_v4(blk + ((ch ^ (r & 7)) << 4), pk[4 * ch], pk[4 * ch + 1],
                                 pk[4 * ch + 2], pk[4 * ch + 3]);
            }
            tc_fence_before();
            mbar_arrive(&bars[S_FREE + st]);
            fence_proxy_async_smem();
            mbar_arrive(&bars[P_FULL]);
            ++it;
        }
        if (ok && !__all_sync(0xffffffffu, mbar_wait(&bars[O_FULL], 0))) ok = false;
        if (ok) {
            tc_fence_after();
            float *yr = args.y + (s.start + i) * (int64_t)p.D + h * DV;
#pragma unroll 1
            for (int c = 0; c < DV / 32; ++c) {
                uint32_t ra[32];
                tmem_ld32(tmem + lane_base + 256 + c * 32, ra);
                tmem_wait_ld();
                reg_fence(ra);
                if (i < s.L) {
                    float4 *dst = reinterpret_cast<float4 *>(yr + c * 32);
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        dst[x] = make_float4(__uint_as_float(ra[4 * x]) * p.inv_N,
                                             __uint_as_float(ra[4 * x + 1]) * p.inv_N,
                                             __uint_as_float(ra[4 * x + 2]) * p.inv_N,
                                             __uint_as_float(ra[4 * x + 3]) * p.inv_N);
                }
            }
        } else {
            report_timeout(p);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 tmap_encode_fn()
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

// [T, H, d] bf16 row-major as a 3-D tensor (d, H, T); box 64 x 1 x 128, 128-byte swizzle.
bool encode_tmap(CUtensorMap *m, const void *base, int d, int H, int64_t T)
{
    auto fn = tmap_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
    cuuint32_t box[3] = {64, 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int DQK, int DV>
cudaError_t launch_tc(const FwdTcArgs &a, cudaStream_t st)
{
    using L = FwdLayout<DQK, DV>;
    auto kern = fwd_tc_kernel<DQK, DV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    dim3 grid((a.p.N + BM - 1) / BM, a.p.B, a.p.H);
    kern<<<grid, kTcThreads, L::ALLOC, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool tc_fwd_supported(int dqk, int dv, int64_t T)
{
    return (dqk == 64 || dqk == 128) && (dv == 64 || dv == 128) && T < ((int64_t)1 << 31);
}

cudaError_t launch_tc_fwd(const DevParams &p, const void *q, const void *k, const void *v,
                          float *y, cudaStream_t st)
{
    FwdTcArgs a;
    std::memset(&a, 0, sizeof(a));
    a.p = p;
    a.y = y;
    if (!encode_tmap(&a.tq, q, p.dqk, p.H, p.T) || !encode_tmap(&a.tk, k, p.dqk, p.H, p.T) ||
        !encode_tmap(&a.tv, v, p.dv, p.H, p.T))
        return cudaErrorInvalidValue;
    if (p.dqk == 128 && p.dv == 128) return launch_tc<128, 128>(a, st);
    if (p.dqk == 128 && p.dv == 64) return launch_tc<128, 64>(a, st);
    if (p.dqk == 64 && p.dv == 128) return launch_tc<64, 128>(a, st);
    if (p.dqk == 64 && p.dv == 64) return launch_tc<64, 64>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace hstu
