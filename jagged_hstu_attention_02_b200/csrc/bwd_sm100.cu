// bwd_sm100.cu -- tensor-core (tcgen05) backward attention of jagged HSTU for B200.
//
// Gradients of Y = (1/N) sum_j A_ij V_j with A_ij = mask * SiLU(alpha q_i.k_j + b_ij), given
// dY (the LayerNorm/gating backward has already run):
//   dV_j += sum_i A_ij dY_i;      dA_ij = dY_i . V_j;      dS_ij = mask dA_ij SiLU'(s_ij) / N
//   dK_j += alpha sum_i dS_ij Q_i;  dQ_i += alpha sum_j dS_ij K_j;
//   d rel[r_ij] += dS_ij;  d time[bucket_ij] += dS_ij.
// The reverse pass of "HSTU tensor by tensor: SiLU aggregation, temporal bias and gating",
// "Similar shape, different aggregation"; the mask multiplies after the nonlinearity, so
// masked pairs get exactly zero gradient ("Do not copy softmax masking mechanically").
//
// One CTA per (128-key tile, sequence, head); it walks the 128-row query tiles that see
// the keys.  Thread = key row = TMEM lane, so scores are computed transposed:
//   S^T = K Q^T and dP^T = V dY^T          (tcgen05, bf16 in smem, fp32 in TMEM)
//   epilogue: A^T (bf16, over S^T in TMEM) and dS^T (bf16, 128B-swizzled in smem)
//   dV += A^T dY (A from TMEM), dK += dS^T Q, dQ_tile = dS K (dS^T read as an MN-major A)
// dV and dK accumulate in TMEM across query tiles; each dQ tile is added to an fp32
// accumulator in global memory with vector atomics.  Table gradients go through
// shared-memory histograms.  Warp roles as in the forward: TMA producer, MMA issuer, TMEM
// owner, query-timestamp staging, and two epilogue warpgroups that split the query
// columns.  Every wait is bounded.
#include <cudaTypedefs.h>

#include <cstring>

#include "bias.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hstu {

using namespace sm100;

namespace {

constexpr int BM = 128, BN = 128, HALF = kHalf;
constexpr int kThreads = 384;
constexpr int kRelSmemMax = 2048;
constexpr uint32_t kTmemCols = 512;
constexpr int kBlockBytes = 128 * 128;
// TMEM columns: S^T -> A^T [0,128); dP^T -> dQ tile [128,256); dV [256,384); dK [384,512)
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;

enum Bar { KV_FULL = 0, QD_FULL = 1, QD_EMPTY = 2, SD_FULL = 3, META_FULL = 4, P_FULL = 5,
           DQ_FULL = 6, DQ_FREE = 7, ACC_FULL = 8, MMA_DONE = 9, NUM_BARS = 10 };

struct QMeta {
    int64_t tmin[2], tmax[2];
    int32_t ok32[2];
    int32_t pad[2];
};

template <int DQK, int DV>
struct BwdLayout {
    static constexpr int KB = BN * DQK * 2;
    static constexpr int VB = BN * DV * 2;
    static constexpr int QB = BM * DQK * 2;
    static constexpr int YB = BM * DV * 2;
    static constexpr int SB = BN * BM * 2;
    static constexpr int K_OFF = 0;
    static constexpr int V_OFF = K_OFF + KB;
    static constexpr int Q_OFF = V_OFF + VB;
    static constexpr int Y_OFF = Q_OFF + QB;
    static constexpr int YL_OFF = Y_OFF + YB;
    static constexpr int DS_OFF = YL_OFF + YB;
    static constexpr int BAR_OFF = DS_OFF + SB;
    static constexpr int SLOT_OFF = BAR_OFF + 8 * 16;
    static constexpr int META_OFF = SLOT_OFF + 16;
    static constexpr int TSQ_OFF = META_OFF + (int)sizeof(QMeta);
    static constexpr int TSQ32_OFF = TSQ_OFF + BM * 8;
    static constexpr int LUT_OFF = TSQ32_OFF + BM * 4;
    static constexpr int THR_OFF = LUT_OFF + kLutCells * 8;
    static constexpr int TB_OFF = THR_OFF + 8 * kMaxTimeBuckets;
    static constexpr int HTB_OFF = TB_OFF + 4 * kMaxTimeBuckets;
    static constexpr int REL_OFF = HTB_OFF + 4 * kMaxTimeBuckets;
    static constexpr int HREL_OFF = REL_OFF + 4 * kRelSmemMax;
    static constexpr int TOTAL = HREL_OFF + 4 * kRelSmemMax;
    static constexpr int ALLOC = TOTAL + 1024;
};

struct BwdTcArgs {
    CUtensorMap tq, tk, tv, tdy, tdyl;   // dY as bf16 hi and lo parts
    DevParams p;
    float *dq_acc;                 // [T, H, d_qk] fp32, zeroed by the caller
    __nv_bfloat16 *dk, *dv;        // [T, H, d]
    float *d_rel, *d_tb;
};

// The query tiles [i0, i0+BM) that see key tile [j0, j0+BN), in order.
struct QTileIter {
    const SeqInfo &s;
    int j0, W, qt, nqt;
    __device__ QTileIter(const SeqInfo &s_, int j0_, int W_)
        : s(s_), j0(j0_), W(W_), qt(-1), nqt((s_.L + BM - 1) / BM) {}
    __device__ bool next()
    {
        while (++qt < nqt)
            if (tile_any_valid(qt * BM, qt * BM + BM - 1, j0, j0 + BN - 1, s, W)) return true;
        return false;
    }
};

__device__ __forceinline__ void report_timeout(const DevParams &p)
{
    flag_error(p, HSTU_DEV_WAIT_TIMEOUT);
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

__device__ __forceinline__ void red_add_v4(float *addr, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
                 "f"(c), "f"(d)
                 : "memory");
}

template <int DQK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_tc_kernel(const __grid_constant__ BwdTcArgs args)
{
    using L = BwdLayout<DQK, DV>;
    const DevParams &p = args.p;
    const int kt = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
    const SeqInfo s = load_seq(p, b, kt == 0 && h == 0 && threadIdx.x == 0);
    const int j0 = kt * BN;
    if (j0 >= s.L) return;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR_OFF);
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT_OFF);
    int32_t *lut_valid = reinterpret_cast<int32_t *>(sm + L::SLOT_OFF + 4);
    QMeta *meta = reinterpret_cast<QMeta *>(sm + L::META_OFF);
    int64_t *tsq = reinterpret_cast<int64_t *>(sm + L::TSQ_OFF);
    int32_t *tsq32 = reinterpret_cast<int32_t *>(sm + L::TSQ32_OFF);
    LutEntry *lut = reinterpret_cast<LutEntry *>(sm + L::LUT_OFF);
    uint64_t *thr = reinterpret_cast<uint64_t *>(sm + L::THR_OFF);
    float *tbs = reinterpret_cast<float *>(sm + L::TB_OFF);
    float *htb = reinterpret_cast<float *>(sm + L::HTB_OFF);
    float *rels = reinterpret_cast<float *>(sm + L::REL_OFF);
    float *hrel = reinterpret_cast<float *>(sm + L::HREL_OFF);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int x = 0; x < NUM_BARS; ++x) mbar_init(&bars[x], 1);
        mbar_init(&bars[META_FULL], 32);
        mbar_init(&bars[P_FULL], 256);
        mbar_init(&bars[DQ_FREE], 256);
        fence_mbar_init();
        *lut_valid = 1;
    }
    if (warp == 2) tmem_alloc(slot, kTmemCols);
    for (int x = threadIdx.x; x < p.n_thr; x += kThreads) thr[x] = p.thr[x];
    for (int x = threadIdx.x; x < p.NB; x += kThreads) {
        tbs[x] = p.tb[x];
        htb[x] = 0.f;
    }
    const bool rel_in_smem = p.R <= kRelSmemMax;
    if (rel_in_smem)
        for (int x = threadIdx.x; x < p.R; x += kThreads) {
            rels[x] = p.rel[x];
            hrel[x] = 0.f;
        }
    __syncthreads();
    if (p.NB > 0) build_lut(thr, p.n_thr, lut, lut_valid);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    const uint32_t sm_base = smem_u32(sm);
    const int row0 = (int)s.start;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- TMA producer
            prefetch_tmap(&args.tq);
            prefetch_tmap(&args.tk);
            prefetch_tmap(&args.tv);
            prefetch_tmap(&args.tdy);
            prefetch_tmap(&args.tdyl);
            mbar_arrive_expect_tx(&bars[KV_FULL], L::KB + L::VB);
            for (int kb = 0; kb < DQK / 64; ++kb)
                tma_load_3d(sm + L::K_OFF + kb * kBlockBytes, &args.tk, &bars[KV_FULL], kb * 64, h,
                            row0 + j0);
            for (int kb = 0; kb < DV / 64; ++kb)
                tma_load_3d(sm + L::V_OFF + kb * kBlockBytes, &args.tv, &bars[KV_FULL], kb * 64, h,
                            row0 + j0);
            QTileIter t(s, j0, p.W);
            int x = 0;
            bool ok = true;
            while (t.next()) {
                if (x >= 1 && !mbar_wait(&bars[QD_EMPTY], (x - 1) & 1)) { ok = false; break; }
                const int i0 = t.qt * BM;
                mbar_arrive_expect_tx(&bars[QD_FULL], L::QB + 2 * L::YB);
                for (int kb = 0; kb < DQK / 64; ++kb)
                    tma_load_3d(sm + L::Q_OFF + kb * kBlockBytes, &args.tq, &bars[QD_FULL], kb * 64,
                                h, row0 + i0);
                for (int kb = 0; kb < DV / 64; ++kb) {
                    tma_load_3d(sm + L::Y_OFF + kb * kBlockBytes, &args.tdy, &bars[QD_FULL],
                                kb * 64, h, row0 + i0);
                    tma_load_3d(sm + L::YL_OFF + kb * kBlockBytes, &args.tdyl, &bars[QD_FULL],
                                kb * 64, h, row0 + i0);
                }
                ++x;
            }
            if (!ok) report_timeout(p);
            bool drained = mbar_wait(&bars[KV_FULL], 0);
            if (x >= 1) drained &= mbar_wait(&bars[QD_FULL], (x - 1) & 1);
            if (!drained) report_timeout(p);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            constexpr uint32_t id_s = idesc_bf16(BN, BM, false, false);      // S^T, dP^T
            constexpr uint32_t id_dv = idesc_bf16(BN, DV, false, true);      // A^T dY
            constexpr uint32_t id_dk = idesc_bf16(BN, DQK, false, true);     // dS^T Q
            constexpr uint32_t id_dq = idesc_bf16(BM, DQK, true, true);      // dS K
            const uint32_t k_addr = sm_base + L::K_OFF, v_addr = sm_base + L::V_OFF;
            const uint32_t q_addr = sm_base + L::Q_OFF, y_addr = sm_base + L::Y_OFF;
            const uint32_t yl_addr = sm_base + L::YL_OFF;
            const uint32_t ds_addr = sm_base + L::DS_OFF;
            bool ok = mbar_wait(&bars[KV_FULL], 0);
            QTileIter t(s, j0, p.W);
            int x = 0;
            while (ok && t.next()) {
                if (!mbar_wait(&bars[QD_FULL], x & 1)) { ok = false; break; }
                // the previous tile's dQ readout is done, so every MMA of it completed and
                // TMEM [0,256) and the dS^T buffer are free
                if (x >= 1 && !mbar_wait(&bars[DQ_FREE], (x - 1) & 1)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kb = 0; kb < DQK / 64; ++kb)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t a = sw128_desc(k_addr + kb * kBlockBytes + ks * 32, 16, 1024);
                        const uint64_t bd = sw128_desc(q_addr + kb * kBlockBytes + ks * 32, 16, 1024);
                        umma_bf16_ss(tmem + kColS, a, bd, id_s, (kb | ks) ? 1u : 0u);
                    }
                // dP^T = V (dY_hi + dY_lo)^T
#pragma unroll
                for (int kb = 0; kb < DV / 64; ++kb)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t a = sw128_desc(v_addr + kb * kBlockBytes + ks * 32, 16, 1024);
                        const uint64_t bd = sw128_desc(y_addr + kb * kBlockBytes + ks * 32, 16, 1024);
                        const uint64_t bl = sw128_desc(yl_addr + kb * kBlockBytes + ks * 32, 16, 1024);
                        umma_bf16_ss(tmem + kColDP, a, bd, id_s, (kb | ks) ? 1u : 0u);
                        umma_bf16_ss(tmem + kColDP, a, bl, id_s, 1u);
                    }
                umma_commit(&bars[SD_FULL]);
                if (!mbar_wait(&bars[P_FULL], x & 1)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < BM / 16; ++kk) {
                    // dV += A^T dY: A^T packed in TMEM (queries 64h.. at columns 64h..64h+31)
                    const uint32_t a_tmem = tmem + kColS + (kk >> 2) * 64 + (kk & 3) * 8;
                    const uint64_t bd = sw128_desc(y_addr + kk * 2048, kBlockBytes, 1024);
                    umma_bf16_ts(tmem + kColDV, a_tmem, bd, id_dv, (x > 0 || kk > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < BM / 16; ++kk) {
                    // dK += dS^T Q: dS^T K-major [keys x queries], Q as MN-major B
                    const uint64_t a = sw128_desc(ds_addr + (kk >> 2) * kBlockBytes + (kk & 3) * 32,
                                                  16, 1024);
                    const uint64_t bd = sw128_desc(q_addr + kk * 2048, kBlockBytes, 1024);
                    umma_bf16_ss(tmem + kColDK, a, bd, id_dk, (x > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&bars[QD_EMPTY]);
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    // dQ = dS K: dS^T read as an MN-major A (queries contiguous per key row)
                    const uint64_t a = sw128_desc(ds_addr + kk * 2048, kBlockBytes, 1024);
                    const uint64_t bd = sw128_desc(k_addr + kk * 2048, kBlockBytes, 1024);
                    umma_bf16_ss(tmem + kColDP, a, bd, id_dq, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bars[DQ_FULL]);
                ++x;
            }
            umma_commit(&bars[ACC_FULL]);
            if (!ok) report_timeout(p);
            umma_commit(&bars[MMA_DONE]);
            if (!mbar_wait(&bars[MMA_DONE], 0)) report_timeout(p);
        }
    } else if (warp == 3) {
        // -------------------------------------------------------------------- query stamps
        const bool use_ts = p.NB > 0;
        QTileIter t(s, j0, p.W);
        int x = 0;
        while (t.next()) {
            // the epilogue of the previous tile has read the staged stamps
            if (x >= 1 && !warp_wait(&bars[P_FULL], (x - 1) & 1)) {
                report_timeout(p);
                break;
            }
            if (use_ts) {
                const int i0 = t.qt * BM;
                int64_t v[4];
                int64_t mn[2] = {INT64_MAX, INT64_MAX}, mx[2] = {INT64_MIN, INT64_MIN};
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int i = i0 + lane + 32 * q4;
                    v[q4] = 0;
                    if (i < s.L) {
                        v[q4] = p.ts[s.start + clamp_pos(i, s.E)];
                        mn[q4 >> 1] = min(mn[q4 >> 1], v[q4]);
                        mx[q4 >> 1] = max(mx[q4 >> 1], v[q4]);
                    }
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        mn[hh] = min(mn[hh], shfl_xor_i64(mn[hh], o));
                        mx[hh] = max(mx[hh], shfl_xor_i64(mx[hh], o));
                    }
                int ok32[2];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    ok32[hh] = mn[hh] > mx[hh] ||
                               (uint64_t)mx[hh] - (uint64_t)mn[hh] < (uint64_t)INT32_MAX;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int c = lane + 32 * q4, hh = q4 >> 1;
                    tsq[c] = v[q4];
                    tsq32[c] = (i0 + c < s.L && ok32[hh])
                                   ? (int32_t)((uint64_t)v[q4] - (uint64_t)mn[hh]) : 0;
                }
                if (lane == 0)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        meta->tmin[hh] = mn[hh];
                        meta->tmax[hh] = mx[hh];
                        meta->ok32[hh] = ok32[hh];
                    }
            }
            __syncwarp();
            mbar_arrive(&bars[META_FULL]);
            ++x;
        }
    } else if (warp >= 4) {
        // -------------------------------------------------------------------- epilogue
        const int wg = (warp - 4) >> 2;              // query columns [64 wg, 64 wg + 64)
        const int r = (warp & 3) * 32 + lane;        // key row in the tile == TMEM lane
        const int j = j0 + r;
        const bool key_in = j < s.L;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const int pj = clamp_pos(j, s.E);
        const bool use_ts = p.NB > 0, use_rel = p.R > 0;
        const int64_t tsj = (use_ts && key_in) ? p.ts[s.start + pj] : 0;
        const float *relp = rel_in_smem ? rels : p.rel;
        const bool lut_ok = *lut_valid != 0;
        const int Em1 = s.E > 0 ? s.E - 1 : 0x7fffffff;   // p(i) = min(i, E-1) when E > 0
        const uint32_t ds_row = sm_base + L::DS_OFF + wg * kBlockBytes + r * 128;
        bool ok = true;
        QTileIter t(s, j0, p.W);
        int x = 0;
        while (t.next()) {
            const int ih = t.qt * BM + wg * HALF;     // first query of this warpgroup's half
            if (!warp_wait(&bars[META_FULL], x & 1) || !warp_wait(&bars[SD_FULL], x & 1)) {
                ok = false;
                break;
            }
            const bool full = tile_all_valid(ih, ih + HALF - 1, j0, j0 + BN - 1, s, p.W);
            const uint64_t vmask = full ? ~0ull : col_valid_bits(j, ih, s, p.W);
            // rel index p(i) - p(j) = rbase + c when no query of the half is a candidate
            const int rbase = ih - pj;
            const bool rdirect = __all_sync(0xffffffffu, !use_rel ||
                                                              (ih + HALF - 1 < s.E && rbase >= 0 &&
                                                               rbase + HALF - 1 <= p.R - 1));
            HalfTime ht = {};
            int tmode = 0;
            if (use_ts) {
                ht = half_time_setup(thr, p.n_thr, tbs, p.NB, key_in, tsj, meta->tmin[wg],
                                     meta->tmax[wg], meta->ok32[wg] != 0, lut_ok, lut);
                tmode = __reduce_max_sync(0xffffffffu, ht.my_mode);
            }
            float tsum_lo = 0.f, tsum_hi = 0.f;    // dS sums per bucket in modes 0/1
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < 2; ++ch) {
                const int cb = ch * 32;
                uint32_t rs[32], rd[32];
                tmem_ld32(tmem + lane_base + kColS + wg * HALF + cb, rs);
                tmem_ld32(tmem + lane_base + kColDP + wg * HALF + cb, rd);
                tmem_wait_ld();
                reg_fence(rs);
                reg_fence(rd);
                const uint32_t vbits = (uint32_t)(vmask >> cb);
                uint32_t pa[16], pd[16];
#pragma unroll
                for (int c2 = 0; c2 < 16; ++c2) {
                    float av[2], dv2[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int c = 2 * c2 + e, cc = cb + c;
                        const int i = ih + cc;
                        const bool valid = full || ((vbits >> c) & 1u);
                        float bias = 0.f;
                        int ri = -1, bk = -1;
                        if (use_rel) {
                            if (rdirect) {
                                ri = rbase + cc;
                            } else {
                                ri = min(i, Em1) - pj;
                                ri = ri < 0 ? 0 : (ri > p.R - 1 ? p.R - 1 : ri);
                            }
                            bias = relp[ri];
                        }
                        if (use_ts)
                            bias += half_time_value(ht, tmode, tsq32[wg * HALF + cc],
                                                    tsq[wg * HALF + cc], tsj, thr, p.n_thr, tbs,
                                                    lut, &bk);
                        // s = alpha q.k + b; SiLU(s) = s sigma(s); SiLU'(s) = sigma (1 + s (1 - sigma)).
                        // sigma from the accurate exponential: table gradients sum dS over many
                        // pairs and can cancel, so dS needs close to fp32 accuracy
                        const float xs = fmaf(p.alpha, __uint_as_float(rs[c]), bias);
                        const float sig = __fdividef(1.0f, 1.0f + __expf(-xs));
                        const float silu = xs * sig;
                        const float dsilu = sig * fmaf(xs, 1.0f - sig, 1.0f);
                        const float a = valid ? silu * p.inv_N : 0.f;
                        const float ds = valid ? __uint_as_float(rd[c]) * dsilu * p.inv_N : 0.f;
                        av[e] = a;
                        dv2[e] = ds;
                        // table gradients
                        if (valid) {
                            if (use_rel) {
                                if (rel_in_smem) atomicAdd(hrel + ri, ds);
                                else atomicAdd(args.d_rel + ri, ds);
                            }
                            if (use_ts) {
                                if (tmode <= 1) {
                                    if (bk == ht.blo) tsum_lo += ds; else tsum_hi += ds;
                                } else {
                                    atomicAdd(htb + bk, ds);
                                }
                            }
                        }
                    }
                    pa[c2] = pack_bf16x2(av[0], av[1]);
                    pd[c2] = pack_bf16x2(dv2[0], dv2[1]);
                }
                // A^T over the first 32 of this warpgroup's S^T columns
                tmem_st16(tmem + lane_base + kColS + wg * HALF + ch * 16, pa);
                // dS^T row r, queries wg*64 + cb .. +31: 16-byte chunks (cb/8 .. cb/8+3), swizzled
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int chunk = (cb >> 3) + q;
                    st_shared_v4(ds_row + ((chunk ^ (r & 7)) << 4), pd[4 * q], pd[4 * q + 1],
                                 pd[4 * q + 2], pd[4 * q + 3]);
                }
            }
            if (use_ts && tmode <= 1) {
                if (tsum_lo != 0.f) atomicAdd(htb + ht.blo, tsum_lo);
                if (tsum_hi != 0.f) atomicAdd(htb + min(ht.blo + 1, p.NB - 1), tsum_hi);
            }
            tmem_wait_st();
            tc_fence_before();
            fence_proxy_async_smem();
            mbar_arrive(&bars[P_FULL]);

            // ---- dQ tile: lanes = query rows of this tile; columns split by warpgroup
            if (!warp_wait(&bars[DQ_FULL], x & 1)) { ok = false; break; }
            tc_fence_after();
            {
                const int i = t.qt * BM + r;
                float *dqr = args.dq_acc + ((s.start + i) * (int64_t)p.H + h) * DQK;
#pragma unroll 1
                for (int c = wg * (DQK / 64); c < (wg + 1) * (DQK / 64); ++c) {
                    uint32_t rq[32];
                    tmem_ld32(tmem + lane_base + kColDP + c * 32, rq);
                    tmem_wait_ld();
                    reg_fence(rq);
                    if (i < s.L) {
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            red_add_v4(dqr + c * 32 + 4 * q, p.alpha * __uint_as_float(rq[4 * q]),
                                       p.alpha * __uint_as_float(rq[4 * q + 1]),
                                       p.alpha * __uint_as_float(rq[4 * q + 2]),
                                       p.alpha * __uint_as_float(rq[4 * q + 3]));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bars[DQ_FREE]);
            ++x;
        }
        // ---- dV and dK of the key rows (every key tile sees at least its diagonal tile)
        if (ok && !warp_wait(&bars[ACC_FULL], 0)) ok = false;
        if (ok && x == 0) {
            if (key_in) {
                __nv_bfloat16 *dvr = args.dv + ((s.start + j) * (int64_t)p.H + h) * DV;
                __nv_bfloat16 *dkr = args.dk + ((s.start + j) * (int64_t)p.H + h) * DQK;
                for (int c = wg * (DV / 2); c < (wg + 1) * (DV / 2); ++c) dvr[c] = __float2bfloat16_rn(0.f);
                for (int c = wg * (DQK / 2); c < (wg + 1) * (DQK / 2); ++c) dkr[c] = __float2bfloat16_rn(0.f);
            }
        } else if (ok) {
            tc_fence_after();
            __nv_bfloat16 *dvr = args.dv + ((s.start + j) * (int64_t)p.H + h) * DV;
            __nv_bfloat16 *dkr = args.dk + ((s.start + j) * (int64_t)p.H + h) * DQK;
#pragma unroll 1
            for (int c = wg * (DV / 64); c < (wg + 1) * (DV / 64); ++c) {
                uint32_t ra[32];
                tmem_ld32(tmem + lane_base + kColDV + c * 32, ra);
                tmem_wait_ld();
                reg_fence(ra);
                if (key_in) {
                    uint4 *dst = reinterpret_cast<uint4 *>(dvr + c * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(
                            pack_bf16x2(__uint_as_float(ra[8 * q]), __uint_as_float(ra[8 * q + 1])),
                            pack_bf16x2(__uint_as_float(ra[8 * q + 2]), __uint_as_float(ra[8 * q + 3])),
                            pack_bf16x2(__uint_as_float(ra[8 * q + 4]), __uint_as_float(ra[8 * q + 5])),
                            pack_bf16x2(__uint_as_float(ra[8 * q + 6]), __uint_as_float(ra[8 * q + 7])));
                }
            }
#pragma unroll 1
            for (int c = wg * (DQK / 64); c < (wg + 1) * (DQK / 64); ++c) {
                uint32_t ra[32];
                tmem_ld32(tmem + lane_base + kColDK + c * 32, ra);
                tmem_wait_ld();
                reg_fence(ra);
                if (key_in) {
                    const float al = p.alpha;
                    uint4 *dst = reinterpret_cast<uint4 *>(dkr + c * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(
                            pack_bf16x2(al * __uint_as_float(ra[8 * q]), al * __uint_as_float(ra[8 * q + 1])),
                            pack_bf16x2(al * __uint_as_float(ra[8 * q + 2]), al * __uint_as_float(ra[8 * q + 3])),
                            pack_bf16x2(al * __uint_as_float(ra[8 * q + 4]), al * __uint_as_float(ra[8 * q + 5])),
                            pack_bf16x2(al * __uint_as_float(ra[8 * q + 6]), al * __uint_as_float(ra[8 * q + 7])));
                }
            }
        } else {
            report_timeout(p);
        }
    }

    tc_fence_before();
    __syncthreads();
    // flush the table-gradient histograms
    if (rel_in_smem)
        for (int x = threadIdx.x; x < p.R; x += kThreads)
            if (hrel[x] != 0.f) atomicAdd(args.d_rel + x, hrel[x]);
    for (int x = threadIdx.x; x < p.NB; x += kThreads)
        if (htb[x] != 0.f) atomicAdd(args.d_tb + x, htb[x]);
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int DQK, int DV>
cudaError_t launch_bwd(const BwdTcArgs &a, cudaStream_t st)
{
    using L = BwdLayout<DQK, DV>;
    auto kern = bwd_tc_kernel<DQK, DV>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    dim3 grid((a.p.N + BN - 1) / BN, a.p.B, a.p.H);
    kern<<<grid, kThreads, L::ALLOC, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool tc_bwd_supported(int dqk, int dv, int64_t T) { return tc_fwd_supported(dqk, dv, T); }

cudaError_t launch_tc_bwd(const DevParams &p, const void *q, const void *k, const void *v,
                          const void *dy_bf16, float *dq_acc, void *dk, void *dv, float *d_rel,
                          float *d_tb, cudaStream_t st)
{
    BwdTcArgs a;
    std::memset(&a, 0, sizeof(a));
    a.p = p;
    a.dq_acc = dq_acc;
    a.dk = reinterpret_cast<__nv_bfloat16 *>(dk);
    a.dv = reinterpret_cast<__nv_bfloat16 *>(dv);
    a.d_rel = d_rel;
    a.d_tb = d_tb;
    const void *dy_lo = reinterpret_cast<const char *>(dy_bf16) + (size_t)p.T * p.D * 2;
    if (!encode_tmap_bf16(&a.tq, q, p.dqk, p.H, p.T) || !encode_tmap_bf16(&a.tk, k, p.dqk, p.H, p.T) ||
        !encode_tmap_bf16(&a.tv, v, p.dv, p.H, p.T) ||
        !encode_tmap_bf16(&a.tdy, dy_bf16, p.dv, p.H, p.T) ||
        !encode_tmap_bf16(&a.tdyl, dy_lo, p.dv, p.H, p.T))
        return cudaErrorInvalidValue;
    if (p.dqk == 128 && p.dv == 128) return launch_bwd<128, 128>(a, st);
    if (p.dqk == 128 && p.dv == 64) return launch_bwd<128, 64>(a, st);
    if (p.dqk == 64 && p.dv == 128) return launch_bwd<64, 128>(a, st);
    if (p.dqk == 64 && p.dv == 64) return launch_bwd<64, 64>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace hstu
