// fwd_sm100.cu -- tensor-core (tcgen05) forward attention of jagged HSTU for B200.
//
// One CTA per (128-row query tile, sequence, head).  For every key tile of 128 that holds a
// valid pair:  S = Q K^T on tcgen05 (bf16 operands staged by TMA in 128-byte-swizzled shared
// memory, fp32 accumulator in TMEM); the epilogue warps read S from TMEM and form
// A = mask ? SiLU(alpha*S + b) : 0 in fp32, where b is the relative-position plus bucketed
// time bias and the mask is applied after the nonlinearity, never as -inf before it ("HSTU
// tensor by tensor: SiLU aggregation, temporal bias and gating", sections "Similar shape,
// different aggregation" and "Do not copy softmax masking mechanically"); A is rounded to
// bf16 and written back over S in TMEM (two elements per 32-bit column), and tcgen05 adds
// A V into the fp32 output accumulator in TMEM with A read from TMEM.  The 1/N scale
// ("HSTU-MUSA: HSTU for Moore Threads (MUSA)", "Accuracy Alignment": N = batch max_seqlen)
// is applied once to the accumulator; Y goes to global memory in fp32.
//
// Warp roles (12 warps): warp 0 lane 0 issues TMA loads (Q once, K/V double-buffered);
// warp 1 lane 0 issues the MMAs; warp 2 owns TMEM; warp 3 stages each key tile's timestamps
// and their range; warps 4-7 and 8-11 are two epilogue warpgroups, each owning 64 of the
// 128 key columns of every query row (thread = row = TMEM lane).  S is double-buffered, so
// QK^T of the next tile runs while the epilogue works on this one.
//
// Bias evaluation per (row, 64-key half tile):  the time bucket is computed once for the
// smallest and largest |dt| the half can produce (from the half's timestamp range); when
// both agree (the common case away from the diagonal) the time bias is a per-row constant.
// The rel index runs p(i)-j down a contiguous window of the table when no clamping occurs.
// Mask evaluation is skipped on tiles the mask covers fully.  Every wait is bounded; a
// timeout sets HSTU_DEV_WAIT_TIMEOUT and the CTA unwinds.
#include <cudaTypedefs.h>

#include <cstring>

#include "bias.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hstu {

using namespace sm100;

namespace {

constexpr int BM = 128, BN = 128, HALF = kHalf;
constexpr int kTcThreads = 384;
constexpr int kRelSmemMax = 4096;
constexpr uint32_t kTmemCols = 512;
constexpr int kBlockBytes = 128 * 128;   // one 128-row x 64-element bf16 swizzle block
constexpr uint32_t kOCol = 256;          // TMEM column of the output accumulator

enum Bar { Q_FULL = 0, KV_FULL = 1, KV_EMPTY = 3, S_FULL = 5, S_FREE = 7, P_FULL = 9,
           META_FULL = 11, O_FULL = 13, MMA_DONE = 14, NUM_BARS = 15 };

struct TileMeta {
    int64_t tmin[2], tmax[2];   // timestamp range of each 64-key half (valid keys only)
    int32_t ok32[2];            // the half's range is below 2^31 - 1: 32-bit relative stamps valid
    int32_t pad[2];
};

template <int DQK, int DV>
struct FwdLayout {
    static constexpr int QB = BM * DQK * 2;
    static constexpr int KB = BN * DQK * 2;
    static constexpr int VB = BN * DV * 2;
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + QB;
    static constexpr int V_OFF = K_OFF + 2 * KB;
    static constexpr int BAR_OFF = V_OFF + 2 * VB;
    static constexpr int SLOT_OFF = BAR_OFF + 8 * 16;
    static constexpr int META_OFF = SLOT_OFF + 16;
    static constexpr int TSK_OFF = META_OFF + 2 * (int)sizeof(TileMeta);
    static constexpr int TSK32_OFF = TSK_OFF + 2 * BN * 8;
    static constexpr int LUT_OFF = TSK32_OFF + 2 * BN * 4;
    static constexpr int THR_OFF = LUT_OFF + kLutCells * 8;
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

__device__ __forceinline__ void report_timeout(const DevParams &p)
{
    flag_error(p, HSTU_DEV_WAIT_TIMEOUT);
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// SPLIT: A enters A V as a pair of bf16 values, hi = bf16(A) and lo = bf16(A - hi), so Y
// carries about 16 significant bits (used when Y is saved for the backward, whose
// LayerNorm gradient is sensitive to the error of Y).
template <int DQK, int DV, bool SPLIT>
__global__ void __launch_bounds__(kTcThreads, 1)
    fwd_tc_kernel(const __grid_constant__ FwdTcArgs args)
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
    TileMeta *meta = reinterpret_cast<TileMeta *>(sm + L::META_OFF);
    int64_t *tsk = reinterpret_cast<int64_t *>(sm + L::TSK_OFF);
    int32_t *tsk32 = reinterpret_cast<int32_t *>(sm + L::TSK32_OFF);
    LutEntry *lutp = reinterpret_cast<LutEntry *>(sm + L::LUT_OFF);
    int32_t *lut_valid = reinterpret_cast<int32_t *>(sm + L::SLOT_OFF + 4);
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
            mbar_init(&bars[S_FREE + x], 1);
            mbar_init(&bars[P_FULL + x], 256);
            mbar_init(&bars[META_FULL + x], 32);
        }
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
    if (threadIdx.x == 0) *lut_valid = 1;
    __syncthreads();
    if (p.NB > 0) build_lut(thr, p.n_thr, lutp, lut_valid);
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
            // loads issued must land before the CTA exits (bounded)
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
            bool ok = mbar_wait(&bars[Q_FULL], 0);
            tc_fence_after();
            auto issue_pv = [&](int x) -> bool {
                const int sx = x & 1;
                if (!mbar_wait(&bars[P_FULL + sx], (x >> 1) & 1)) return false;
                tc_fence_after();
                const uint32_t v_addr = sm_base + L::V_OFF + sx * L::VB;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    // keys 16kk..16kk+15.  Packed A of half h (keys 64h..64h+63) lives in that
                    // half's S columns: without SPLIT at [64h, 64h+32); with SPLIT each 32-key
                    // chunk c holds hi at [64h+32c, +16) and lo at [64h+32c+16, +16)
                    const uint32_t a_tmem =
                        SPLIT ? tmem + sx * 128 + (kk >> 2) * 64 + ((kk >> 1) & 1) * 32 + (kk & 1) * 8
                              : tmem + sx * 128 + (kk >> 2) * 64 + (kk & 3) * 8;
                    const uint64_t bd = sw128_desc(v_addr + kk * 2048, kBlockBytes, 1024);
                    umma_bf16_ts(tmem + kOCol, a_tmem, bd, idesc_pv, (x > 0 || kk > 0) ? 1u : 0u);
                    if (SPLIT) umma_bf16_ts(tmem + kOCol, a_tmem + 16, bd, idesc_pv, 1u);
                }
                umma_commit(&bars[S_FREE + sx]);
                umma_commit(&bars[KV_EMPTY + sx]);
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
#pragma unroll
                for (int kb = 0; kb < DQK / 64; ++kb)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t a = sw128_desc(q_addr + kb * kBlockBytes + ks * 32, 16, 1024);
                        const uint64_t bd = sw128_desc(k_addr + kb * kBlockBytes + ks * 32, 16, 1024);
                        umma_bf16_ss(tmem + st * 128, a, bd, idesc_qk, (kb | ks) ? 1u : 0u);
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
    } else if (warp == 3) {
        // -------------------------------------------------------------------- tile metadata
        const bool use_ts = p.NB > 0;
        TileIter t(s, i0, p.W);
        int it = 0;
        while (t.next()) {
            const int st = it & 1;
            if (it >= 2 && !warp_wait(&bars[S_FREE + st], ((it >> 1) - 1) & 1)) {
                report_timeout(p);
                break;
            }
            if (use_ts) {
                const int j0 = t.kt * BN;
                int64_t v[4];
                int64_t mn[2] = {INT64_MAX, INT64_MAX}, mx[2] = {INT64_MIN, INT64_MIN};
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int c = lane + 32 * q4;
                    const int j = j0 + c;
                    v[q4] = 0;
                    if (j < s.L) {
                        v[q4] = p.ts[s.start + clamp_pos(j, s.E)];
                        mn[q4 >> 1] = min(mn[q4 >> 1], v[q4]);
                        mx[q4 >> 1] = max(mx[q4 >> 1], v[q4]);
                    }
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        mn[hh] = min(mn[hh], shfl_xor_i64(mn[hh], o));
                        mx[hh] = max(mx[hh], shfl_xor_i64(mx[hh], o));
                    }
                }
                int ok32[2];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    ok32[hh] = mn[hh] > mx[hh] ||
                               (uint64_t)mx[hh] - (uint64_t)mn[hh] < (uint64_t)INT32_MAX;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int c = lane + 32 * q4, hh = q4 >> 1;
                    tsk[st * BN + c] = v[q4];
                    // stamps relative to the half's minimum (0 for keys past the sequence)
                    const int j = j0 + c;
                    tsk32[st * BN + c] =
                        (j < s.L && ok32[hh]) ? (int32_t)((uint64_t)v[q4] - (uint64_t)mn[hh]) : 0;
                }
                if (lane == 0) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        meta[st].tmin[hh] = mn[hh];
                        meta[st].tmax[hh] = mx[hh];
                        meta[st].ok32[hh] = ok32[hh];
                    }
                }
            }
            __syncwarp();
            mbar_arrive(&bars[META_FULL + st]);
            ++it;
        }
    } else if (warp >= 4) {
        // -------------------------------------------------------------------- epilogue
        const int wg = (warp - 4) >> 2;               // 0: keys 0..63, 1: keys 64..127
        const int r = (warp & 3) * 32 + lane;         // query row in the tile == TMEM lane
        const int i = i0 + r;
        const bool row_in = i < s.L;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const int pi = clamp_pos(i, s.E);
        const bool use_ts = p.NB > 0;
        const bool use_rel = p.R > 0;
        const int64_t tsi = (use_ts && row_in) ? p.ts[s.start + pi] : 0;
        const float *relp = rel_in_smem ? rels : p.rel;
        const float half_alpha = 0.5f * p.alpha;
        const bool lut_ok = *lut_valid != 0;
        bool ok = true;
        TileIter t(s, i0, p.W);
        int it = 0;
        while (t.next()) {
            const int st = it & 1;
            const int jh = t.kt * BN + wg * HALF;     // first key of this warpgroup's half
            const bool full = tile_all_valid(i0, i0 + BM - 1, jh, jh + HALF - 1, s, p.W);
            if (!warp_wait(&bars[META_FULL + st], (it >> 1) & 1) ||
                !warp_wait(&bars[S_FULL + st], (it >> 1) & 1)) {
                ok = false;
                break;
            }

            // ---- per (row, half tile) structure; path choices are made warp-uniform
            const uint64_t vmask = full ? ~0ull : row_valid_bits(i, jh, s, p.W);
            const int rbase = pi - jh;                // rel index of key jh + c is rbase - c
            const bool rdirect = __all_sync(0xffffffffu, !use_rel || (rbase - (HALF - 1) >= 0 &&
                                                                        rbase <= p.R - 1));
            // time bias: tmode 0 = per-row constant, 1 = one bucket boundary (compare in
            // 32-bit relative stamps), 2 = exact lookup table, 3 = 64-bit search
            int tmode = 0;
            float tb_lo = 0.f, tb_hi = 0.f;
            int32_t cmpA = INT32_MIN, cmpB = INT32_MAX, tsi_rel = 0;
            int blo = 0, bhi = 0;
            bool lane_const = true;
            if (use_ts) {
                const int64_t hmin = meta[st].tmin[wg], hmax = meta[st].tmax[wg];
                const bool h32 = meta[st].ok32[wg] != 0;
                int my_mode = 0;
                if (row_in && hmin <= hmax) {
                    uint64_t dlo, dhi;
                    if (tsi >= hmax) {
                        dlo = (uint64_t)tsi - (uint64_t)hmax;
                        dhi = (uint64_t)tsi - (uint64_t)hmin;
                    } else if (tsi <= hmin) {
                        dlo = (uint64_t)hmin - (uint64_t)tsi;
                        dhi = (uint64_t)hmax - (uint64_t)tsi;
                    } else {
                        dlo = 0;
                        const uint64_t a = (uint64_t)tsi - (uint64_t)hmin;
                        const uint64_t c = (uint64_t)hmax - (uint64_t)tsi;
                        dhi = a > c ? a : c;
                    }
                    blo = bucket_in(thr, 0, p.n_thr, dlo);
                    bhi = bucket_in(thr, blo, p.n_thr, dhi);
                    const bool fits = h32 && dhi < (uint64_t)(INT32_MAX - 1);
                    if (fits) tsi_rel = (int32_t)((uint64_t)tsi - (uint64_t)hmin);
                    if (bhi == blo) {
                        my_mode = 0;
                    } else if (bhi == blo + 1 && fits) {
                        my_mode = 1;
                        // |tsi - tsj| >= T  <=>  tsj <= tsi - T  or  tsj >= tsi + T
                        const int64_t T = (int64_t)thr[blo];
                        const int64_t A = (int64_t)tsi_rel - T, B = (int64_t)tsi_rel + T;
                        cmpA = (int32_t)max((int64_t)INT32_MIN, min((int64_t)INT32_MAX, A));
                        cmpB = (int32_t)max((int64_t)INT32_MIN, min((int64_t)INT32_MAX, B));
                    } else {
                        my_mode = (fits && lut_ok) ? 2 : 3;
                    }
                }
                lane_const = my_mode == 0;
                tmode = __reduce_max_sync(0xffffffffu, my_mode);
                tb_lo = tbs[blo];
                tb_hi = tbs[min(blo + 1, p.NB - 1)];
            }
            const int32_t *tk32 = tsk32 + st * BN + wg * HALF;
            const int64_t *tk64 = tsk + st * BN + wg * HALF;

            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < 2; ++ch) {
                const uint32_t s_col = tmem + lane_base + st * 128 + wg * HALF + ch * 32;
                uint32_t ra[32];
                tmem_ld32(s_col, ra);
                tmem_wait_ld();
                reg_fence(ra);
                const uint32_t vbits = (uint32_t)(vmask >> (32 * ch));
                const int cb = ch * 32;
                float av[32];
                // bias: rel part
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    float bias = 0.f;
                    if (use_rel) {
                        if (rdirect) {
                            bias = relp[rbase - cb - c];
                        } else {
                            int ri = rbase - cb - c;
                            ri = ri < 0 ? 0 : (ri > p.R - 1 ? p.R - 1 : ri);
                            bias = relp[ri];
                        }
                    }
                    av[c] = bias;
                }
                // bias: time part
                if (tmode == 0) {
#pragma unroll
                    for (int c = 0; c < 32; ++c) av[c] += tb_lo;
                } else if (tmode == 1) {
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int32_t tj = tk32[cb + c];
                        av[c] += (tj <= cmpA || tj >= cmpB) ? tb_hi : tb_lo;
                    }
                } else if (tmode == 2) {
                    const LutEntry *lut = reinterpret_cast<const LutEntry *>(lutp);
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        int32_t d = tsi_rel - tk32[cb + c];
                        uint32_t dt = (uint32_t)(d < 0 ? -d : d);
                        dt = min(dt, (uint32_t)INT32_MAX - 1u);
                        const LutEntry e = lut[lut_cell(dt)];
                        const float v = tbs[e.base + (dt >= e.next ? e.jump : 0)];
                        av[c] += lane_const ? tb_lo : v;
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        av[c] += tbs[bucket_search(thr, p.n_thr, abs_diff_u64(tsi, tk64[cb + c]))];
                }
                // SiLU(x) = x sigmoid(x) = h + h tanh(h), h = x/2; mask after the nonlinearity
                uint32_t pk[16];
                float a_full[32];
#pragma unroll
                for (int c2 = 0; c2 < 16; ++c2) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int c = 2 * c2 + e;
                        float a;
                        if (SPLIT) {   // accurate sigmoid for the training forward
                            const float xs = fmaf(p.alpha, __uint_as_float(ra[c]), av[c]);
                            a = xs * __fdividef(1.0f, 1.0f + __expf(-xs));
                        } else {
                            const float hx = fmaf(half_alpha, __uint_as_float(ra[c]), 0.5f * av[c]);
                            a = fmaf(hx, tanh_approx(hx), hx);
                        }
                        a_full[c] = full ? a : (((vbits >> c) & 1u) ? a : 0.f);
                    }
                    pk[c2] = pack_bf16x2(a_full[2 * c2], a_full[2 * c2 + 1]);
                }
                // bf16 A written back over S columns this thread has already read
                if (SPLIT) {
                    uint32_t plo[16];
#pragma unroll
                    for (int c2 = 0; c2 < 16; ++c2) {
                        const float h0 = __uint_as_float(pk[c2] << 16);
                        const float h1 = __uint_as_float(pk[c2] & 0xFFFF0000u);
                        plo[c2] = pack_bf16x2(a_full[2 * c2] - h0, a_full[2 * c2 + 1] - h1);
                    }
                    tmem_st16(tmem + lane_base + st * 128 + wg * HALF + ch * 32, pk);
                    tmem_st16(tmem + lane_base + st * 128 + wg * HALF + ch * 32 + 16, plo);
                } else {
                    tmem_st16(tmem + lane_base + st * 128 + wg * HALF + ch * 16, pk);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[P_FULL + st]);
            ++it;
        }
        if (ok && !warp_wait(&bars[O_FULL], 0)) ok = false;
        if (ok) {
            tc_fence_after();
            float *yr = args.y + (s.start + i) * (int64_t)p.D + h * DV;
#pragma unroll 1
            for (int c = wg * (DV / 64); c < (wg + 1) * (DV / 64); ++c) {
                uint32_t ra[32];
                tmem_ld32(tmem + lane_base + kOCol + c * 32, ra);
                tmem_wait_ld();
                reg_fence(ra);
                if (row_in) {
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

template <int DQK, int DV>
cudaError_t launch_tc(const FwdTcArgs &a, bool split, cudaStream_t st)
{
    using L = FwdLayout<DQK, DV>;
    auto kern = split ? fwd_tc_kernel<DQK, DV, true> : fwd_tc_kernel<DQK, DV, false>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    dim3 grid((a.p.N + BM - 1) / BM, a.p.B, a.p.H);
    kern<<<grid, kTcThreads, L::ALLOC, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

static PFN_cuTensorMapEncodeTiled_v12000 tmap_encode_fn()
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
bool encode_tmap_bf16(CUtensorMap *m, const void *base, int d, int H, int64_t T)
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

bool tc_fwd_supported(int dqk, int dv, int64_t T)
{
    return (dqk == 64 || dqk == 128) && (dv == 64 || dv == 128) && T < ((int64_t)1 << 31);
}

cudaError_t launch_tc_fwd(const DevParams &p, const void *q, const void *k, const void *v,
                          float *y, bool training, cudaStream_t st)
{
    FwdTcArgs a;
    std::memset(&a, 0, sizeof(a));
    a.p = p;
    a.y = y;
    if (!encode_tmap_bf16(&a.tq, q, p.dqk, p.H, p.T) || !encode_tmap_bf16(&a.tk, k, p.dqk, p.H, p.T) ||
        !encode_tmap_bf16(&a.tv, v, p.dv, p.H, p.T))
        return cudaErrorInvalidValue;
    if (p.dqk == 128 && p.dv == 128) return launch_tc<128, 128>(a, training, st);
    if (p.dqk == 128 && p.dv == 64) return launch_tc<128, 64>(a, training, st);
    if (p.dqk == 64 && p.dv == 128) return launch_tc<64, 128>(a, training, st);
    if (p.dqk == 64 && p.dv == 64) return launch_tc<64, 64>(a, training, st);
    return cudaErrorInvalidValue;
}

}  // namespace hstu
