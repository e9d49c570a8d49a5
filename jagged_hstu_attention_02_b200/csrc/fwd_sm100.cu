// fwd_sm100.cu -- tensor-core (tcgen05) forward attention of jagged HSTU for B200.
//
// A work unit is (128-row query tile, sequence, head).  For every key tile of 128 that holds
// a valid pair:  S = Q K^T on tcgen05 (bf16 operands staged by TMA in 128-byte-swizzled
// shared memory, fp32 accumulator in TMEM); the epilogue warps read S from TMEM and form
// A = mask ? SiLU(alpha*S + b) : 0, where b is the relative-position plus bucketed time
// bias and the mask is applied after the nonlinearity, never as -inf before it ("HSTU
// tensor by tensor: SiLU aggregation, temporal bias and gating", sections "Similar shape,
// different aggregation" and "Do not copy softmax masking mechanically") -- in packed bf16
// pairs for inference, in fp32 with A split into bf16 hi + lo parts for training; A goes
// into its own TMEM columns (two bf16 elements per 32-bit column), and tcgen05 adds A V
// into an fp32 output accumulator in TMEM with A read from TMEM.  The 1/N scale
// ("HSTU-MUSA: HSTU for Moore Threads (MUSA)", "Accuracy Alignment": N = batch max_seqlen)
// is applied once to the accumulator; Y goes to global memory in fp32.
//
// Persistent: one CTA per SM takes units from a global counter in longest-first order
// (query tiles from the last to the first, so the tiles with the most keys start first;
// units.cuh), so the per-CTA set-up (barriers, TMEM, bias tables, bucket lookup table)
// happens once per SM and the loads of the next unit (Q is double-buffered) overlap the
// tail of the current one.  Warp roles (20
// warps): warp 0 lane 0 loads Q and K, warp 2 lane 0 loads V (warp 2 also owns TMEM), warp
// 1 lane 0 issues the MMAs, warp 3 stages each key tile's timestamps and per-quarter
// ranges, warps 4-19 are four epilogue warpgroups, each owning 32 of the 128 key columns
// of every query row (thread = row = TMEM lane).  TMEM: S double-buffered [0,256), A in
// its own columns [256,384) so S is released as soon as the epilogue has read it, output
// accumulator [384,512).
//
// Bias evaluation per (row, 32-key quarter tile):  the time bucket is computed once for
// the smallest and largest |dt| the quarter can produce (from its timestamp range); when
// both agree (the common case away from the diagonal) the time bias is a per-row constant.
// The rel index runs p(i)-j down a contiguous window of the table when no clamping occurs
// (inference: a guard-banded table of bf16 key pairs, one load per two keys).  Blocks
// without a valid pair only write zeros; the training body skips the mask on fully valid
// blocks, the inference body always applies it (one byte permute per key pair).  Every
// wait is bounded; a timeout sets HSTU_DEV_WAIT_TIMEOUT and the CTA unwinds.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>

#include "kernels.h"
#include "sm100.cuh"
#include "tiles.cuh"
#include "units.cuh"

namespace hstu {

using namespace sm100;

namespace {

constexpr int BM = 128, BN = 128, QW = 32;   // QW: key columns per epilogue warpgroup
static_assert(BM == kTile && BN == kTile && QW == kBlk, "tile shapes of tiles.cuh");
constexpr int kEpiWarps = 16;                  // four warpgroups
constexpr int kTcThreads = 128 + 32 * kEpiWarps;
constexpr int kRelSmemMax = 4352;   // words of the shared rel table region
// Inference: the rel table is held as bf16 key pairs with kRelGuard entries on both sides
// (see fwd_quarter_inf); it fits in shared memory for R up to kRelSmemMax - 2 kRelGuard.
constexpr int kRelGuard = 32;
constexpr int kRelPairMax = kRelSmemMax - 2 * kRelGuard;
constexpr uint32_t kTmemCols = 512;
constexpr int kBlockBytes = 128 * 128;   // one 128-row x 64-element bf16 swizzle block
constexpr uint32_t kPCol = 256;          // TMEM columns of A (packed bf16)
constexpr uint32_t kOCol = 384;          // TMEM columns of the output accumulator
constexpr int KST = 2, VST = 2, QST = 2; // K, V and Q stages

enum Bar { Q_FULL = 0, Q_EMPTY = 2, K_FULL = 4, K_EMPTY = 6, V_FULL = 8, V_EMPTY = 10,
           S_FULL = 12, S_FREE = 14, P_FULL = 16, P_FREE = 18, META_FULL = 20, EPI_DONE = 22,
           O_FULL = 24, O_FREE = 25, MMA_DONE = 26, UNIT_FULL = 27, UNIT_EMPTY = 31,  // +4
           NEVER = 35,   // nothing arrives on it (the stall test's wait)
           NUM_BARS = 36 };
static_assert(NUM_BARS <= 40, "barrier area");

struct TileMeta {
    int64_t tmin[4], tmax[4];   // timestamp range of each 32-key quarter (valid keys only)
    int32_t ok32[4];            // the quarter's range is below 2^31 - 1: 32-bit stamps valid
};

template <int DQK, int DV>
struct FwdLayout {
    static constexpr int QB = BM * DQK * 2;
    static constexpr int KB = BN * DQK * 2;
    static constexpr int VB = BN * DV * 2;
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + QST * QB;
    static constexpr int V_OFF = K_OFF + KST * KB;
    static constexpr int BAR_OFF = V_OFF + VST * VB;
    static constexpr int SLOT_OFF = BAR_OFF + 8 * 40;
    static constexpr int UNIT_OFF = SLOT_OFF + 16;                 // kUnitRing unit slots
    static constexpr int META_OFF = UNIT_OFF + (int)sizeof(UnitSlot) * kUnitRing;
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
    unsigned long long *unit_ctr;   // next work unit to hand out (zeroed by the caller)
    int nqt;   // query tiles of the longest admissible sequence: ceil(N / 128)
};

__device__ __forceinline__ void report_timeout(const DevParams &p)
{
    flag_error(p, HSTU_DEV_WAIT_TIMEOUT);
}


// SPLIT: A enters A V as a pair of bf16 values, hi = bf16(A) and lo = bf16(A - hi), so Y
// carries about 16 significant bits (used when Y is saved for the backward, whose
// LayerNorm gradient is sensitive to the error of Y).  Without SPLIT, A has two TMEM
// buffers of 64 columns; with SPLIT one buffer of 128 (per 32-key quarter w: hi at
// 32w..32w+15, lo at 32w+16..32w+31).
// Training: one 32-row x 32-key block of the epilogue (thread = row = TMEM lane): the bias,
// SiLU, the mask, and A (hi and lo parts) into TMEM, in fp32 with the accurate sigmoid.
// The inference body is fwd_quarter_inf.  The mode choices are template parameters, so the body has no
// branch and the compiler can overlap the loads and arithmetic of neighbouring keys:
//   TM   time bias: 0 one bucket, 1 one boundary, 2 lookup table, 3 64-bit search
//   RD   rel index rbase - c without clamping
//   FULL every pair of the block is valid (no mask)
struct FwdEpi {
    uint32_t t_s;              // TMEM address of the block's S columns
    uint32_t t_a;              // TMEM address of the block's A columns
    const int32_t *tk32;       // key stamps relative to the quarter's minimum
    const int64_t *tk64;       // and absolute
    const float *relp;         // rel table (relp * rel_sc = half bias)
    float rel_sc;
    const uint32_t *relp2;     // inference: bf16 pair table, relp2[x] = {rel[x], rel[x-1]} / 2
    const float *relg;         // inference, clamped blocks: the fp32 table (R >= 1 entries)
    int rbase, R;              // rel index of key c: rbase - c (clamped unless RD)
    int cand0, rcand;          // clamped blocks: keys c >= cand0 are candidates, p(i) - p(j) = rcand
    bool rabs;                 // rel index min(|p(i) - p(j)|, R-1) (mask variant)
    float half_alpha, alpha;
    const float *tbh;          // half time-bias table
    const LutEntry *lut;
    const uint64_t *thr;
    int n_thr;
    int64_t tsi;               // the row's stamp
};

template <int TM, bool RD, bool FULL>
__device__ __forceinline__ void fwd_quarter(const FwdEpi &e, const HalfTime &ht, uint32_t vmask)
{
    // one-boundary test as a single unsigned compare: the key is in the lower bucket when
    // cmpA < t < cmpB
    const uint32_t a1 = (uint32_t)ht.cmpA + 1u;
    const int64_t sp = (int64_t)ht.cmpB - (int64_t)ht.cmpA - 1;
    const uint32_t span = sp > 0 ? (uint32_t)sp : 0u;
    const float2 ha2 = make_float2(e.half_alpha, e.half_alpha);
    const float2 rs2 = make_float2(e.rel_sc, e.rel_sc);
#pragma unroll 1   // one copy of the 4-key body per mode combination (instruction cache)
    for (int ch = 0; ch < 8; ++ch) {
        const int cb = ch * 4;
        uint32_t ra[4];
        tmem_ld4(e.t_s + cb, ra);
        float tb[4], rv[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (TM == 0) {
                tb[c] = ht.tb_lo;
            } else if (TM == 1) {
                const bool lo = (uint32_t)e.tk32[cb + c] - a1 < span;
                tb[c] = lo ? ht.tb_lo : ht.tb_hi;
            } else if (TM == 2) {
                const int32_t d = ht.t_rel - e.tk32[cb + c];
                uint32_t dt = (uint32_t)(d < 0 ? -d : d);
                dt = min(dt, (uint32_t)INT32_MAX - 1u);
                const float v = e.tbh[lut_bucket(e.lut, dt)];
                tb[c] = ht.lane_const ? ht.tb_lo : v;
            } else {
                tb[c] = e.tbh[bucket_search(e.thr, e.n_thr, abs_diff_u64(e.tsi, e.tk64[cb + c]))];
            }
            int ri = e.rbase - cb - c;
            if (!RD) ri = rel_index(cb + c < e.cand0 ? ri : e.rcand, e.R, e.rabs);
            rv[c] = e.relp[ri];
        }
        float2 bh[2];
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2)
            bh[c2] = __ffma2_rn(make_float2(rv[2 * c2], rv[2 * c2 + 1]), rs2,
                                make_float2(tb[2 * c2], tb[2 * c2 + 1]));
        tmem_wait_ld();
        reg_fence(ra);
        const uint32_t vb = vmask >> cb;
        uint32_t pk[2], plo[2];
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
            const float2 h = __ffma2_rn(ha2, make_float2(__uint_as_float(ra[2 * c2]),
                                                         __uint_as_float(ra[2 * c2 + 1])),
                                        bh[c2]);
            float a[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int c = 2 * c2 + q;
                const float xs = 2.0f * (q ? h.y : h.x);
                const float v = xs * __fdividef(1.0f, 1.0f + __expf(-xs));
                a[q] = (FULL || ((vb >> c) & 1u)) ? v : 0.f;
            }
            pk[c2] = pack_bf16x2(a[0], a[1]);
            plo[c2] = pack_bf16x2(a[0] - __uint_as_float(pk[c2] << 16),
                                  a[1] - __uint_as_float(pk[c2] & 0xFFFF0000u));
        }
        tmem_st2(e.t_a + ch * 2, pk);
        tmem_st2(e.t_a + 16 + ch * 2, plo);
    }
}

// Byte permute of x with sign replication: selector nibble 8 + k gives byte k's top bit
// repeated over a byte (0x9988: bytes 0 and 1 to halves 0 and 1; 0xBBAA: bytes 2 and 3).
__device__ __forceinline__ uint32_t sign_bytes(uint32_t x, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(d) : "r"(x), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t add_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Inference: 8 keys (cb .. cb+7) of one row in packed bf16 pairs (key c in the low half,
// c + 1 in the high half).  With the half bias b/2 and h = (alpha s + b) / 2:
// SiLU(2h) / 2 = h + h tanh(h), computed as fma(h, tanh(h), h); every conversion rounds to
// nearest even.  s holds the 8 keys' scores (fp32 bits), a receives the 4 A columns.
template <int TM, bool RD, bool FULL>
__device__ __forceinline__ void inf_chunk(const FwdEpi &e, const HalfTime &ht, uint32_t vmask,
                                          int cb, const uint32_t (&s)[8], uint32_t ha2,
                                          uint32_t tlo2, uint32_t thi2, uint32_t a1,
                                          uint32_t span, uint32_t (&a)[4])
{
    // the 8 keys' stamps (relative to the quarter's minimum) in two 16-byte loads
    int32_t tk[8];
    if (TM == 1 || TM == 2) {
        const int4 x0 = *reinterpret_cast<const int4 *>(e.tk32 + cb);
        const int4 x1 = *reinterpret_cast<const int4 *>(e.tk32 + cb + 4);
        tk[0] = x0.x; tk[1] = x0.y; tk[2] = x0.z; tk[3] = x0.w;
        tk[4] = x1.x; tk[5] = x1.y; tk[6] = x1.z; tk[7] = x1.w;
    }
    // the keys' valid bits moved to the sign bits of bytes: key 4h + b -> bit 7 of byte b of
    // z[h] (a multiply by 2^7 + 2^14 + 2^21 + 2^28 places non-overlapping copies of the 4
    // bits), so that one byte permute with sign replication gives a pair's half masks
    uint32_t z[2] = {0u, 0u};
    if (!FULL) {
        const uint32_t v8 = vmask >> cb;
        z[0] = (v8 & 0xFu) * 0x10204080u;
        z[1] = ((v8 >> 4) & 0xFu) * 0x10204080u;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int c = cb + 2 * q;
        uint32_t r2;
        if (RD) {
            r2 = e.relp2[e.rbase - c];           // guard-banded: no clamp needed here
        } else {
            // the key's own position p(j): candidate keys take the last history position
            const int x0 = rel_index(c < e.cand0 ? e.rbase - c : e.rcand, e.R, e.rabs);
            const int x1 = rel_index(c + 1 < e.cand0 ? e.rbase - c - 1 : e.rcand, e.R, e.rabs);
            r2 = pack_bf16x2(0.5f * e.relg[x0], 0.5f * e.relg[x1]);
        }
        uint32_t t2;
        if (TM == 0) {
            t2 = tlo2;
        } else if (TM == 1) {
            const bool h0 = (uint32_t)tk[2 * q] - a1 >= span;
            const bool h1 = (uint32_t)tk[2 * q + 1] - a1 >= span;
            t2 = ((h0 ? thi2 : tlo2) & 0x0000FFFFu) | ((h1 ? thi2 : tlo2) & 0xFFFF0000u);
        } else if (TM == 2) {
            float v[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int32_t d = ht.t_rel - tk[2 * q + k];
                uint32_t dt = (uint32_t)(d < 0 ? -d : d);
                dt = min(dt, (uint32_t)INT32_MAX - 1u);
                const float tv = e.tbh[lut_bucket(e.lut, dt)];
                v[k] = ht.lane_const ? ht.tb_lo : tv;
            }
            t2 = pack_bf16x2(v[0], v[1]);
        } else {
            t2 = pack_bf16x2(e.tbh[bucket_search(e.thr, e.n_thr, abs_diff_u64(e.tsi, e.tk64[c]))],
                             e.tbh[bucket_search(e.thr, e.n_thr,
                                                 abs_diff_u64(e.tsi, e.tk64[c + 1]))]);
        }
        const uint32_t s2 = pack_bf16x2(__uint_as_float(s[2 * q]), __uint_as_float(s[2 * q + 1]));
        const uint32_t h2 = add_bf16x2(fma_bf16x2(ha2, s2, r2), t2);
        uint32_t a2 = fma_bf16x2(h2, tanh_bf16x2(h2), h2);
        if (!FULL) a2 &= sign_bytes(z[q >> 1], (q & 1) ? 0xBBAAu : 0x9988u);
        a[q] = a2;
    }
}

// Inference: one 32-row x 32-key block (thread = row = TMEM lane), 8 keys per loop turn.
// The loop is kept rolled: with a dozen of these bodies in the kernel, the instruction
// cache, not load latency, limits the epilogue (unrolled or software-pipelined forms
// measured 6-25 % slower on the long-history and windowed workloads).
//   RD  the rel index rbase - c of every key lies within the guard-banded pair table:
//       relp2[rbase - c] holds the biases of keys c and c + 1 (clamped entries in the
//       guard bands), one shared load for two keys;
//   otherwise each key's clamped index is read from the fp32 table.
template <int TM, bool RD, bool FULL>
__device__ __forceinline__ void fwd_quarter_inf(const FwdEpi &e, const HalfTime &ht,
                                                uint32_t vmask)
{
    const uint32_t ha2 = pack_bf16x2(e.half_alpha, e.half_alpha);
    const uint32_t tlo2 = pack_bf16x2(ht.tb_lo, ht.tb_lo);
    const uint32_t thi2 = pack_bf16x2(ht.tb_hi, ht.tb_hi);
    // one-boundary test as a single unsigned compare (see fwd_quarter)
    const uint32_t a1 = (uint32_t)ht.cmpA + 1u;
    const int64_t sp = (int64_t)ht.cmpB - (int64_t)ht.cmpA - 1;
    const uint32_t span = sp > 0 ? (uint32_t)sp : 0u;
    uint32_t s0[8], a[4];
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
        tmem_ld8(e.t_s + ch * 8, s0);
        tmem_wait_ld();
        reg_fence(s0);
        inf_chunk<TM, RD, FULL>(e, ht, vmask, ch * 8, s0, ha2, tlo2, thi2, a1, span, a);
        tmem_st4(e.t_a + ch * 4, a);
    }
}

template <int DQK, int DV, bool SPLIT>
__global__ void __launch_bounds__(kTcThreads, 1)
    fwd_tc_kernel(const __grid_constant__ FwdTcArgs args)
{
    using L = FwdLayout<DQK, DV>;
    constexpr int NP = SPLIT ? 1 : 2;   // A buffers
    const DevParams &p = args.p;

    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, by an offset from the shared array (keeps the compiler aware
    // that every table below lives in shared memory: 32-bit addresses, shared loads)
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR_OFF);
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT_OFF);
    int32_t *lut_valid = reinterpret_cast<int32_t *>(sm + L::SLOT_OFF + 4);
    // Work units: query tiles from the last down (the longest rows first), sequence, head.
    const FeedRing ring{bars + UNIT_FULL, bars + UNIT_EMPTY,
                        reinterpret_cast<UnitSlot *>(sm + L::UNIT_OFF), args.unit_ctr};
    TileMeta *meta = reinterpret_cast<TileMeta *>(sm + L::META_OFF);
    int64_t *tsk = reinterpret_cast<int64_t *>(sm + L::TSK_OFF);
    int32_t *tsk32 = reinterpret_cast<int32_t *>(sm + L::TSK32_OFF);
    LutEntry *lutp = reinterpret_cast<LutEntry *>(sm + L::LUT_OFF);
    uint64_t *thr = reinterpret_cast<uint64_t *>(sm + L::THR_OFF);
    float *tbh = reinterpret_cast<float *>(sm + L::TB_OFF);    // scaled half time table
    float *relh = reinterpret_cast<float *>(sm + L::REL_OFF);  // scaled half rel table
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int x = 0; x < NUM_BARS; ++x) mbar_init(&bars[x], 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars[S_FREE + x], kEpiWarps);
            mbar_init(&bars[P_FULL + x], kEpiWarps);
            mbar_init(&bars[META_FULL + x], 32);
            mbar_init(&bars[EPI_DONE + x], kEpiWarps);
        }
        mbar_init(&bars[O_FREE], kEpiWarps);
        for (int x = 0; x < kUnitRing; ++x) mbar_init(&bars[UNIT_EMPTY + x], 3 + kEpiWarps);
        fence_mbar_init();
        *lut_valid = 1;
    }
    if (warp == 2) tmem_alloc(slot, kTmemCols);
    // Tables hold half the bias.  Training: the fp32 rel table.  Inference: bf16 key pairs,
    // entry x = {rel[c(x)], rel[c(x-1)]} / 2 for x in [-kRelGuard, R - 1 + kRelGuard], with
    // c() the clamp into [0, R-1] (zeros without a table).
    const float tscale = 0.5f;
    for (int x = threadIdx.x; x < p.n_thr; x += kTcThreads) thr[x] = p.thr[x];
    for (int x = threadIdx.x; x < p.NB; x += kTcThreads) tbh[x] = tscale * p.tb[x];
    const bool rel_in_smem = SPLIT ? p.R <= kRelSmemMax : p.R <= kRelPairMax;
    uint32_t *relp2 = reinterpret_cast<uint32_t *>(relh) + kRelGuard;
    if (rel_in_smem) {
        if (SPLIT) {
            for (int x = threadIdx.x; x < p.R; x += kTcThreads) relh[x] = tscale * p.rel[x];
        } else {
            const int Re = p.R > 0 ? p.R : 1;
            const bool rabs = (p.flags & HSTU_FLAG_REL_ABS) != 0;
            for (int x = threadIdx.x - kRelGuard; x < Re + kRelGuard; x += kTcThreads) {
                const int x0 = rel_index(x, Re, rabs), x1 = rel_index(x - 1, Re, rabs);
                relp2[x] = p.R > 0 ? pack_bf16x2(tscale * p.rel[x0], tscale * p.rel[x1]) : 0u;
            }
        }
    }
    if (p.R == 0 && threadIdx.x == 0 && SPLIT) relh[0] = 0.f;   // read, times zero bias
    fill_seq_tiles(p, kTcThreads);
    for (int b = blockIdx.x; b < p.B; b += gridDim.x) {   // rows no unit writes: zero Y
        RowRange rr[3];
        const int n = skipped_rows(p, b, rr);
        for (int x = 0; x < n; ++x) zero_rows(args.y, p.D, rr[x], threadIdx.x, kTcThreads);
    }
    __syncthreads();
    if (p.NB > 0) build_lut(thr, p.n_thr, lutp, lut_valid);
    grid_dep_release();   // the LayerNorm behind this kernel may be scheduled
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    const uint32_t sm_base = smem_u32(sm);

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- Q and K loads
            prefetch_tmap(&args.tq);
            prefetch_tmap(&args.tk);
            UnitFeed<FEED_PRODUCER, false, BM> un(p, ring, args.nqt);
            int n = 0, g = 0;
            bool ok = true;
            while (ok && un.next()) {
                const int i0 = un.tile * BM, row0 = (int)un.s.start, qs = n % QST;
                if (n >= QST && !mbar_wait(&bars[Q_EMPTY + qs], (n / QST - 1) & 1, p.wait_limit)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bars[Q_FULL + qs], L::QB);
                for (int kb = 0; kb < DQK / 64; ++kb)
                    tma_load_3d(sm + L::Q_OFF + qs * L::QB + kb * kBlockBytes, &args.tq,
                                &bars[Q_FULL + qs], kb * 64, un.h, row0 + i0);
                TileIter t(un.s, i0, p.W);
                while (t.next()) {
                    const int st = g % KST;
                    if (g >= KST && !mbar_wait(&bars[K_EMPTY + st], (g / KST - 1) & 1, p.wait_limit)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars[K_FULL + st], L::KB);
                    for (int kb = 0; kb < DQK / 64; ++kb)
                        tma_load_3d(sm + L::K_OFF + st * L::KB + kb * kBlockBytes, &args.tk,
                                    &bars[K_FULL + st], kb * 64, un.h, row0 + t.kt * BN);
                    ++g;
                }
                ++n;
            }
            if (!ok || !un.ok) report_timeout(p);
            // loads issued must land before the CTA exits (bounded)
            bool drained = true;
            for (int x = n - 1; x >= 0 && x >= n - QST; --x)
                drained &= mbar_wait(&bars[Q_FULL + x % QST], (x / QST) & 1, kWaitLimitCycles);
            for (int x = g - 1; x >= 0 && x >= g - KST; --x)
                drained &= mbar_wait(&bars[K_FULL + x % KST], (x / KST) & 1, kWaitLimitCycles);
            if (!drained) report_timeout(p);
        }
    } else if (warp == 2) {
        if (lane == 0) {
            // ---------------------------------------------------------------- V loads
            prefetch_tmap(&args.tv);
            UnitFeed<FEED_THREAD, false, BM> un(p, ring, args.nqt);
            int g = 0;
            bool ok = true;
            while (ok && un.next()) {
                const int row0 = (int)un.s.start;
                TileIter t(un.s, un.tile * BM, p.W);
                while (t.next()) {
                    const int st = g % VST;
                    if (g >= VST && !mbar_wait(&bars[V_EMPTY + st], (g / VST - 1) & 1, p.wait_limit)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars[V_FULL + st], L::VB);
                    for (int kb = 0; kb < DV / 64; ++kb)
                        tma_load_3d(sm + L::V_OFF + st * L::VB + kb * kBlockBytes, &args.tv,
                                    &bars[V_FULL + st], kb * 64, un.h, row0 + t.kt * BN);
                    ++g;
                }
            }
            if (!ok || !un.ok) report_timeout(p);
            bool drained = true;
            for (int x = g - 1; x >= 0 && x >= g - VST; --x)
                drained &= mbar_wait(&bars[V_FULL + x % VST], (x / VST) & 1, kWaitLimitCycles);
            if (!drained) report_timeout(p);
        }
    }
    else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            constexpr uint32_t idesc_qk = idesc_bf16(BM, BN, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16(BM, DV, false, true);
            const uint32_t o_tmem = tmem + kOCol;
            // A V for tile g of unit n; first/last tile of the unit
            auto issue_pv = [&](int g, int n, bool first, bool last) -> bool {
                const int ps = g % NP;
                if (!mbar_wait(&bars[P_FULL + ps], (g / NP) & 1, p.wait_limit)) return false;
                if (!mbar_wait(&bars[V_FULL + g % VST], (g / VST) & 1, p.wait_limit)) return false;
                if (first && n >= 1 && !mbar_wait(&bars[O_FREE], (n - 1) & 1, p.wait_limit)) return false;
                tc_fence_after();
                const uint32_t v_addr = sm_base + L::V_OFF + (g % VST) * L::VB;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    // keys 16kk..16kk+15; see the layout of A above
                    const uint32_t a_tmem =
                        SPLIT ? tmem + kPCol + (kk >> 1) * 32 + (kk & 1) * 8
                              : tmem + kPCol + ps * 64 + kk * 8;
                    const uint64_t bd = sw128_desc(v_addr + kk * 2048, kBlockBytes, 1024);
                    umma_bf16_ts(o_tmem, a_tmem, bd, idesc_pv, (!first || kk > 0) ? 1u : 0u);
                    if (SPLIT) umma_bf16_ts(o_tmem, a_tmem + 16, bd, idesc_pv, 1u);
                }
                umma_commit(&bars[P_FREE + ps]);
                umma_commit(&bars[V_EMPTY + g % VST]);
                if (last) umma_commit(&bars[O_FULL]);
                return true;
            };
            UnitFeed<FEED_THREAD, false, BM> un(p, ring, args.nqt);
            int n = 0, g = 0;
            // the stall test: a wait that runs out, then the same unwinding as any timeout
            bool ok = !p.stall_test || mbar_wait(&bars[NEVER], 0, p.wait_limit);
            bool pend = false;                  // an A V waiting for its A
            int pg = 0, pn = 0;
            bool pfirst = false;
            while (ok && un.next()) {
                const int qs = n % QST;
                if (!mbar_wait(&bars[Q_FULL + qs], (n / QST) & 1, p.wait_limit)) { ok = false; break; }
                tc_fence_after();
                const uint32_t q_addr = sm_base + L::Q_OFF + qs * L::QB;
                TileIter t(un.s, un.tile * BM, p.W);
                bool first = true, more = t.next();
                while (more) {
                    const int st = g & 1, ks = g % KST;
                    if (!mbar_wait(&bars[K_FULL + ks], (g / KST) & 1, p.wait_limit) ||
                        (g >= 2 && !mbar_wait(&bars[S_FREE + st], ((g >> 1) - 1) & 1, p.wait_limit))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t k_addr = sm_base + L::K_OFF + ks * L::KB;
#pragma unroll
                    for (int kb = 0; kb < DQK / 64; ++kb)
#pragma unroll
                        for (int kq = 0; kq < 4; ++kq) {
                            const uint64_t a = sw128_desc(q_addr + kb * kBlockBytes + kq * 32, 16, 1024);
                            const uint64_t bd = sw128_desc(k_addr + kb * kBlockBytes + kq * 32, 16, 1024);
                            umma_bf16_ss(tmem + st * 128, a, bd, idesc_qk, (kb | kq) ? 1u : 0u);
                        }
                    umma_commit(&bars[S_FULL + st]);
                    umma_commit(&bars[K_EMPTY + ks]);
                    more = t.next();
                    if (!more) umma_commit(&bars[Q_EMPTY + qs]);   // Q free after its last QK^T
                    // the previous tile's A V (possibly of the previous unit, which it closes)
                    if (pend && !issue_pv(pg, pn, pfirst, pn != n)) { ok = false; break; }
                    pend = true;
                    pg = g;
                    pn = n;
                    pfirst = first;
                    first = false;
                    ++g;
                }
                ++n;
            }
            if (ok && pend) ok = issue_pv(pg, pn, pfirst, true);
            if (!ok || !un.ok) report_timeout(p);
            // every MMA issued must complete before TMEM is released (bounded)
            umma_commit(&bars[MMA_DONE]);
            if (!mbar_wait(&bars[MMA_DONE], 0, kWaitLimitCycles)) report_timeout(p);
        }
    } else if (warp == 3) {
        // -------------------------------------------------------------------- tile metadata
        const bool use_ts = p.NB > 0;
        UnitFeed<FEED_WARP, false, BM> un(p, ring, args.nqt);
        int g = 0;
        bool ok = true;
        while (ok && un.next()) {
            const SeqInfo &s = un.s;
            TileIter t(s, un.tile * BM, p.W);
            while (t.next()) {
                const int st = g & 1;
                // the epilogue is done with this stage's stamps (tile g - 2)
                if (g >= 2 && !warp_wait(&bars[EPI_DONE + st], ((g >> 1) - 1) & 1, p.wait_limit)) {
                    report_timeout(p);
                    ok = false;
                    break;
                }
                if (use_ts) {
                    const int j0 = t.kt * BN;
                    int64_t v[4], mn[4], mx[4];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {      // key lane + 32 q4 lies in quarter q4
                        const int j = j0 + lane + 32 * q4;
                        v[q4] = 0;
                        mn[q4] = INT64_MAX;
                        mx[q4] = INT64_MIN;
                        if (j < s.L) {
                            v[q4] = p.ts[s.start + clamp_pos(j, s.E)];
                            mn[q4] = mx[q4] = v[q4];
                        }
                    }
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) {
                            mn[q4] = min(mn[q4], shfl_xor_i64(mn[q4], o));
                            mx[q4] = max(mx[q4], shfl_xor_i64(mx[q4], o));
                        }
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int c = lane + 32 * q4;
                        const bool ok32 = mn[q4] > mx[q4] ||
                                          (uint64_t)mx[q4] - (uint64_t)mn[q4] < (uint64_t)INT32_MAX;
                        tsk[st * BN + c] = v[q4];
                        // stamps relative to the quarter's minimum (0 for keys past the sequence)
                        tsk32[st * BN + c] = (j0 + c < s.L && ok32)
                                                 ? (int32_t)((uint64_t)v[q4] - (uint64_t)mn[q4])
                                                 : 0;
                        if (lane == 0) {
                            meta[st].tmin[q4] = mn[q4];
                            meta[st].tmax[q4] = mx[q4];
                            meta[st].ok32[q4] = ok32;
                        }
                    }
                }
                __syncwarp();
                mbar_arrive(&bars[META_FULL + st]);
                ++g;
            }
        }
    }
    else if (warp >= 4) {
        // -------------------------------------------------------------------- epilogue
        const int wq = (warp - 4) >> 2;               // key quarter: columns [32 wq, 32 wq + 32)
        const int r = (warp & 3) * 32 + lane;         // query row in the tile == TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const bool use_ts = p.NB > 0;
        const bool use_rel = p.R > 0;
        const float *relp = rel_in_smem ? relh : p.rel;
        const float rel_sc = rel_in_smem ? 1.0f : tscale;  // relp * rel_sc = scaled half rel bias
        const float half_alpha = 0.5f * p.alpha;
        const bool lut_ok = *lut_valid != 0;
        UnitFeed<FEED_WARP, false, BM> un(p, ring, args.nqt);
        int n = 0, g = 0;
        bool ok = true;
        while (ok && un.next()) {
            const SeqInfo &s = un.s;
            const int i0 = un.tile * BM;
            const int i = i0 + r;
            const bool row_in = i < s.L;
            const int pi = clamp_pos(i, s.E);
            const int64_t tsi = (use_ts && row_in) ? p.ts[s.start + pi] : 0;
            TileIter t(s, i0, p.W);
            while (t.next()) {
                const int st = g & 1, ps = g % NP;
                const int jq = t.kt * BN + wq * QW;      // first key of this warpgroup's quarter
                const BlockMask bm = fwd_block_mask(s, i0, jq, i, p.W);
                const bool full = bm.full;
                // the set-up below needs only the stamps; S is waited for afterwards
                if (!warp_wait(&bars[META_FULL + st], (g >> 1) & 1, p.wait_limit)) {
                    ok = false;
                    break;
                }
                // ---- per (row, quarter tile) structure; path choices are made warp-uniform
                const uint32_t vmask = bm.bits;
                const int rbase = pi - jq;            // rel index of key jq + c is rbase - c
                // a 32 x 32 block without a valid pair only writes zeros into A
                const bool blk_any = __any_sync(0xffffffffu, vmask != 0u);
                // training: without a rel table the clamped path reads the single zero entry;
                // inference: the guard bands take indices up to kRelGuard outside the table
                const int guard = SPLIT ? 0 : kRelGuard;
                const int rb_ = use_rel ? rbase : 0;
                // (the direct index uses j for p(j): right for candidate keys only when negative
                // distances clamp to 0, so the |p(i) - p(j)| variant takes such blocks clamped)
                const bool rabs = (p.flags & HSTU_FLAG_REL_ABS) != 0;
                const bool rdirect =
                    (SPLIT ? use_rel : rel_in_smem) && (!rabs || jq + QW - 1 < s.E) &&
                    __all_sync(0xffffffffu, rb_ - (QW - 1) >= -guard &&
                                                rb_ <= (use_rel ? p.R : 1) - 1 + guard);
                HalfTime ht = {};
                int tmode = 0;
                if (use_ts) {
                    ht = half_time_setup(thr, p.n_thr, tbh, p.NB, row_in, tsi, meta[st].tmin[wq],
                                         meta[st].tmax[wq], meta[st].ok32[wq] != 0, lut_ok, lutp);
                    tmode = __reduce_max_sync(0xffffffffu, ht.my_mode);
                }
                FwdEpi e;
                e.t_s = tmem + lane_base + st * 128 + wq * QW;
                e.t_a = SPLIT ? tmem + lane_base + kPCol + wq * 32
                              : tmem + lane_base + kPCol + ps * 64 + wq * 16;
                e.tk32 = tsk32 + st * BN + wq * QW;
                e.tk64 = tsk + st * BN + wq * QW;
                e.relp = use_rel ? relp : relh;
                e.rel_sc = rel_sc;
                e.relp2 = relp2;
                e.relg = use_rel ? p.rel : relh;
                e.rbase = use_rel ? rbase : 0;
                e.R = use_rel ? p.R : 1;
                e.cand0 = s.E > 0 ? s.E - jq : (1 << 30);   // E = 0: positions unclamped
                e.rcand = use_rel ? pi - (s.E - 1) : 0;
                e.rabs = rabs;
                e.half_alpha = half_alpha;
                e.alpha = p.alpha;
                e.tbh = tbh;
                e.lut = lutp;
                e.thr = thr;
                e.n_thr = p.n_thr;
                e.tsi = tsi;
                // S of this tile; A's buffer is free once the A V of tile g - NP has completed
                if (!warp_wait(&bars[S_FULL + st], (g >> 1) & 1, p.wait_limit) ||
                    (g >= NP && !warp_wait(&bars[P_FREE + ps], ((g / NP) - 1) & 1, p.wait_limit))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (!blk_any) {
                    // this quarter's A columns (SPLIT: hi and lo parts, 32 columns)
                    tmem_zero16(e.t_a);
                    if constexpr (SPLIT) tmem_zero16(e.t_a + 16);
                } else if constexpr (!SPLIT) {
                    if (tmode == 3) fwd_quarter_inf<3, false, false>(e, ht, vmask);
                    else if (!rdirect) {
                        if (tmode == 0) fwd_quarter_inf<0, false, false>(e, ht, vmask);
                        else if (tmode == 1) fwd_quarter_inf<1, false, false>(e, ht, vmask);
                        else fwd_quarter_inf<2, false, false>(e, ht, vmask);
                    } else {
                        // fully valid blocks run the masked bodies too (vmask all ones): fewer
                        // bodies measured faster than a specialised one (instruction cache)
                        if (tmode == 0) fwd_quarter_inf<0, true, false>(e, ht, vmask);
                        else if (tmode == 1) fwd_quarter_inf<1, true, false>(e, ht, vmask);
                        else fwd_quarter_inf<2, true, false>(e, ht, vmask);
                    }
                } else if (tmode == 3) {
                    fwd_quarter<3, false, false>(e, ht, vmask);
                } else if (full && rdirect) {
                    if (tmode == 0) fwd_quarter<0, true, true>(e, ht, vmask);
                    else if (tmode == 1) fwd_quarter<1, true, true>(e, ht, vmask);
                    else fwd_quarter<2, true, true>(e, ht, vmask);
                } else if (rdirect) {
                    if (tmode == 0) fwd_quarter<0, true, false>(e, ht, vmask);
                    else if (tmode == 1) fwd_quarter<1, true, false>(e, ht, vmask);
                    else fwd_quarter<2, true, false>(e, ht, vmask);
                } else {
                    if (tmode == 0) fwd_quarter<0, false, false>(e, ht, vmask);
                    else if (tmode == 1) fwd_quarter<1, false, false>(e, ht, vmask);
                    else fwd_quarter<2, false, false>(e, ht, vmask);
                }
                tc_fence_before();
                warp_arrive(&bars[S_FREE + st]);      // S has been read
                tmem_wait_st();
                tc_fence_before();
                warp_arrive(&bars[P_FULL + ps]);
                warp_arrive(&bars[EPI_DONE + st]);    // stamps and ranges of this stage read
                ++g;
            }
            if (!ok) break;
            // ---- the unit's output: Y = (1/N) O; this warpgroup's quarter of the columns
            if (!warp_wait(&bars[O_FULL], n & 1, p.wait_limit)) { ok = false; break; }
            tc_fence_after();
            constexpr int OC = DV / 4;                // 32 or 16 output columns per warpgroup
            uint32_t ro[32];
            if (OC == 32) {
                tmem_ld32(tmem + lane_base + kOCol + wq * OC, ro);
            } else {
                uint32_t (&r16)[16] = *reinterpret_cast<uint32_t(*)[16]>(ro);
                tmem_ld16(tmem + lane_base + kOCol + wq * OC, r16);
            }
            tmem_wait_ld();
            reg_fence(ro);
            tc_fence_before();
            warp_arrive(&bars[O_FREE]);
            {
                // lanes of a group of OC/4 write one row's chunks side by side
                constexpr int NCH = OC / 4;
                float4 yc[NCH];
#pragma unroll
                for (int x = 0; x < NCH; ++x)
                    yc[x] = make_float4(__uint_as_float(ro[4 * x]) * p.inv_N,
                                        __uint_as_float(ro[4 * x + 1]) * p.inv_N,
                                        __uint_as_float(ro[4 * x + 2]) * p.inv_N,
                                        __uint_as_float(ro[4 * x + 3]) * p.inv_N);
                transpose_chunks<NCH>(yc);
                const int j = lane % NCH, r0 = i - j;         // rows r0 .. r0 + NCH - 1
                // (head dims below DV run padded: only the first p.dv columns are real)
                const int col = wq * OC + 4 * j;
                float *yb = args.y + (s.start + r0) * (int64_t)p.D + un.h * p.dv + col;
#pragma unroll
                for (int c = 0; c < NCH; ++c)
                    if (r0 + c < s.L && col < p.dv)
                        *reinterpret_cast<float4 *>(yb + (int64_t)c * p.D) = yc[c];
            }
            ++n;
        }
        if (!ok || !un.ok) report_timeout(p);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

int num_sms()
{
    // cached per device ordinal (a process may drive GPUs of different sizes)
    constexpr int kMaxDev = 64;
    static std::atomic<int> cache[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < kMaxDev) {
        const int v = cache[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
    }
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
        return 148;
    if (dev < kMaxDev) cache[dev].store(v, std::memory_order_relaxed);
    return v;
}

namespace {

template <int DQK, int DV>
cudaError_t launch_tc(const FwdTcArgs &a, bool split, cudaStream_t st)
{
    using L = FwdLayout<DQK, DV>;
    static_assert(L::ALLOC + kSeqTileCache <= 232448,
                  "shared memory layout exceeds the per-CTA limit");
    auto kern = split ? fwd_tc_kernel<DQK, DV, true> : fwd_tc_kernel<DQK, DV, false>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    const int64_t units = (int64_t)a.nqt * a.p.B * a.p.H;
    const int grid = (int)(units < num_sms() ? units : num_sms());
    if (grid <= 0) return cudaSuccess;
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

// Head dims: multiples of 16 up to 128.  Below 64 (or between 64 and 128) the kernel for 64
// (128) runs on zero-padded tiles: the TMA boxes past d read zeros, which add nothing to
// Q K^T, and the output columns past d_v are not stored.
bool tc_fwd_supported(int dqk, int dv, int64_t T)
{
    return dqk >= 16 && dqk <= 128 && dqk % 16 == 0 && dv >= 16 && dv <= 128 && dv % 16 == 0 &&
           T < ((int64_t)1 << 31);
}

cudaError_t launch_tc_fwd(const DevParams &p, const void *q, const void *k, const void *v,
                          float *y, unsigned long long *unit_ctr, bool training,
                          cudaStream_t st)
{
    FwdTcArgs a;
    std::memset(&a, 0, sizeof(a));
    a.p = p;
    a.y = y;
    a.unit_ctr = unit_ctr;
    a.nqt = (p.N + BM - 1) / BM;
    if (!encode_tmap_bf16(&a.tq, q, p.dqk, p.H, p.T) || !encode_tmap_bf16(&a.tk, k, p.dqk, p.H, p.T) ||
        !encode_tmap_bf16(&a.tv, v, p.dv, p.H, p.T))
        return cudaErrorInvalidValue;
    const int dq = p.dqk <= 64 ? 64 : 128, dvp = p.dv <= 64 ? 64 : 128;   // padded dims
    if (dq == 128 && dvp == 128) return launch_tc<128, 128>(a, training, st);
    if (dq == 128 && dvp == 64) return launch_tc<128, 64>(a, training, st);
    if (dq == 64 && dvp == 128) return launch_tc<64, 128>(a, training, st);
    return launch_tc<64, 64>(a, training, st);
}

}  // namespace hstu
