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
// Persistent CTAs walk work units (128-key tile, sequence, head), units with the most query
// tiles first; a unit walks the 128-row query tiles that see its keys.  Thread = key row =
// TMEM lane, so scores are computed transposed:
//   S^T = K Q^T and dP^T = V dY^T          (tcgen05, bf16 in smem, fp32 in TMEM)
//   epilogue: A^T (bf16, over S^T in TMEM) and dS^T (bf16, 128B-swizzled in smem, in the
//             buffer of the dY low parts, which dP^T has finished with)
//   dV += A^T dY (A from TMEM), dK += dS^T Q, dQ_tile = dS K (dS^T read as an MN-major A)
// dV and dK accumulate in TMEM across the query tiles of a unit; each dQ tile is added to an
// fp32 accumulator in global memory with vector reductions.
//
// Table gradients never take a shared-memory atomic per pair (a float atomic add on shared
// memory retries under contention, and the pairs of one query hit few buckets):
//   rel: within a 32-key x 32-query block the index is the diagonal i - j, so each warp sums
//        the diagonals in registers by shifting partial sums one lane per column, and adds
//        the 63 diagonal sums with two scatters; candidate rows (index p(E-1) - p(j))
//        go to a per-lane sum; the rare blocks with bidirectional contextual or
//        out-of-table pairs add each pair into the output with a global reduction.
//   time: along a key row the bucket changes rarely (timestamps ascend with position), so
//        each lane sums runs of equal buckets and adds a run with one fire-and-forget global
//        reduction into a histogram private to the CTA, folded into the output at the end.
// Warp roles: TMA producer, MMA issuer, TMEM owner, query-timestamp staging, and four
// epilogue warpgroups that split the query columns.  Every wait is bounded.
#include <cudaTypedefs.h>

#include <cstring>

#include "kernels.h"
#include "sm100.cuh"
#include "tiles.cuh"
#include "units.cuh"

namespace hstu {

using namespace sm100;

namespace {

constexpr int BM = 128, BN = 128;
constexpr int QW = 32;                  // query columns per epilogue warpgroup
static_assert(BM == kTile && BN == kTile && QW == kBlk, "tile shapes of tiles.cuh");
constexpr int kEpiWarps = 16;
constexpr int kEpiWarp0 = 3;            // warps 0-2: TMA, MMA, TMEM owner + query stamps
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int kRelSmemMax = 2048;
constexpr int kRelGuard = 32;           // zero entries on both sides of the shared rel table
constexpr uint32_t kTmemCols = 512;
constexpr int kBlockBytes = 128 * 128;
// TMEM columns: S^T -> A^T [0,128); dP^T -> dQ tile [128,256); dV [256,384); dK [384,512)
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;

enum Bar {
    KV_FULL = 0, KV_EMPTY = 1, QD_FULL = 2, QD_EMPTY = 3, SD_FULL = 4, META_FULL = 5,  // +2
    EPI_DONE = 7,                                                                     // +2
    P_FULL = 9, DQ_FULL = 10, DQ_FREE = 11, ACC_FULL = 12, ACC_FREE = 13, MMA_DONE = 14,
    UNIT_FULL = 15, UNIT_EMPTY = 19,                                                  // +4
    NEVER = 23,   // nothing arrives on it (the stall test's wait)
    NUM_BARS = 24
};

// Time-stamp ranges of the four 32-query quarters of a query tile.
struct QMeta {
    int64_t tmin[4], tmax[4];
    int32_t ok32[4];
};

template <int DQK, int DV>
struct BwdLayout {
    static constexpr int KB = BN * DQK * 2;
    static constexpr int VB = BN * DV * 2;
    static constexpr int QB = BM * DQK * 2;
    static constexpr int YB = BM * DV * 2;
    static constexpr int SB = BN * BM * 2;        // dS^T, bf16
    static constexpr int LB = YB > SB ? YB : SB;  // dY low parts, then dS^T
    static constexpr int K_OFF = 0;
    static constexpr int V_OFF = K_OFF + KB;
    static constexpr int Q_OFF = V_OFF + VB;
    static constexpr int Y_OFF = Q_OFF + QB;
    static constexpr int YL_OFF = Y_OFF + YB;     // also DS
    static constexpr int BAR_OFF = YL_OFF + LB;
    static constexpr int SLOT_OFF = BAR_OFF + 8 * 32;
    static constexpr int UNIT_OFF = SLOT_OFF + 16;                 // kUnitRing unit slots
    static constexpr int META_OFF = UNIT_OFF + (int)sizeof(UnitSlot) * kUnitRing;
    static constexpr int TSQ_OFF = META_OFF + 2 * (int)sizeof(QMeta);
    static constexpr int TSQ32_OFF = TSQ_OFF + 2 * BM * 8;
    static constexpr int LUT_OFF = TSQ32_OFF + 2 * BM * 4;
    static constexpr int THR_OFF = LUT_OFF + kLutCells * 8;
    static constexpr int TB_OFF = THR_OFF + 8 * kMaxTimeBuckets;
    static constexpr int REL_OFF = TB_OFF + 4 * kMaxTimeBuckets;
    static constexpr int HREL_OFF = REL_OFF + 4 * (kRelSmemMax + 2 * kRelGuard);
    static constexpr int TOTAL = HREL_OFF + 4 * kRelSmemMax;
    static constexpr int ALLOC = TOTAL + 1024;
    static_assert(NUM_BARS <= 32, "barrier area");
    static_assert(TSQ_OFF % 8 == 0 && LUT_OFF % 8 == 0, "alignment");
};

struct BwdTcArgs {
    CUtensorMap tq, tk, tv, tdy, tdyl;   // dY as bf16 hi and lo parts
    DevParams p;
    float *dq_acc;                 // [T, H, d_qk] fp32, zeroed by the caller
    __nv_bfloat16 *dk, *dv;        // [T, H, d]
    float *d_rel, *d_tb;
    float *tb_slots;               // [gridDim.x, kMaxTimeBuckets] scratch, one row per CTA
    unsigned long long *unit_ctr;  // next work unit to hand out (zeroed by the caller)
    int nkt;                       // key tiles of the longest admissible sequence
};

__device__ __forceinline__ void report_timeout(const DevParams &p)
{
    flag_error(p, HSTU_DEV_WAIT_TIMEOUT);
}


__device__ __forceinline__ void red_add_v4(float *addr, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
                 "f"(c), "f"(d)
                 : "memory");
}

// No "memory" clobber: the target never aliases what the epilogue loads, and a clobber
// would stop the compiler from overlapping the loads of neighbouring pairs.  Volatile asm
// keeps its order relative to the fence_gpu() that precedes the read-back.
__device__ __forceinline__ void red_add(float *addr, float a)
{
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(a));
}

// red_add when `pred` holds, as a predicated instruction (no branch).  A zero value adds
// nothing, so it is not tested.
__device__ __forceinline__ void red_add_if(float *addr, float a, bool pred)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %2, 0;\n\t@p red.global.add.f32 [%0], %1;\n\t}" ::"l"(addr),
        "f"(a), "r"((int)pred));
}

__device__ __forceinline__ void fence_gpu()
{
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

__device__ __forceinline__ float ld_cg(const float *addr)
{
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(addr) : "memory");
    return v;
}

// Adds v to the rel-bias gradient at index ri (shared histogram or the global output).
__device__ __forceinline__ void rel_add(float *hrel, float *d_rel, bool in_smem, int ri, float v)
{
    if (in_smem) atomicAdd(hrel + ri, v);
    else red_add(d_rel + ri, v);
}

// Per-lane state of one epilogue thread (key row j of the unit) across the query tiles.
struct KeyLane {
    int j, pj;
    bool key_in;
    int64_t tsj;
    // rel gradient: shifted diagonal sums (A: diagonals 31 - lane, B: -1 - lane of the
    // 32 x 32 block) and the candidate-row pairs (index p(E-1) - p(j))
    float sysA, sysB, cand;
    // time gradient: the open run of equal buckets
    int cur_b;
    float run;
};

// One 32-key x 32-query block of the epilogue: reads S^T and dP^T of the block from TMEM,
// writes A^T (bf16 pairs, over the block's own S^T columns) and dS^T (bf16, swizzled smem),
// and accumulates the table gradients into the lane state.  TM is the warp-uniform time
// mode of half_time_setup (0 when there is no time bias).
struct EpiBlock {
    uint32_t t_s, t_dp;           // TMEM addresses of the block's S^T (then A^T) and dP^T
    uint32_t ds_row;              // smem address of this key's dS^T row (first 16-byte chunk)
    int ds_chunk0, rsw;           // first chunk of the block in the row, swizzle (row & 7)
    int iq;                       // first query of the block
    int rbase;                    // p(iq) - p(j) in direct blocks (history columns)
    int fc, rc;                   // first candidate column; this key's rel index for it
    float *d_rel;                 // the rel-gradient output (kind 2 adds into it directly)
    int Em1;                      // p(i) = min(i, Em1)
    bool full, use_rel, use_ts, rel_in_smem;
    uint32_t vbits;               // valid queries of this key (bit c <-> query iq + c)
    const int32_t *tq32;          // the block's query stamps relative to the quarter minimum
    const int64_t *tq64;          // and absolute
    const float *relp;
    const uint64_t *thr;
    const float *tbs;
    const LutEntry *lut;
    float *tb_slot;
};

// Rel index of a pair, by KIND:
//   0  direct: every valid pair has index p(i) - p(j) = rbase + c in [0, R) (no candidate
//      row, no clamping); the table sits in shared memory with a guard band that keeps the
//      reads of masked pairs (at most 31 entries off) in bounds;
//   1  direct for the history columns, and the candidate columns (c >= fc, p(i) = E - 1)
//      at the lane's constant index rc;
//   2  every index clamped; each pair adds into the output directly (rare blocks).
template <int TM, int KIND>
__device__ __forceinline__ void epi_block(const DevParams &p, const EpiBlock &e,
                                          const HalfTime &ht, KeyLane &k, float &t_lo,
                                          float &t_hi)
{
    // The body is free of branches (selects and predicated reductions only), so the
    // compiler can overlap the loads and the arithmetic of neighbouring pairs.
    const int lane = threadIdx.x & 31;
    if (TM == 0 && e.use_ts && k.key_in) {
        if (ht.blo != k.cur_b) {
            if (k.run != 0.f) red_add(e.tb_slot + k.cur_b, k.run);
            k.cur_b = ht.blo;
            k.run = 0.f;
        }
    }
    const bool lane0 = lane == 0;
    const int src = (lane + 31) & 31;
#pragma unroll 1
    for (int ch = 0; ch < 8; ++ch) {
        // 4 query columns: half a 16-byte chunk of the dS^T row, 2 TMEM columns of A^T
        uint32_t rs[4], rd[4];
        tmem_ld4(e.t_s + ch * 4, rs);   // S and dP arrive while the biases are formed
        tmem_ld4(e.t_dp + ch * 4, rd);
        float bias[4];
        int bkv[4], riv[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int cc = ch * 4 + c;
            const int i = e.iq + cc;
            int bk = 0;
            if (TM == 0) {
                bias[c] = ht.tb_lo;
            } else if (TM == 1) {
                const int32_t t = e.tq32[cc];
                const bool hi = t <= ht.cmpA || t >= ht.cmpB;
                bias[c] = hi ? ht.tb_hi : ht.tb_lo;
                bk = hi ? 1 : 0;
            } else if (TM == 2) {
                const int32_t d = ht.t_rel - e.tq32[cc];
                uint32_t dt = (uint32_t)(d < 0 ? -d : d);
                dt = min(dt, (uint32_t)INT32_MAX - 1u);
                const int b = lut_bucket(e.lut, dt);
                bk = ht.lane_const ? ht.blo : b;
                bias[c] = ht.lane_const ? ht.tb_lo : e.tbs[b];
            } else {
                bk = bucket_search(e.thr, p.n_thr, abs_diff_u64(k.tsj, e.tq64[cc]));
                bias[c] = e.tbs[bk];
            }
            int ri;
            if (KIND == 0) {
                ri = e.rbase + cc;
            } else if (KIND == 1) {
                ri = cc >= e.fc ? e.rc : e.rbase + cc;
            } else {
                ri = rel_index(min(i, e.Em1) - k.pj, p.R, (p.flags & HSTU_FLAG_REL_ABS) != 0);
            }
            bias[c] += e.relp[ri];
            bkv[c] = bk;
            riv[c] = ri;
        }
        tmem_wait_ld();
        reg_fence(rs);
        reg_fence(rd);
        uint32_t pa[2], pd[2];
        int tbk[4];        // TM >= 2: bucket of each pair (-1: masked) and its dS
        float tds[4];
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
            float av[2], dv2[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int c = 2 * c2 + q, cc = ch * 4 + c;
                const bool valid = (e.vbits >> cc) & 1u;
                const int bk = bkv[c], ri = riv[c];
                const float bias_c = bias[c];
                // ---- s = alpha q.k + b; SiLU(s) = s sigma(s); SiLU'(s) = sigma (1 + s (1 - sigma)).
                // sigma from the accurate exponential: table gradients sum dS over many pairs
                // and can cancel, so dS needs close to fp32 accuracy
                const float xs = fmaf(p.alpha, __uint_as_float(rs[c]), bias_c);
                const float sig = __fdividef(1.0f, 1.0f + __expf(-xs));
                const float silu = xs * sig;
                const float dsilu = sig * fmaf(xs, 1.0f - sig, 1.0f);
                const float a = valid ? silu * p.inv_N : 0.f;
                const float ds = valid ? __uint_as_float(rd[c]) * dsilu * p.inv_N : 0.f;
                av[q] = a;
                dv2[q] = ds;
                // ---- rel gradient: shift the diagonal sums one lane down, add this column
                float vd = ds;
                if (KIND == 1) {
                    const bool candc = cc >= e.fc;           // warp-uniform
                    k.cand += candc ? ds : 0.f;
                    vd = candc ? 0.f : ds;
                } else if (KIND == 2) {
                    // rare blocks (bidirectional contextual or out-of-table pairs): every
                    // pair, masked ones adding zero, straight into the output at its index
                    atomicAdd(e.d_rel + ri, ds);
                }
                if (KIND != 2) {
                    const float ain = __shfl_sync(0xffffffffu, k.sysA, src);
                    const float bin = __shfl_sync(0xffffffffu, k.sysB, src);
                    k.sysB = lane0 ? ain : bin;
                    k.sysA = (lane0 ? 0.f : ain) + vd;
                }
                // ---- time gradient
                if (TM == 0) {
                    k.run += ds;
                } else if (TM == 1) {
                    t_hi += bk ? ds : 0.f;
                    t_lo += bk ? 0.f : ds;
                } else {
                    tbk[c] = valid ? bk : -1;
                    tds[c] = ds;
                }
            }
            pa[c2] = pack_bf16x2(av[0], av[1]);
            pd[c2] = pack_bf16x2(dv2[0], dv2[1]);
        }
        if (TM >= 2) {
            // runs of equal buckets over the chunk's pairs, after all of its loads: a flush
            // (inline asm) inside the pair loop would hold the next pairs' loads behind it
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const bool chg = tbk[c] >= 0 && tbk[c] != k.cur_b;
                red_add_if(e.tb_slot + k.cur_b, k.run, chg && e.use_ts);
                k.cur_b = chg ? tbk[c] : k.cur_b;
                k.run = (chg ? 0.f : k.run) + tds[c];
            }
        }
        tmem_st2(e.t_s + ch * 2, pa);
        st_shared_v2(e.ds_row + (((e.ds_chunk0 + (ch >> 1)) ^ e.rsw) << 4) + (ch & 1) * 8, pd[0],
                     pd[1]);
    }
}

// Adds the rel-gradient sums of a finished block and resets them.  Diagonal d (relative to
// the block) has index iq - jw + d, jw = the warp's first key.
__device__ __forceinline__ void flush_rel(const DevParams &p, KeyLane &k, int iq, int jw,
                                          int Em1, float *hrel, float *d_rel, bool in_smem)
{
    const int lane = threadIdx.x & 31;
    const int base = iq - jw;
    const int ra = base + 31 - lane, rb = base - 1 - lane;
    if (k.sysA != 0.f && ra >= 0 && ra < p.R) rel_add(hrel, d_rel, in_smem, ra, k.sysA);
    if (k.sysB != 0.f && rb >= 0 && rb < p.R) rel_add(hrel, d_rel, in_smem, rb, k.sysB);
    if (k.cand != 0.f) {
        int rc = Em1 - k.pj;
        rc = rc < 0 ? 0 : (rc > p.R - 1 ? p.R - 1 : rc);
        rel_add(hrel, d_rel, in_smem, rc, k.cand);
    }
    k.sysA = k.sysB = k.cand = 0.f;
}

// Adds v to the time-gradient run state for bucket b (closing the open run if it differs).
__device__ __forceinline__ void run_add(KeyLane &k, float *slot, int b, float v)
{
    if (v == 0.f) return;
    if (b != k.cur_b) {
        if (k.run != 0.f) red_add(slot + k.cur_b, k.run);
        k.cur_b = b;
        k.run = v;
    } else {
        k.run += v;
    }
}

// Reads NC fp32 columns of this lane's TMEM row starting at taddr, in pieces of up to 32.
template <int NC, typename F>
__device__ __forceinline__ void tmem_row_foreach(uint32_t taddr, F &&f)
{
    if constexpr (NC >= 32) {
#pragma unroll
        for (int cq = 0; cq < NC / 32; ++cq) {
            uint32_t v[32];
            tmem_ld32(taddr + cq * 32, v);
            tmem_wait_ld();
            reg_fence(v);
            f(cq * 32, v);
        }
    } else {
        uint32_t v[16];
        tmem_ld16(taddr, v);
        tmem_wait_ld();
        reg_fence(v);
        f(0, v);
    }
}

// Stores n fp32 values (times sc) as bf16, 8 per 16-byte store.
template <int N>
__device__ __forceinline__ void store_bf16_row(__nv_bfloat16 *dst, const uint32_t (&v)[N], float sc)
{
    uint4 *dp = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int q = 0; q < N / 8; ++q)
        dp[q] = make_uint4(
            pack_bf16x2(sc * __uint_as_float(v[8 * q]), sc * __uint_as_float(v[8 * q + 1])),
            pack_bf16x2(sc * __uint_as_float(v[8 * q + 2]), sc * __uint_as_float(v[8 * q + 3])),
            pack_bf16x2(sc * __uint_as_float(v[8 * q + 4]), sc * __uint_as_float(v[8 * q + 5])),
            pack_bf16x2(sc * __uint_as_float(v[8 * q + 6]), sc * __uint_as_float(v[8 * q + 7])));
}

template <int DQK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_tc_kernel(const __grid_constant__ BwdTcArgs args)
{
    using L = BwdLayout<DQK, DV>;
    const DevParams &p = args.p;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, by an offset from the shared array (keeps the compiler aware
    // that every table below lives in shared memory: 32-bit addresses, shared loads)
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BAR_OFF);
    uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::SLOT_OFF);
    int32_t *lut_valid = reinterpret_cast<int32_t *>(sm + L::SLOT_OFF + 4);
    // Work units: key tiles from the first up (the most query tiles first), sequence, head.
    const FeedRing ring{bars + UNIT_FULL, bars + UNIT_EMPTY,
                        reinterpret_cast<UnitSlot *>(sm + L::UNIT_OFF), args.unit_ctr};
    QMeta *meta = reinterpret_cast<QMeta *>(sm + L::META_OFF);
    int64_t *tsq = reinterpret_cast<int64_t *>(sm + L::TSQ_OFF);
    int32_t *tsq32 = reinterpret_cast<int32_t *>(sm + L::TSQ32_OFF);
    LutEntry *lut = reinterpret_cast<LutEntry *>(sm + L::LUT_OFF);
    uint64_t *thr = reinterpret_cast<uint64_t *>(sm + L::THR_OFF);
    float *tbs = reinterpret_cast<float *>(sm + L::TB_OFF);
    float *rels = reinterpret_cast<float *>(sm + L::REL_OFF) + kRelGuard;
    float *hrel = reinterpret_cast<float *>(sm + L::HREL_OFF);
    float *tb_slot = args.tb_slots + (size_t)blockIdx.x * kMaxTimeBuckets;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int x = 0; x < NUM_BARS; ++x) mbar_init(&bars[x], 1);
        mbar_init(&bars[EPI_DONE], kEpiWarps);
        mbar_init(&bars[EPI_DONE + 1], kEpiWarps);
        mbar_init(&bars[P_FULL], kEpiWarps);
        mbar_init(&bars[DQ_FREE], kEpiWarps);
        mbar_init(&bars[ACC_FREE], kEpiWarps);
        for (int x = 0; x < kUnitRing; ++x) mbar_init(&bars[UNIT_EMPTY + x], 2 + kEpiWarps);
        fence_mbar_init();
        *lut_valid = 1;
    }
    if (warp == 2) tmem_alloc(slot, kTmemCols);
    for (int x = threadIdx.x; x < p.n_thr; x += kThreads) thr[x] = p.thr[x];
    for (int x = threadIdx.x; x < p.NB; x += kThreads) {
        tbs[x] = p.tb[x];
        tb_slot[x] = 0.f;
    }
    const bool rel_in_smem = p.R <= kRelSmemMax;
    if (rel_in_smem) {
        for (int x = threadIdx.x; x < p.R; x += kThreads) {
            rels[x] = p.rel[x];
            hrel[x] = 0.f;
        }
        for (int x = threadIdx.x; x < kRelGuard; x += kThreads) {
            rels[-1 - x] = 0.f;
            rels[p.R + x] = 0.f;
        }
    }
    fill_seq_tiles(p, kThreads);
    for (int b = blockIdx.x; b < p.B; b += gridDim.x) {   // rows no unit writes: zero dK, dV
        RowRange rr[3];
        const int n = skipped_rows(p, b, rr);
        for (int x = 0; x < n; ++x) {
            zero_rows(args.dk, (int64_t)p.H * p.dqk, rr[x], threadIdx.x, kThreads);
            zero_rows(args.dv, (int64_t)p.H * p.dv, rr[x], threadIdx.x, kThreads);
        }
    }
    __threadfence();   // the zeroed slot row is in place before any reduction into it
    __syncthreads();
    if (p.NB > 0) build_lut(thr, p.n_thr, lut, lut_valid);
    // the set-up above reads inputs only; dY and the zeroed accumulators come from the
    // LayerNorm backward ahead on the stream
    grid_dep_wait();
    grid_dep_release();
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
            prefetch_tmap(&args.tdy);
            prefetch_tmap(&args.tdyl);
            UnitFeed<FEED_PRODUCER, true, BN> un(p, ring, args.nkt);
            int n = 0, g = 0;
            bool ok = true;
            while (ok && un.next()) {
                const int row0 = (int)un.s.start, j0 = un.tile * BN;
                if (n >= 1 && !mbar_wait(&bars[KV_EMPTY], (n - 1) & 1, p.wait_limit)) { ok = false; break; }
                mbar_arrive_expect_tx(&bars[KV_FULL], L::KB + L::VB);
                for (int kb = 0; kb < DQK / 64; ++kb)
                    tma_load_3d(sm + L::K_OFF + kb * kBlockBytes, &args.tk, &bars[KV_FULL],
                                kb * 64, un.h, row0 + j0);
                for (int kb = 0; kb < DV / 64; ++kb)
                    tma_load_3d(sm + L::V_OFF + kb * kBlockBytes, &args.tv, &bars[KV_FULL],
                                kb * 64, un.h, row0 + j0);
                ++n;
                QTileIter t(un.s, j0, p.W);
                while (t.next()) {
                    if (g >= 1 && !mbar_wait(&bars[QD_EMPTY], (g - 1) & 1, p.wait_limit)) { ok = false; break; }
                    const int i0 = t.qt * BM;
                    mbar_arrive_expect_tx(&bars[QD_FULL], L::QB + 2 * L::YB);
                    for (int kb = 0; kb < DQK / 64; ++kb)
                        tma_load_3d(sm + L::Q_OFF + kb * kBlockBytes, &args.tq, &bars[QD_FULL],
                                    kb * 64, un.h, row0 + i0);
                    for (int kb = 0; kb < DV / 64; ++kb) {
                        tma_load_3d(sm + L::Y_OFF + kb * kBlockBytes, &args.tdy, &bars[QD_FULL],
                                    kb * 64, un.h, row0 + i0);
                        tma_load_3d(sm + L::YL_OFF + kb * kBlockBytes, &args.tdyl, &bars[QD_FULL],
                                    kb * 64, un.h, row0 + i0);
                    }
                    ++g;
                }
            }
            if (!ok || !un.ok) report_timeout(p);
            // every copy has landed before the CTA may exit
            bool drained = true;
            if (n >= 1) drained &= mbar_wait(&bars[KV_FULL], (n - 1) & 1, kWaitLimitCycles);
            if (g >= 1) drained &= mbar_wait(&bars[QD_FULL], (g - 1) & 1, kWaitLimitCycles);
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
            const uint32_t yl_addr = sm_base + L::YL_OFF, ds_addr = sm_base + L::YL_OFF;
            UnitFeed<FEED_THREAD, true, BN> un(p, ring, args.nkt);
            int n = 0, g = 0;
            // the stall test: a wait that runs out, then the same unwinding as any timeout
            bool ok = !p.stall_test || mbar_wait(&bars[NEVER], 0, p.wait_limit);
            while (ok && un.next()) {
                if (!mbar_wait(&bars[KV_FULL], n & 1, p.wait_limit)) { ok = false; break; }
                QTileIter t(un.s, un.tile * BN, p.W);
                int x = 0;
                while (t.next()) {
                    if (!mbar_wait(&bars[QD_FULL], g & 1, p.wait_limit)) { ok = false; break; }
                    // the previous tile's dQ has been read: every MMA of it completed, so the
                    // S^T/A^T and dP^T/dQ columns are free
                    if (g >= 1 && !mbar_wait(&bars[DQ_FREE], (g - 1) & 1, p.wait_limit)) { ok = false; break; }
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
                    if (!mbar_wait(&bars[P_FULL], g & 1, p.wait_limit)) { ok = false; break; }
                    // dV and dK of the previous unit have been read out
                    if (x == 0 && n >= 1 && !mbar_wait(&bars[ACC_FREE], (n - 1) & 1, p.wait_limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < BM / 16; ++kk) {
                        // dV += A^T dY: queries 16kk.. packed at columns 32(kk/2) + 8(kk%2)
                        const uint32_t a_tmem = tmem + kColS + (kk >> 1) * 32 + (kk & 1) * 8;
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
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk) {
                        // dQ = dS K: dS^T read as an MN-major A (queries contiguous per key row)
                        const uint64_t a = sw128_desc(ds_addr + kk * 2048, kBlockBytes, 1024);
                        const uint64_t bd = sw128_desc(k_addr + kk * 2048, kBlockBytes, 1024);
                        umma_bf16_ss(tmem + kColDP, a, bd, id_dq, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&bars[QD_EMPTY]);
                    umma_commit(&bars[DQ_FULL]);
                    ++x;
                    ++g;
                }
                if (!ok) break;
                umma_commit(&bars[KV_EMPTY]);
                umma_commit(&bars[ACC_FULL]);
                ++n;
            }
            if (!ok || !un.ok) report_timeout(p);
            umma_commit(&bars[MMA_DONE]);
            if (!mbar_wait(&bars[MMA_DONE], 0, kWaitLimitCycles)) report_timeout(p);
        }
    } else if (warp == 2) {
        // -------------------------------------------------------------------- query stamps
        const bool use_ts = p.NB > 0;
        UnitFeed<FEED_WARP, true, BN> un(p, ring, args.nkt);
        int g = 0;
        bool ok = true;
        while (ok && un.next()) {
            const SeqInfo &s = un.s;
            QTileIter t(s, un.tile * BN, p.W);
            while (t.next()) {
                const int st = g & 1;
                // the epilogue has finished with the stamps of tile g - 2
                if (g >= 2 && !warp_wait(&bars[EPI_DONE + st], ((g >> 1) - 1) & 1, p.wait_limit)) {
                    ok = false;
                    break;
                }
                if (use_ts) {
                    const int i0 = t.qt * BM;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int c = lane + 32 * q4, i = i0 + c;
                        const bool in = i < s.L;
                        const int64_t v = in ? p.ts[s.start + clamp_pos(i, s.E)] : 0;
                        int64_t mn = in ? v : INT64_MAX, mx = in ? v : INT64_MIN;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) {
                            mn = min(mn, shfl_xor_i64(mn, o));
                            mx = max(mx, shfl_xor_i64(mx, o));
                        }
                        const bool ok32 =
                            mn > mx || (uint64_t)mx - (uint64_t)mn < (uint64_t)INT32_MAX;
                        tsq[st * BM + c] = v;
                        tsq32[st * BM + c] = (in && ok32) ? (int32_t)((uint64_t)v - (uint64_t)mn) : 0;
                        if (lane == 0) {
                            meta[st].tmin[q4] = mn;
                            meta[st].tmax[q4] = mx;
                            meta[st].ok32[q4] = ok32 ? 1 : 0;
                        }
                    }
                }
                warp_arrive(&bars[META_FULL + st]);
                ++g;
            }
        }
        if (!ok || !un.ok) report_timeout(p);
    } else if (warp >= kEpiWarp0) {
        // -------------------------------------------------------------------- epilogue
        constexpr int kGroups = kEpiWarps / 4;        // warpgroups
        constexpr int kQPer = 4 / kGroups;            // 32-query blocks per warp and tile
        const int wg = (warp - kEpiWarp0) >> 2;      // query columns [128/kGroups * wg, ...)
        const int r = (warp & 3) * 32 + lane;        // key row in the tile == TMEM lane
        const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const bool use_ts = p.NB > 0, use_rel = p.R > 0;
        const bool lut_ok = *lut_valid != 0;
        EpiBlock e;
        e.rsw = r & 7;
        e.use_rel = use_rel;
        e.use_ts = use_ts;
        e.rel_in_smem = rel_in_smem;
        e.relp = rel_in_smem ? rels : p.rel;
        e.thr = thr;
        e.tbs = tbs;
        e.lut = lut;
        e.tb_slot = tb_slot;
        e.d_rel = args.d_rel;
        UnitFeed<FEED_WARP, true, BN> un(p, ring, args.nkt);
        int n = 0, g = 0;
        bool ok = true;
        while (ok && un.next()) {
            const SeqInfo &s = un.s;
            const int j0 = un.tile * BN, jw = j0 + (warp & 3) * 32;
            KeyLane k;
            k.j = j0 + r;
            k.key_in = k.j < s.L;
            k.pj = clamp_pos(k.j, s.E);
            k.tsj = (use_ts && k.key_in) ? p.ts[s.start + k.pj] : 0;
            k.sysA = k.sysB = k.cand = 0.f;
            k.cur_b = 0;
            k.run = 0.f;
            e.Em1 = s.E > 0 ? s.E - 1 : 0x7fffffff;
            QTileIter t(s, j0, p.W);
            int x = 0;
            while (t.next()) {
                const int st = g & 1;
                if (!warp_wait(&bars[META_FULL + st], (g >> 1) & 1, p.wait_limit) ||
                    !warp_wait(&bars[SD_FULL], g & 1, p.wait_limit)) {
                    ok = false;
                    break;
                }
#pragma unroll 1
                for (int qq = 0; qq < kQPer; ++qq) {
                    const int wq = wg * kQPer + qq;          // query columns [32 wq, 32 wq + 32)
                    e.iq = t.qt * BM + wq * QW;
                    e.t_s = tl + kColS + wq * QW;
                    e.t_dp = tl + kColDP + wq * QW;
                    e.ds_row = sm_base + L::YL_OFF + (wq >> 1) * kBlockBytes + r * 128;
                    e.ds_chunk0 = (wq & 1) * 4;
                    const BlockMask bm = bwd_block_mask(s, j0, e.iq, k.j, p.W);
                    e.full = bm.full;
                    e.vbits = bm.bits;
                    const uint32_t vb = e.vbits;
                    const bool idle = vb == 0u;
                    if (!__any_sync(0xffffffffu, !idle)) {
                        // no valid pair in the block: A and dS are zero, no table gradient
                        const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                        tmem_st8(e.t_s, z);
                        tmem_st8(e.t_s + 8, z);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            st_shared_v4(e.ds_row + (((e.ds_chunk0 + q) ^ e.rsw) << 4), 0u, 0u,
                                         0u, 0u);
                        continue;
                    }
                    // block kind (see epi_block): the history columns are direct when every
                    // valid pair there has rel index p(i) - p(j) = rbase + c within the table
                    // (lanes without a valid history pair read the guarded table at base 0)
                    const int fc = e.Em1 - e.iq + 1;           // first candidate column
                    const uint32_t candbits = fc >= QW ? 0u : (fc <= 0 ? ~0u : (~0u << fc));
                    const int rb = e.iq - k.pj;
                    const uint32_t vh = vb & ~candbits;        // valid history columns
                    const bool idle_h = vh == 0u;
                    const int c_lo = __ffs(vh) - 1, c_hi = 31 - __clz(vh);
                    const bool lane_ok = idle_h || (rb + c_lo >= 0 && rb + c_hi <= p.R - 1);
                    const bool no_cand = __all_sync(0xffffffffu, (vb & candbits) == 0u);
                    const bool all_ok =
                        !use_rel || (rel_in_smem && __all_sync(0xffffffffu, lane_ok));
                    // 0: direct, 1: direct with candidate columns, 2: general
                    const int kind = !use_rel ? 0 : (all_ok ? (no_cand ? 0 : 1) : 2);
                    e.rbase = (idle_h || !use_rel) ? 0 : rb;   // R = 0: all-zero guard band
                    e.fc = fc;
                    {
                        const int rc = e.Em1 - k.pj;
                        e.rc = rc < 0 ? 0 : (rc > p.R - 1 ? p.R - 1 : rc);
                    }
                    e.tq32 = tsq32 + st * BM + wq * QW;
                    e.tq64 = tsq + st * BM + wq * QW;
                    HalfTime ht = {};
                    int tmode = 0;
                    if (use_ts) {
                        ht = half_time_setup(thr, p.n_thr, tbs, p.NB, k.key_in, k.tsj,
                                             meta[st].tmin[wq], meta[st].tmax[wq],
                                             meta[st].ok32[wq] != 0, lut_ok, lut);
                        tmode = __reduce_max_sync(0xffffffffu, ht.my_mode);
                    }
                    float t_lo = 0.f, t_hi = 0.f;
                    tc_fence_after();
                    if (tmode == 3) {
                        epi_block<3, 2>(p, e, ht, k, t_lo, t_hi);
                    } else if (kind == 0) {
                        if (tmode == 0) epi_block<0, 0>(p, e, ht, k, t_lo, t_hi);
                        else if (tmode == 1) epi_block<1, 0>(p, e, ht, k, t_lo, t_hi);
                        else epi_block<2, 0>(p, e, ht, k, t_lo, t_hi);
                    } else if (kind == 1) {
                        if (tmode == 0) epi_block<0, 1>(p, e, ht, k, t_lo, t_hi);
                        else if (tmode == 1) epi_block<1, 1>(p, e, ht, k, t_lo, t_hi);
                        else epi_block<2, 1>(p, e, ht, k, t_lo, t_hi);
                    } else {
                        if (tmode == 0) epi_block<0, 2>(p, e, ht, k, t_lo, t_hi);
                        else if (tmode == 1) epi_block<1, 2>(p, e, ht, k, t_lo, t_hi);
                        else epi_block<2, 2>(p, e, ht, k, t_lo, t_hi);
                    }
                    if (use_ts && tmode == 1) {
                        run_add(k, tb_slot, ht.blo, t_lo);
                        run_add(k, tb_slot, ht.blo + 1, t_hi);
                    }
                    if (use_rel) flush_rel(p, k, e.iq, jw, e.Em1, hrel, args.d_rel, rel_in_smem);
                }
                tmem_wait_st();
                tc_fence_before();
                fence_proxy_async_smem();
                warp_arrive(&bars[P_FULL]);
                warp_arrive(&bars[EPI_DONE + st]);

                // ---- dQ tile: lanes = query rows of this tile; columns split by warpgroup
                if (!warp_wait(&bars[DQ_FULL], g & 1, p.wait_limit)) { ok = false; break; }
                tc_fence_after();
                {
                    constexpr int QC = DQK / kGroups;          // 16, 32 or 64 columns
                    const int i = t.qt * BM + r;
                    float *dqr = args.dq_acc + ((s.start + i) * (int64_t)p.H + un.h) * DQK + wg * QC;
                    const float al = p.alpha;
                    tmem_row_foreach<QC>(tl + kColDP + wg * QC, [&](int c0, const auto &v) {
                        constexpr int NV = sizeof(v) / sizeof(v[0]);
                        if (c0 + NV >= QC) {                     // the last piece is in registers
                            tc_fence_before();
                            warp_arrive(&bars[DQ_FREE]);
                        }
                        // the NV/4 lanes of a group add one row's chunks side by side
                        constexpr int NCH = NV / 4;
                        float4 xc[NCH];
#pragma unroll
                        for (int q = 0; q < NCH; ++q)
                            xc[q] = make_float4(al * __uint_as_float(v[4 * q]),
                                                al * __uint_as_float(v[4 * q + 1]),
                                                al * __uint_as_float(v[4 * q + 2]),
                                                al * __uint_as_float(v[4 * q + 3]));
                        transpose_chunks<NCH>(xc);
                        const int jl = lane % NCH, r0 = i - jl;   // rows r0 .. r0 + NCH - 1
                        float *dqb = dqr - (int64_t)jl * p.H * DQK + c0 + 4 * jl;
#pragma unroll
                        for (int c = 0; c < NCH; ++c)
                            if (r0 + c < s.L)
                                red_add_v4(dqb + (int64_t)c * p.H * DQK, xc[c].x, xc[c].y,
                                           xc[c].z, xc[c].w);
                    });
                }
                ++x;
                ++g;
            }
            if (!ok) break;
            if (use_ts && k.run != 0.f) red_add(tb_slot + k.cur_b, k.run);
            // ---- dV and dK of the key rows (every key tile sees at least its diagonal tile)
            if (!warp_wait(&bars[ACC_FULL], n & 1, p.wait_limit)) { ok = false; break; }
            tc_fence_after();
            {
                constexpr int VC = DV / kGroups, KC = DQK / kGroups;
                const int64_t row = (s.start + k.j) * (int64_t)p.H + un.h;
                const float sv = x > 0 ? 1.0f : 0.f, sk = x > 0 ? p.alpha : 0.f;
                __nv_bfloat16 *dvr = args.dv + row * DV + wg * VC;
                __nv_bfloat16 *dkr = args.dk + row * DQK + wg * KC;
                const bool key_in = k.key_in;
                tmem_row_foreach<VC>(tl + kColDV + wg * VC, [&](int c0, const auto &v) {
                    if (key_in) store_bf16_row(dvr + c0, v, sv);
                });
                tmem_row_foreach<KC>(tl + kColDK + wg * KC, [&](int c0, const auto &v) {
                    if (key_in) store_bf16_row(dkr + c0, v, sk);
                });
                tc_fence_before();
                warp_arrive(&bars[ACC_FREE]);
            }
            ++n;
        }
        if (!ok || !un.ok) report_timeout(p);
    }

    tc_fence_before();
    fence_gpu();   // reductions into the slot row are complete before it is read back
    __syncthreads();
    // fold this CTA's table-gradient histograms into the outputs
    if (rel_in_smem)
        for (int x = threadIdx.x; x < p.R; x += kThreads)
            if (hrel[x] != 0.f) atomicAdd(args.d_rel + x, hrel[x]);
    for (int x = threadIdx.x; x < p.NB; x += kThreads) {
        const float v = ld_cg(tb_slot + x);
        if (v != 0.f) atomicAdd(args.d_tb + x, v);
    }
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int DQK, int DV>
cudaError_t launch_bwd(const BwdTcArgs &a, cudaStream_t st)
{
    using L = BwdLayout<DQK, DV>;
    static_assert(L::ALLOC + kSeqTileCache <= 232448,
                  "shared memory layout exceeds the per-CTA limit");
    auto kern = bwd_tc_kernel<DQK, DV>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    const int64_t units = (int64_t)a.nkt * a.p.B * a.p.H;
    int grid = num_sms();
    if (grid > kBwdMaxCtas) grid = kBwdMaxCtas;
    if (units < grid) grid = (int)units;
    if (grid <= 0) return cudaSuccess;
    return launch_pdl(kern, dim3(grid), dim3(kThreads), L::ALLOC, st, a);
}

}  // namespace

bool tc_bwd_supported(int dqk, int dv, int64_t T)
{
    return (dqk == 64 || dqk == 128) && (dv == 64 || dv == 128) && T < ((int64_t)1 << 31);
}

cudaError_t launch_tc_bwd(const DevParams &p, const void *q, const void *k, const void *v,
                          const void *dy_bf16, float *dq_acc, void *dk, void *dv, float *d_rel,
                          float *d_tb, float *tb_slots, unsigned long long *unit_ctr,
                          cudaStream_t st)
{
    BwdTcArgs a;
    std::memset(&a, 0, sizeof(a));
    a.p = p;
    a.dq_acc = dq_acc;
    a.dk = reinterpret_cast<__nv_bfloat16 *>(dk);
    a.dv = reinterpret_cast<__nv_bfloat16 *>(dv);
    a.d_rel = d_rel;
    a.d_tb = d_tb;
    a.tb_slots = tb_slots;
    a.unit_ctr = unit_ctr;
    a.nkt = (p.N + BN - 1) / BN;
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
