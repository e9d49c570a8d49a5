// bias.cuh -- shared pieces of the bias evaluation of the tensor-core kernels: the exact
// time-bucket lookup table, bounded bucket searches, and the per-row valid-key bit masks
// of a 64-key half tile.  The bias and mask they implement are those of include/hstu_attn.h
// ("HSTU tensor by tensor: SiLU aggregation, temporal bias and gating", sections "Relative
// time adds information content similarity lacks" and "Temporal bias is not simply fixed
// forgetting"; "HSTU-MUSA: HSTU for Moore Threads (MUSA)", "Mathematical Equivalence").
#pragma once

#include "common.cuh"

namespace hstu {

constexpr int kHalf = 64;   // keys (forward) or queries (backward) per epilogue warpgroup

// Exact time-bucket lookup on y = |dt| + 1 < 2^31: cell q = 32*floor(log2 y) + (next 5 bits of
// y), i.e. the top bits of y's float representation.  A cell spans less than 1/32 of its
// value while distinct bucket thresholds differ by a larger factor (checked when the
// table is built), so at most one distinct threshold falls inside a cell:
//   bucket(dt) = base + (dt >= next ? jump : 0).
struct LutEntry {
    uint32_t next;   // the threshold inside the cell (UINT32_MAX: none)
    int16_t base;    // bucket of the cell's smallest |dt|
    int16_t jump;    // thresholds equal to `next` (buckets gained at it)
};
constexpr int kLutCells = 1024;

__device__ __forceinline__ int lut_cell(uint32_t dt)
{
    // converted toward zero, y keeps its exponent and its leading mantissa bits exactly
    const float f = __uint2float_rz(dt + 1u);
    return (int)(__float_as_uint(f) >> 18) - (127 << 5);
}

// Bucket of dt known to lie in [lo, hi]: number of thresholds <= dt (thr[k-1] opens bucket k).
__device__ __forceinline__ int bucket_in(const uint64_t *thr, int lo, int hi, uint64_t dt)
{
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (thr[mid - 1] <= dt) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Keys [a, b] intersected with [jh, jh+63], as bits relative to jh.
__device__ __forceinline__ uint64_t range_bits(int a, int b, int jh)
{
    const int lo = max(a, jh) - jh, hi = min(b, jh + kHalf - 1) - jh;
    if (lo > hi) return 0ull;
    const int n = hi - lo + 1;
    const uint64_t m = n >= 64 ? ~0ull : ((1ull << n) - 1ull);
    return m << lo;
}

// Valid keys of row i among [jh, jh+63] (bit c <-> key jh + c): the contextual prefix for
// every row; for non-contextual rows the causal (windowed) history keys up to p(i); for a
// candidate row also itself.  Equivalent to pair_valid over the half tile.
__device__ __forceinline__ uint64_t row_valid_bits(int i, int jh, const SeqInfo &s, int W)
{
    if (i >= s.L) return 0ull;
    if (i < s.c) return range_bits(0, (s.cfull ? s.E : s.c) - 1, jh);   // contextual row
    uint64_t m = range_bits(0, s.c - 1, jh);
    const int pi = clamp_pos(i, s.E);
    const int lo = W > 0 ? max(s.c, pi - W) : s.c;
    m |= range_bits(lo, min(pi, s.E - 1), jh);
    if (i >= s.E) m |= range_bits(i, i, jh);
    return m;
}

// Fills the time-bucket lookup table; clears *valid when some cell holds two thresholds
// (bucket thresholds closer than the cell resolution), which disables the table.
static __device__ void build_lut(const uint64_t *thr, int n_thr, LutEntry *lut, int32_t *valid)
{
    for (int q = threadIdx.x; q < kLutCells; q += blockDim.x) {
        const int e = q >> 5, m = q & 31;
        const uint64_t ylo = (((uint64_t)(32 + m) << e) + 31) >> 5;      // ceil(2^e (32+m)/32)
        const uint64_t yhi = ((((uint64_t)(33 + m) << e) + 31) >> 5) - 1; // last y in the cell
        LutEntry ent;
        ent.next = 0xFFFFFFFFu;
        ent.base = 0;
        ent.jump = 0;
        if (ylo >= 1 && ylo <= yhi) {
            const uint64_t dlo = ylo - 1, dhi = yhi - 1;
            const int b = bucket_search(thr, n_thr, dlo);
            ent.base = (int16_t)b;
            if (b < n_thr && thr[b] <= dhi) {
                int n = 1;
                while (b + n < n_thr && thr[b + n] == thr[b]) ++n;
                if (b + n < n_thr && thr[b + n] <= dhi) atomicAnd(valid, 0);
                if (thr[b] > 0xFFFFFFFEull) atomicAnd(valid, 0);
                ent.next = (uint32_t)min(thr[b], (uint64_t)0xFFFFFFFEull);
                ent.jump = (int16_t)n;
            }
        }
        lut[q] = ent;
    }
}

__device__ __forceinline__ int64_t shfl_xor_i64(int64_t v, int m)
{
    return (int64_t)__shfl_xor_sync(0xffffffffu, (long long)v, m);
}


// Query rows i in [ih, ih+63] that see key j (bit c <-> query ih + c): the transpose of
// row_valid_bits, used by the backward where a thread owns a key.
__device__ __forceinline__ uint64_t col_valid_bits(int j, int ih, const SeqInfo &s, int W)
{
    if (j >= s.L) return 0ull;
    if (j >= s.E) return range_bits(j, j, ih);                 // candidate key: itself
    if (j < s.c) return range_bits(0, s.L - 1, ih);            // contextual key: every row
    // history key: history rows from j (window j+W) and, within the window of E-1,
    // every candidate row
    const int hi = W > 0 ? min(s.E - 1, j + W) : s.E - 1;
    uint64_t m = range_bits(max(j, s.c), hi, ih);
    if (s.cfull) m |= range_bits(0, s.c - 1, ih);               // variant: contextual rows
    if (W <= 0 || (s.E - 1) - j <= W) m |= range_bits(s.E, s.L - 1, ih);
    return m;
}

// Time bias of one (row, 64-column half tile).  The bucket is evaluated at the smallest
// and largest |dt| the half can produce; `mode` (made warp-uniform by the caller) selects
// how the columns are evaluated: 0 = one bucket for the whole row half, 1 = one bucket
// boundary (compare 32-bit stamps relative to the half's minimum), 2 = exact lookup table,
// 3 = 64-bit threshold search.  Every lane gets exact values in any mode >= its own.
struct HalfTime {
    int my_mode;
    bool lane_const;
    int blo;
    float tb_lo, tb_hi;
    int32_t cmpA, cmpB, t_rel;
};

// Exact bucket of dt < 2^31 - 1 through the lookup table.
__device__ __forceinline__ int lut_bucket(const LutEntry *lut, uint32_t dt)
{
    const LutEntry e = lut[lut_cell(dt)];
    return e.base + (dt >= e.next ? e.jump : 0);
}

__device__ __forceinline__ HalfTime half_time_setup(const uint64_t *thr, int n_thr,
                                                    const float *tbs, int NB, bool row_in,
                                                    int64_t t_row, int64_t hmin, int64_t hmax,
                                                    bool h32, bool lut_ok, const LutEntry *lut)
{
    HalfTime h;
    h.my_mode = 0;
    h.blo = 0;
    h.cmpA = INT32_MIN;
    h.cmpB = INT32_MAX;
    h.t_rel = 0;
    int bhi = 0;
    if (row_in && hmin <= hmax) {
        uint64_t dlo, dhi;
        if (t_row >= hmax) {
            dlo = (uint64_t)t_row - (uint64_t)hmax;
            dhi = (uint64_t)t_row - (uint64_t)hmin;
        } else if (t_row <= hmin) {
            dlo = (uint64_t)hmin - (uint64_t)t_row;
            dhi = (uint64_t)hmax - (uint64_t)t_row;
        } else {
            dlo = 0;
            const uint64_t a = (uint64_t)t_row - (uint64_t)hmin;
            const uint64_t c = (uint64_t)hmax - (uint64_t)t_row;
            dhi = a > c ? a : c;
        }
        if (lut_ok && dhi < (uint64_t)(INT32_MAX - 1)) {
            // the bucket of dhi only matters as blo, blo + 1 or beyond: compare dhi with the
            // next two thresholds instead of a second lookup (equal thresholds skip a bucket)
            h.blo = lut_bucket(lut, (uint32_t)dlo);
            const uint64_t t1 = h.blo < n_thr ? thr[h.blo] : ~0ull;
            const uint64_t t2 = h.blo + 1 < n_thr ? thr[h.blo + 1] : ~0ull;
            bhi = dhi < t1 ? h.blo : (dhi < t2 ? h.blo + 1 : h.blo + 2);
        } else {
            h.blo = bucket_in(thr, 0, n_thr, dlo);
            bhi = bucket_in(thr, h.blo, n_thr, dhi);
        }
        const bool fits = h32 && dhi < (uint64_t)(INT32_MAX - 1);
        if (fits) h.t_rel = (int32_t)((uint64_t)t_row - (uint64_t)hmin);
        if (bhi == h.blo) {
            h.my_mode = 0;
        } else if (bhi == h.blo + 1 && fits) {
            h.my_mode = 1;
            // |t_row - t_col| >= T  <=>  t_col <= t_row - T  or  t_col >= t_row + T
            const int64_t T = (int64_t)thr[h.blo];
            const int64_t A = (int64_t)h.t_rel - T, B = (int64_t)h.t_rel + T;
            h.cmpA = (int32_t)max((int64_t)INT32_MIN, min((int64_t)INT32_MAX, A));
            h.cmpB = (int32_t)max((int64_t)INT32_MIN, min((int64_t)INT32_MAX, B));
        } else {
            h.my_mode = (fits && lut_ok) ? 2 : 3;
        }
    }
    h.lane_const = h.my_mode == 0;
    h.tb_lo = tbs[h.blo];
    h.tb_hi = tbs[min(h.blo + 1, NB - 1)];
    return h;
}

// Time bias of one column in mode `mode` (warp-uniform); t32/t64 are the column's stamp
// relative to the half's minimum and absolute; *bucket receives the bucket (for gradients).
__device__ __forceinline__ float half_time_value(const HalfTime &h, int mode, int32_t t32,
                                                 int64_t t64, int64_t t_row, const uint64_t *thr,
                                                 int n_thr, const float *tbs,
                                                 const LutEntry *lut, int *bucket)
{
    if (mode == 0) {
        *bucket = h.blo;
        return h.tb_lo;
    }
    if (mode == 1) {
        const bool hi = t32 <= h.cmpA || t32 >= h.cmpB;
        *bucket = h.blo + (hi ? 1 : 0);
        return hi ? h.tb_hi : h.tb_lo;
    }
    if (mode == 2) {
        if (h.lane_const) {
            *bucket = h.blo;
            return h.tb_lo;
        }
        const int32_t d = h.t_rel - t32;
        uint32_t dt = (uint32_t)(d < 0 ? -d : d);
        dt = min(dt, (uint32_t)INT32_MAX - 1u);
        const LutEntry e = lut[lut_cell(dt)];
        const int b = e.base + (dt >= e.next ? e.jump : 0);
        *bucket = b;
        return tbs[b];
    }
    const int b = bucket_search(thr, n_thr, abs_diff_u64(t_row, t64));
    *bucket = b;
    return tbs[b];
}

}  // namespace hstu
