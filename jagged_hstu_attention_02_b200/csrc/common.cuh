// common.cuh -- device-side definitions shared by the jagged HSTU attention kernels.
//
// The mask family and bias follow "HSTU-MUSA: HSTU for Moore Threads (MUSA)",
// section "Mathematical Equivalence" (contextual bidirectional prefix, candidate position
// clamping, target group masking, max attention length) and "HSTU tensor by tensor: SiLU
// aggregation, temporal bias and gating", sections "Relative time adds information content
// similarity lacks" and "Do not copy softmax masking mechanically".  The exact reading of
// each rule is stated in include/hstu_attn.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu_attn.h"

namespace hstu {

constexpr int kMaxTimeBuckets = 256;

// Everything a kernel needs, passed by value as a __grid_constant__ parameter.
struct DevParams {
    int32_t B, H, dqk, dv, N, W;
    int64_t T;
    int32_t D;            // H * dv
    float alpha, inv_N, eps;
    int32_t R, NB;
    int32_t n_thr;        // reachable thresholds (<= NB - 1)
    const int64_t *offsets;
    const int32_t *ctx, *tgt;
    const int64_t *ts;
    const float *rel, *tb;
    int32_t *status;
    int32_t flags;          // HSTU_FLAG_* mask variants
    long long wait_limit;   // cycles a pipeline wait may take before the kernel gives up
    int32_t stall_test;     // test only: the MMA issuer first waits on a barrier nothing completes
    // smallest |dt| of bucket k+1 (fp64-decided on the host), ascending
    uint64_t thr[kMaxTimeBuckets - 1];
};

struct SeqInfo {
    int64_t start;
    int L, c, t, E;
    bool ok;
    bool cfull;   // contextual rows see every key before the candidates (mask variant)
};

__device__ __forceinline__ void flag_error(const DevParams &p, int bits)
{
    atomicOr(p.status, bits);
}

// Reads and validates sequence b.  Invalid sequences are reported and skipped.
__device__ __forceinline__ SeqInfo load_seq(const DevParams &p, int b, bool report)
{
    SeqInfo s;
    int64_t a = p.offsets[b], e = p.offsets[b + 1];
    int64_t L = e - a;
    s.start = a;
    s.c = p.ctx ? p.ctx[b] : 0;
    s.t = p.tgt ? p.tgt[b] : 0;
    s.ok = true;
    s.cfull = (p.flags & HSTU_FLAG_CTX_SEES_HISTORY) != 0;
    int bits = 0;
    if (a < 0 || L < 0 || e > p.T) { bits |= HSTU_DEV_BAD_OFFSETS; }
    // the offsets must start at row 0 and end at row T
    if ((b == 0 && a != 0) || (b == p.B - 1 && e != p.T)) { bits |= HSTU_DEV_BAD_OFFSETS; }
    if (L > p.N) { bits |= HSTU_DEV_SEQ_TOO_LONG; }
    if (bits == 0 && (s.c < 0 || s.t < 0 || (int64_t)s.c + s.t > L)) bits |= HSTU_DEV_BAD_COUNTS;
    if (bits) {
        s.ok = false;
        if (report) flag_error(p, bits);
        L = 0;
    }
    s.L = (int)L;
    s.E = s.L - s.t;
    return s;
}

// Token rows that sequence b leaves without a computed output, clipped to [0, T): its own
// rows when it is skipped for invalid data, and for the first (last) sequence the rows
// before seq_offsets[0] (from seq_offsets[B] on).  The kernels that write per-token outputs
// zero these rows, so that every output row is defined whenever the offsets are
// non-decreasing (overlapping sequences leave the overlap unspecified).
struct RowRange {
    int64_t a, e;
};

__device__ __forceinline__ int skipped_rows(const DevParams &p, int b, RowRange (&r)[3])
{
    int n = 0;
    const int64_t a = p.offsets[b], e = p.offsets[b + 1];
    if (!load_seq(p, b, false).ok) r[n++] = RowRange{max(a, (int64_t)0), min(e, p.T)};
    if (b == 0 && a > 0) r[n++] = RowRange{0, min(a, p.T)};
    if (b == p.B - 1 && e < p.T) r[n++] = RowRange{max(e, (int64_t)0), p.T};
    return n;
}

// Zeroes rows [r.a, r.e) of a row-major array with `width` elements per row, element-wise
// by `nthr` threads (tid = this thread's index among them).  Rare path: invalid data only.
template <typename T>
__device__ __forceinline__ void zero_rows(T *base, int64_t width, const RowRange &r, int tid,
                                          int nthr)
{
    if (!base || r.e <= r.a) return;
    for (int64_t x = r.a * width + tid; x < r.e * width; x += nthr) base[x] = T(0.f);
}

// Tiles of 128 rows of each sequence (ceil(L/128), saturated at 255; 0 for an invalid
// sequence, which is reported here), cached in shared memory by the persistent kernels so
// that their work-unit iterators step over units past a sequence's end without a chain of
// global loads.  A static array: its address is a constant, so the iterators keep no
// pointer to it.  Batches of more than kSeqTileCache sequences skip the cache.
constexpr int kSeqTileCache = 2048;
static __shared__ uint8_t s_seq_tiles[kSeqTileCache];

__device__ __forceinline__ void fill_seq_tiles(const DevParams &p, int nthreads)
{
    if (p.B > kSeqTileCache) return;
    for (int b = threadIdx.x; b < p.B; b += nthreads) {
        const SeqInfo s = load_seq(p, b, true);
        s_seq_tiles[b] = (uint8_t)min((s.L + 127) / 128, 255);
    }
}

// False only when the cache shows that sequence b has no tile t.
__device__ __forceinline__ bool seq_may_have_tile(const DevParams &p, int b, int t)
{
    if (p.B > kSeqTileCache) return true;
    const int n = s_seq_tiles[b];
    return t < n || n == 255;
}

// Programmatic dependent launch.  A kernel started with launch_pdl may begin (its set-up:
// tables, shared memory, TMEM) while the kernel ahead of it on the stream is still running.
// grid_dep_wait() blocks until that kernel has completed and its writes are visible (a no-op
// for a normal launch); grid_dep_release() lets the kernel behind this one start early.
__device__ __forceinline__ void grid_dep_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void grid_dep_release()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Transposes 16-byte chunks within groups of NCH lanes: on entry lane l holds chunks
// 0..NCH-1 of row l; on exit lane l, j = l % NCH, holds chunk j of rows l - j .. l - j +
// NCH-1 (slot c = row l - j + c).  Lets the NCH lanes of a group write one row's NCH
// chunks side by side (whole 128-byte lines for NCH = 8) instead of each lane writing its
// own row.  Butterfly of xor shuffles, log2(NCH) rounds.
template <int NCH>
__device__ __forceinline__ void transpose_chunks(float4 (&x)[NCH])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int m = NCH / 2; m >= 1; m >>= 1) {
        const bool hi = (lane & m) != 0;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            if (c & m) continue;
            const float4 snd = hi ? x[c] : x[c | m];
            float4 rcv;
            rcv.x = __shfl_xor_sync(0xffffffffu, snd.x, m);
            rcv.y = __shfl_xor_sync(0xffffffffu, snd.y, m);
            rcv.z = __shfl_xor_sync(0xffffffffu, snd.z, m);
            rcv.w = __shfl_xor_sync(0xffffffffu, snd.w, m);
            if (hi) x[c] = rcv; else x[c | m] = rcv;
        }
    }
}

// p(x): candidates take the last history position.
__device__ __forceinline__ int clamp_pos(int x, int E) { return (E > 0 && x >= E) ? E - 1 : x; }

// Index into the rel table of positions with p(i) - p(j) = d: clamp(d, 0, R-1), or, with the
// |p(i) - p(j)| variant, min(|d|, R-1).
__device__ __forceinline__ int rel_index(int d, int R, bool rabs)
{
    if (d < 0) d = rabs ? -d : 0;
    return d > R - 1 ? R - 1 : d;
}

__device__ __forceinline__ bool pair_valid(int i, int j, const SeqInfo &s, int W)
{
    if (j >= s.E) return i == j;          // candidate key: itself only
    if (i < s.c) return s.cfull || j < s.c;   // contextual row: prefix (variant: all history)
    if (j < s.c) return true;             // contextual key: every row
    int pi = clamp_pos(i, s.E);
    return j <= pi && (W <= 0 || pi - j <= W);
}

// True when some pair of rows [i0,i1] x keys [j0,j1] (inclusive) is valid.  Never false
// for a tile that holds a valid pair.
__device__ __forceinline__ bool tile_any_valid(int i0, int i1, int j0, int j1, const SeqInfo &s,
                                               int W)
{
    i1 = min(i1, s.L - 1);
    j1 = min(j1, s.L - 1);
    if (i0 > i1 || j0 > j1) return false;
    if (j0 < s.c) return true;                              // contextual keys: every row
    if (s.cfull && i0 < s.c && j0 < s.E) return true;       // variant: contextual rows see all
    int a = max(j0, s.E);
    if (a <= j1 && max(i0, a) <= min(i1, j1)) return true;  // candidate diagonal
    int ha = max(j0, s.c), hb = min(j1, s.E - 1);           // history keys
    if (ha > hb) return false;
    int ra = max(i0, s.c), rb = min(i1, s.E - 1);           // history rows
    if (ra <= rb && rb >= ha && (W <= 0 || ra - hb <= W)) return true;
    if (i1 >= s.E && (W <= 0 || (s.E - 1) - hb <= W)) return true;   // candidate rows
    return false;
}

// True when every pair of the (in-sequence) tile is valid and no pair needs the
// candidate clamp: the bias then is rel[i-j] + tb[bucket(|ts_i - ts_j|)] without clamping
// of positions.  Conservative: may return false for a full tile.
__device__ __forceinline__ bool tile_all_valid(int i0, int i1, int j0, int j1, const SeqInfo &s,
                                               int W)
{
    if (i1 >= s.L || j1 >= s.L || i1 >= s.E) return false;
    if (j1 < s.c) return true;                               // all contextual keys
    if (i0 < s.c || j1 >= s.E) return false;
    // history x history (or contextual keys): needs j <= i for all, window for all
    int jmin_hist = max(j0, s.c);
    if (j1 > i0) return false;
    if (W > 0 && i1 - jmin_hist > W) return false;
    return true;
}

__device__ __forceinline__ uint64_t abs_diff_u64(int64_t a, int64_t b)
{
    return a >= b ? (uint64_t)a - (uint64_t)b : (uint64_t)b - (uint64_t)a;
}

// Number of thresholds <= dt (thresholds ascending, in shared or constant memory).
__device__ __forceinline__ int bucket_search(const uint64_t *thr, int n, uint64_t dt)
{
    int lo = 0, hi = n;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if (thr[mid] <= dt) lo = mid + 1; else hi = mid;
    }
    return lo;
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x)
{
    return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x)
{
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float silu_f32(float x) { return x / (1.0f + expf(-x)); }

__device__ __forceinline__ float silu_grad_f32(float x)
{
    float sg = 1.0f / (1.0f + expf(-x));
    return sg * (1.0f + x * (1.0f - sg));
}

}  // namespace hstu
