// jagged.cu -- jagged-tensor operations around the attention: Stochastic Length selection,
// row gathering and per-sequence concatenation.
//
//  - "Scaling HSTU: ragged execution, candidate amortization and content features",
//    section "Variable length is a central systems issue": jagged storage = values + offsets;
//    Stochastic Length samples sequence lengths during training.  Reading (the page gives no
//    formula): a sequence keeps its contextual prefix and its candidates, and of its h
//    history tokens the min(h, budget) whose random keys are smallest (the earlier position
//    first on equal keys), in their original order.  The random keys are inputs.
//  - "HSTU-MUSA: HSTU for Moore Threads (MUSA)", section "Project Structure": jagged tensor
//    concatenation: per sequence, the parts one after another.
#include "kernels.h"

namespace hstu {

namespace {

constexpr int kSelThreads = 256;

// Length of sequence b after Stochastic Length (0 for a sequence with invalid counts).
__device__ __forceinline__ int64_t sl_new_len(const DevParams &p, int b, int budget, bool report)
{
    const SeqInfo s = load_seq(p, b, report);
    if (!s.ok) return 0;
    const int h = s.E - s.c;
    return (int64_t)s.c + s.t + (h > budget ? budget : h);
}

// One block: new offsets [B + 1] as the exclusive prefix sum of the new lengths.
__global__ void __launch_bounds__(1024) sl_offsets_kernel(const __grid_constant__ DevParams p,
                                                          int budget, int64_t *out_offsets)
{
    __shared__ int64_t part[1024];
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (p.B + nt - 1) / nt, b0 = tid * per, b1 = min(p.B, b0 + per);
    int64_t sum = 0;
    for (int b = b0; b < b1; ++b) sum += sl_new_len(p, b, budget, true);
    part[tid] = sum;
    __syncthreads();
    for (int o = 1; o < nt; o <<= 1) {             // inclusive scan of the per-thread sums
        const int64_t v = tid >= o ? part[tid - o] : 0;
        __syncthreads();
        part[tid] += v;
        __syncthreads();
    }
    int64_t run = tid > 0 ? part[tid - 1] : 0;
    if (tid == 0) out_offsets[0] = 0;
    for (int b = b0; b < b1; ++b) {
        run += sl_new_len(p, b, budget, false);
        out_offsets[b + 1] = run;
    }
}

// Monotone map of a float's bits to an unsigned integer (order of the values, NaN excluded).
__device__ __forceinline__ uint32_t ordered_bits(float x)
{
    const uint32_t u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One block per sequence: the kept rows, in order, at out_rows[out_offsets[b] ...].
__global__ void __launch_bounds__(kSelThreads)
    sl_select_kernel(const __grid_constant__ DevParams p, const float *__restrict__ keys,
                     int budget, const int64_t *__restrict__ out_offsets,
                     int64_t *__restrict__ out_rows)
{
    __shared__ uint32_t hist[256];
    __shared__ uint64_t sel[2];                    // prefix, remaining rank
    __shared__ uint32_t wsum[kSelThreads / 32];
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const SeqInfo s = load_seq(p, b, false);
    if (!s.ok) return;
    const int h = s.E - s.c;
    int64_t *dst = out_rows + out_offsets[b];
    if (h <= budget) {                              // everything kept
        for (int j = tid; j < s.L; j += kSelThreads) dst[j] = s.start + j;
        return;
    }
    // The budget-th smallest of the unique 64-bit values (key bits, position) over the
    // history positions, by eight passes of an 8-bit most-significant-digit radix select.
    auto value = [&](int j) -> uint64_t {
        return ((uint64_t)ordered_bits(keys[s.start + j]) << 32) | (uint32_t)j;
    };
    if (tid == 0) {
        sel[0] = 0;
        sel[1] = (uint64_t)budget;                  // rank (1-based) still to find
    }
    uint64_t mask = 0;
    for (int pass = 0; pass < 8; ++pass) {
        const int shift = 56 - 8 * pass;
        for (int x = tid; x < 256; x += kSelThreads) hist[x] = 0;
        __syncthreads();
        const uint64_t prefix = sel[0];
        for (int j = s.c + tid; j < s.E; j += kSelThreads) {
            const uint64_t v = value(j);
            if ((v & mask) == prefix) atomicAdd(&hist[(v >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid == 0) {
            uint64_t rem = sel[1], cum = 0;
            int d = 0;
            for (; d < 255 && cum + hist[d] < rem; ++d) cum += hist[d];
            sel[0] = prefix | ((uint64_t)d << shift);
            sel[1] = rem - cum;
        }
        mask |= (uint64_t)255u << shift;
        __syncthreads();
    }
    const uint64_t thr = sel[0];
    // order-preserving compaction: kept = contextual, candidate, or history value <= thr
    int64_t run = 0;
    for (int j0 = 0; j0 < s.L; j0 += kSelThreads) {
        const int j = j0 + tid;
        const bool keep = j < s.L && (j < s.c || j >= s.E || value(j) <= thr);
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) wsum[wid] = __popc(bal);
        __syncthreads();
        int64_t before = run;
        int64_t total = 0;
        for (int w = 0; w < kSelThreads / 32; ++w) {
            if (w < wid) before += wsum[w];
            total += wsum[w];
        }
        if (keep) dst[before + __popc(bal & ((1u << lane) - 1u))] = s.start + j;
        run += total;
        __syncthreads();
    }
}

__global__ void gather_rows_kernel(const uint8_t *__restrict__ src, int64_t row_bytes,
                                   const int64_t *__restrict__ rows,
                                   const int64_t *__restrict__ n_rows, int64_t max_rows,
                                   uint8_t *__restrict__ dst)
{
    const int64_t n = min(*n_rows, max_rows);
    const bool vec = (row_bytes & 15) == 0 && (((uintptr_t)src | (uintptr_t)dst) & 15) == 0;
    const int64_t per = vec ? row_bytes / 16 : row_bytes;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n * per;
         x += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = x / per, c = x % per;
        const int64_t sr = rows[r];
        if (vec)
            reinterpret_cast<uint4 *>(dst + r * row_bytes)[c] =
                reinterpret_cast<const uint4 *>(src + sr * row_bytes)[c];
        else
            dst[r * row_bytes + c] = src[sr * row_bytes + c];
    }
}

struct ConcatArgs {
    const uint8_t *values[kMaxConcatParts];
    const int64_t *offsets[kMaxConcatParts];
    int n_parts, B;
    int64_t row_bytes;
    uint8_t *out;
    int64_t *out_offsets;
};

// One block per sequence: its rows of part 0, then part 1, ...
__global__ void concat_kernel(const __grid_constant__ ConcatArgs a)
{
    const int b = blockIdx.x;
    int64_t o = 0;
    for (int q = 0; q < a.n_parts; ++q) o += a.offsets[q][b];
    if (threadIdx.x == 0) {
        int64_t e = 0;
        for (int q = 0; q < a.n_parts; ++q) e += a.offsets[q][b + 1];
        a.out_offsets[b + 1] = e;
        if (b == 0) a.out_offsets[0] = 0;
    }
    const bool vec = (a.row_bytes & 15) == 0;
    for (int q = 0; q < a.n_parts; ++q) {
        const int64_t r0 = a.offsets[q][b], n = a.offsets[q][b + 1] - r0;
        const uint8_t *src = a.values[q] + r0 * a.row_bytes;
        uint8_t *dst = a.out + o * a.row_bytes;
        const bool v = vec && (((uintptr_t)src | (uintptr_t)dst) & 15) == 0;
        const int64_t total = v ? n * a.row_bytes / 16 : n * a.row_bytes;
        for (int64_t x = threadIdx.x; x < total; x += blockDim.x) {
            if (v) reinterpret_cast<uint4 *>(dst)[x] = reinterpret_cast<const uint4 *>(src)[x];
            else dst[x] = src[x];
        }
        o += n > 0 ? n : 0;
    }
}

}  // namespace

cudaError_t launch_stochastic_length(const DevParams &p, const float *keys, int budget,
                                     int64_t *out_rows, int64_t *out_offsets, cudaStream_t st)
{
    sl_offsets_kernel<<<1, 1024, 0, st>>>(p, budget, out_offsets);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || p.B == 0) return e;
    sl_select_kernel<<<p.B, kSelThreads, 0, st>>>(p, keys, budget, out_offsets, out_rows);
    return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void *src, int64_t row_bytes, const int64_t *rows,
                               const int64_t *n_rows, int64_t max_rows, void *dst,
                               cudaStream_t st)
{
    if (max_rows <= 0) return cudaSuccess;
    const int64_t per = (row_bytes & 15) == 0 ? row_bytes / 16 : row_bytes;
    int64_t blocks = (max_rows * per + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    gather_rows_kernel<<<(unsigned)blocks, 256, 0, st>>>(
        reinterpret_cast<const uint8_t *>(src), row_bytes, rows, n_rows, max_rows,
        reinterpret_cast<uint8_t *>(dst));
    return cudaGetLastError();
}

cudaError_t launch_jagged_concat(int n_parts, const void *const *values,
                                 const int64_t *const *offsets, int B, int64_t row_bytes,
                                 void *out, int64_t *out_offsets, cudaStream_t st)
{
    ConcatArgs a;
    for (int q = 0; q < kMaxConcatParts; ++q) {
        a.values[q] = q < n_parts ? reinterpret_cast<const uint8_t *>(values[q]) : nullptr;
        a.offsets[q] = q < n_parts ? offsets[q] : nullptr;
    }
    a.n_parts = n_parts;
    a.B = B;
    a.row_bytes = row_bytes;
    a.out = reinterpret_cast<uint8_t *>(out);
    a.out_offsets = out_offsets;
    if (B <= 0) return cudaSuccess;
    concat_kernel<<<B, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace hstu
