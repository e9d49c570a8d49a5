// debug.cu -- test hooks: export the mask of one sequence as the device evaluates it, one
// bit per (query, key) pair.
//
//  - debug_mask_kernel: the pair predicate pair_valid of common.cuh (the CUDA-core kernels).
//  - debug_kernel_mask_kernel: the decisions of the tensor-core kernels (tiles.cuh): a pair
//    is valid when its tile is visited (TileIter / QTileIter) and its 32-wide block marks it
//    (fwd_block_mask / bwd_block_mask), for pairs past the sequence's end too, so a test
//    can check that the padding rows and keys of a tile stay masked.
#include "kernels.h"
#include "tiles.cuh"

namespace hstu {

__global__ void debug_mask_kernel(const __grid_constant__ DevParams p, int seq, int seq_len,
                                  uint32_t *bits)
{
    const SeqInfo s = load_seq(p, seq, false);
    const int L = min(seq_len, s.L);
    const int64_t n = (int64_t)seq_len * seq_len;
    const int64_t words = (n + 31) / 32;
    for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words;
         w += (int64_t)gridDim.x * blockDim.x) {
        uint32_t word = 0;
        for (int b = 0; b < 32; ++b) {
            const int64_t idx = w * 32 + b;
            if (idx >= n) break;
            const int i = (int)(idx / seq_len), j = (int)(idx % seq_len);
            if (i < L && j < L && pair_valid(i, j, s, p.W)) word |= 1u << b;
        }
        bits[w] = word;
    }
}

cudaError_t launch_debug_mask(const DevParams &p, int seq, int seq_len, uint32_t *bits,
                              cudaStream_t st)
{
    const int64_t words = ((int64_t)seq_len * seq_len + 31) / 32;
    int64_t blocks = (words + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks < 1) blocks = 1;
    debug_mask_kernel<<<(unsigned)blocks, 256, 0, st>>>(p, seq, seq_len, bits);
    return cudaGetLastError();
}

// One thread per (query row, 32-key word) of rows [row0, row0 + nrows) x keys [0, nkeys).
__global__ void debug_kernel_mask_kernel(const __grid_constant__ DevParams p, int seq,
                                         int kernel, int row0, int nrows, int nkeys,
                                         uint32_t *bits)
{
    const SeqInfo s = load_seq(p, seq, false);
    const int wpr = nkeys / kBlk;                       // words per row
    const int64_t words = (int64_t)nrows * wpr;
    const int nt = (s.L + kTile - 1) / kTile;
    for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words;
         w += (int64_t)gridDim.x * blockDim.x) {
        const int i = row0 + (int)(w / wpr);
        const int jq = (int)(w % wpr) * kBlk;
        const int qt = i / kTile, kt = jq / kTile;
        uint32_t word = 0;
        if (kernel == 0) {
            // forward: a work unit per query tile inside the sequence; its visited key tiles
            if (qt < nt && kt < nt && fwd_visits(s, qt * kTile, kt, p.W))
                word = fwd_block_mask(s, qt * kTile, jq, i, p.W).bits;
        } else {
            // backward: a work unit per key tile; the query tiles it visits; each key lane
            // holds the bits of its 32-query block
            if (qt < nt && kt < nt && bwd_visits(s, kt * kTile, qt, p.W)) {
                const int iq = i / kBlk * kBlk;
                for (int c = 0; c < kBlk; ++c) {
                    const uint32_t col = bwd_block_mask(s, kt * kTile, iq, jq + c, p.W).bits;
                    word |= ((col >> (i - iq)) & 1u) << c;
                }
            }
        }
        bits[w] = word;
    }
}

cudaError_t launch_debug_kernel_mask(const DevParams &p, int seq, int kernel, int row0,
                                     int nrows, int nkeys, uint32_t *bits, cudaStream_t st)
{
    const int64_t words = (int64_t)nrows * (nkeys / kBlk);
    int64_t blocks = (words + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks < 1) blocks = 1;
    debug_kernel_mask_kernel<<<(unsigned)blocks, 256, 0, st>>>(p, seq, kernel, row0, nrows,
                                                                nkeys, bits);
    return cudaGetLastError();
}

}  // namespace hstu
