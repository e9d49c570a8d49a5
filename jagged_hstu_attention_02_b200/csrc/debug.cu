// debug.cu -- test hook: exports the mask of one sequence exactly as the kernels evaluate it
// (the pair_valid predicate of common.cuh), one bit per (query, key) pair.
#include "kernels.h"

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

}  // namespace hstu
