// tiles.cuh -- which 128 x 128 tiles, and which pairs inside them, the tensor-core kernels
// treat as valid.  The forward and backward kernels and the test export of their masks
// (hstu_attn_debug_kernel_mask, debug.cu) all call these functions, so the export shows the
// decisions the kernels take, not a re-derivation of them.
//
// The mask itself is the family of "HSTU-MUSA: HSTU for Moore Threads (MUSA)", section
// "Mathematical Equivalence" (contextual bidirectional prefix, candidate position clamping,
// target group masking, max attention length), applied after the nonlinearity as "HSTU
// tensor by tensor: SiLU aggregation, temporal bias and gating", section "Do not copy
// softmax masking mechanically" requires.  Its exact reading is stated in
// include/hstu_attn.h.
#pragma once

#include "bias.cuh"

namespace hstu {

constexpr int kTile = 128;   // query and key tile height of both tensor-core kernels
constexpr int kBlk = 32;     // the 32-wide blocks inside a tile the epilogues decide on

// Forward: the key tiles of query tile [i0, i0+128) that hold a valid pair, from the last
// one down.  Valid pairs have j <= i, except contextual rows, which see the whole
// contextual prefix: the first candidate key tile is the later of the diagonal and the
// prefix's end.  Descending order puts the diagonal tile, the most expensive one of a unit
// (masks, clamped positions, many time buckets), first, where the double-buffered scores
// absorb the spread between warps.
struct TileIter {
    const SeqInfo &s;
    int i0, W, kt;
    // (with the variant in which contextual rows see the whole history, a tile holding
    // contextual rows starts from the last tile)
    __device__ TileIter(const SeqInfo &s_, int i0_, int W_)
        : s(s_), i0(i0_), W(W_),
          kt((s_.cfull && i0_ < s_.c)
                 ? (s_.L + kTile - 1) / kTile
                 : min((s_.L + kTile - 1) / kTile, max(i0_ / kTile, (s_.c - 1) / kTile) + 1)) {}
    __device__ bool next()
    {
        while (--kt >= 0)
            if (tile_any_valid(i0, i0 + kTile - 1, kt * kTile, kt * kTile + kTile - 1, s, W))
                return true;
        return false;
    }
};

// Backward: the query tiles [i0, i0+128) that see key tile [j0, j0+128), in ascending order.
struct QTileIter {
    const SeqInfo &s;
    int j0, W, qt, nqt;
    __device__ QTileIter(const SeqInfo &s_, int j0_, int W_)
        : s(s_), j0(j0_), W(W_), qt(-1), nqt((s_.L + kTile - 1) / kTile) {}
    __device__ bool next()
    {
        while (++qt < nqt)
            if (tile_any_valid(qt * kTile, qt * kTile + kTile - 1, j0, j0 + kTile - 1, s, W))
                return true;
        return false;
    }
};

// The valid pairs of one 32-wide block, as an epilogue lane sees them.  `full` (the same for
// every lane of the block) says that every pair is valid and no position needs the
// candidate clamp; the lane's `bits` are then all set.
struct BlockMask {
    bool full;
    uint32_t bits;
};

// Forward: keys [jq, jq+32) for query row i of the query tile that starts at i0 (bit c <->
// key jq + c).
__device__ __forceinline__ BlockMask fwd_block_mask(const SeqInfo &s, int i0, int jq, int i,
                                                    int W)
{
    BlockMask m;
    m.full = tile_all_valid(i0, i0 + kTile - 1, jq, jq + kBlk - 1, s, W);
    m.bits = m.full ? 0xFFFFFFFFu : (uint32_t)row_valid_bits(i, jq, s, W);
    return m;
}

// Backward: queries [iq, iq+32) that see key j of the key tile that starts at j0 (bit c <->
// query iq + c).
__device__ __forceinline__ BlockMask bwd_block_mask(const SeqInfo &s, int j0, int iq, int j,
                                                    int W)
{
    BlockMask m;
    m.full = tile_all_valid(iq, iq + kBlk - 1, j0, j0 + kTile - 1, s, W);
    m.bits = m.full ? 0xFFFFFFFFu : (uint32_t)col_valid_bits(j, iq, s, W);
    return m;
}

// True when the forward visits key tile kt for the query tile that starts at i0.
__device__ __forceinline__ bool fwd_visits(const SeqInfo &s, int i0, int kt, int W)
{
    TileIter t(s, i0, W);
    while (t.next())
        if (t.kt == kt) return true;
    return false;
}

// True when the backward visits query tile qt for the key tile that starts at j0.
__device__ __forceinline__ bool bwd_visits(const SeqInfo &s, int j0, int qt, int W)
{
    QTileIter t(s, j0, W);
    while (t.next())
        if (t.qt == qt) return true;
    return false;
}

}  // namespace hstu
