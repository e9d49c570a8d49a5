"""Host-side work accounting: valid pairs, FLOPs and algorithmic bytes.

 - "Scaling HSTU: ragged execution, candidate amortization and content features",
   section "Variable length is a central systems issue": padded vs ragged token
   positions and the dense / per-sequence pair-work ratio (theoretical work only).
 - The valid-pair count of one sequence follows the mask family named on
   "HSTU-MUSA: HSTU for Moore Threads (MUSA)", section "Mathematical Equivalence",
   in closed form (contextual prefix, causal history with an optional window W,
   candidates that see the prefix, the history and themselves).

FLOPs count valid (unmasked) pairs only:  fwd = P*H*2*(d_qk + d_v),
bwd = P*H*2*(2*d_qk + 2*d_v) (no recompute); bwd_recompute = P*H*2*(3*d_qk + 2*d_v).
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def padding_stats(lengths):
    """(padded token positions, ragged token positions, dense/per-sequence pair-work ratio)."""
    lengths = [int(x) for x in lengths]
    n = len(lengths)
    m = max(lengths) if lengths else 0
    padded = n * m
    ragged = sum(lengths)
    denom = sum(x * x for x in lengths)
    ratio = Fraction(n * m * m, denom) if denom else Fraction(0)
    return padded, ragged, ratio


def _capped_triangle(n: int, K) -> int:
    """sum_{m=1..n} min(m, K); K=None means no cap."""
    if n <= 0:
        return 0
    if K is None or n <= K:
        return n * (n + 1) // 2
    return K * (K + 1) // 2 + (n - K) * K


CTX_SEES_HISTORY = 1   # mask variant: contextual rows see every key before the candidates


def valid_pairs_seq(L: int, c: int = 0, t: int = 0, W: int = 0, flags: int = 0) -> int:
    """Number of valid (query, key) pairs of one sequence of length L."""
    if L <= 0:
        return 0
    E = L - t
    if E <= 0:
        return L                       # only candidates: each sees itself
    K = (W + 1) if W > 0 else None
    hist = E - c
    # contextual rows see the contextual prefix (or, variant, every key before the candidates)
    n = c * (E if flags & CTX_SEES_HISTORY else c)
    n += c * hist                      # history rows see every contextual key ...
    n += _capped_triangle(hist, K)     # ... and causal (windowed) history keys
    seen = hist if K is None else min(hist, K)
    n += t * (1 + c + seen)            # candidates: themselves, the prefix, the last history keys
    return n


def valid_pairs(batch) -> int:
    L = np.diff(batch.seq_offsets)
    B = len(L)
    c = batch.num_contextuals if batch.num_contextuals is not None else np.zeros(B, np.int32)
    t = batch.num_targets if batch.num_targets is not None else np.zeros(B, np.int32)
    f = int(getattr(batch, "mask_flags", 0))
    return int(sum(valid_pairs_seq(int(L[b]), int(c[b]), int(t[b]), int(batch.max_attn_len), f)
                   for b in range(B)))


def fwd_flops(batch, pairs=None) -> int:
    P = valid_pairs(batch) if pairs is None else pairs
    return P * batch.num_heads * 2 * (batch.d_qk + batch.d_v)


def bwd_flops(batch, pairs=None) -> int:
    P = valid_pairs(batch) if pairs is None else pairs
    return P * batch.num_heads * 2 * (2 * batch.d_qk + 2 * batch.d_v)


def bwd_flops_recompute(batch, pairs=None) -> int:
    P = valid_pairs(batch) if pairs is None else pairs
    return P * batch.num_heads * 2 * (3 * batch.d_qk + 2 * batch.d_v)


def elem_size(dtype: str) -> int:
    return {"f32": 4, "bf16": 2}[dtype]


def fwd_bytes(batch, training: bool = False) -> int:
    """Algorithmic HBM bytes of one forward: read Q, K, V, U (+ timestamps, metadata,
    tables), write O (+ fp32 Y, mean and rstd when training)."""
    T, H, s = batch.total_tokens, batch.num_heads, elem_size(batch.dtype)
    B = batch.batch
    n = T * (2 * H * batch.d_qk + 2 * H * batch.d_v) * s   # Q, K, V, U
    n += T * H * batch.d_v * s                               # O
    if batch.time_bias_len > 0:
        n += 8 * T
    n += 8 * (B + 1) + 4 * B * 2
    n += 4 * (batch.rel_bias_len + batch.time_bias_len)
    if training:
        n += 4 * T * H * batch.d_v + 8 * T
    return n


def bwd_bytes(batch) -> int:
    """Algorithmic HBM bytes of one backward: read dO, Q, K, V, U, fp32 Y, mean, rstd
    (+ timestamps, metadata, tables); write dQ, dK, dV, dU and the table gradients."""
    T, H, s = batch.total_tokens, batch.num_heads, elem_size(batch.dtype)
    B = batch.batch
    D = H * batch.d_v
    n = T * D * s                                            # dO
    n += T * (2 * H * batch.d_qk + 2 * H * batch.d_v) * s    # Q, K, V, U
    n += 4 * T * D + 8 * T                                   # Y, mean, rstd
    n += T * (2 * H * batch.d_qk + 2 * H * batch.d_v) * s    # dQ, dK, dV, dU
    if batch.time_bias_len > 0:
        n += 8 * T
    n += 8 * (B + 1) + 4 * B * 2
    n += 2 * 4 * (batch.rel_bias_len + batch.time_bias_len)
    return n


# ------------------------------------------------------------------ per-kernel bytes
#
# Algorithmic HBM bytes of each kernel of the path: what it must read and write at least
# once, whatever its tiling.  Bias tables, per-sequence counts and offsets are counted with
# the attention kernels.

def _meta_bytes(batch) -> int:
    B = batch.batch
    return 8 * (B + 1) + 4 * B * 2 + 4 * (batch.rel_bias_len + batch.time_bias_len)


def _ts_bytes(batch) -> int:
    return 8 * batch.total_tokens if batch.time_bias_len > 0 else 0


def fwd_attn_bytes(batch, training: bool = False, fused_norm: bool = False) -> int:
    """Forward attention kernel: read Q, K, V (+ timestamps, metadata, tables); write Y in
    fp32.  With the LayerNorm and U gating fused into it, also read U and write O, and write
    Y only when training (plus mean and rstd)."""
    T, H, s = batch.total_tokens, batch.num_heads, elem_size(batch.dtype)
    D = H * batch.d_v
    n = T * H * (2 * batch.d_qk + batch.d_v) * s + _ts_bytes(batch) + _meta_bytes(batch)
    if fused_norm:
        n += 2 * T * D * s                       # U read, O written
        if training:
            n += 4 * T * D + 8 * T               # Y, mean, rstd
    else:
        n += 4 * T * D                           # Y
    return n


def fwd_norm_bytes(batch, training: bool = False) -> int:
    """Separate LayerNorm + gating kernel: read Y (fp32) and U, write O (+ mean, rstd)."""
    T, s = batch.total_tokens, elem_size(batch.dtype)
    D = batch.num_heads * batch.d_v
    return T * D * (4 + 2 * s) + (8 * T if training else 0)


def bwd_norm_bytes(batch) -> int:
    """LayerNorm + gating backward: read dO, U, Y (fp32), mean, rstd; write dU and dY (fp32)."""
    T, s = batch.total_tokens, elem_size(batch.dtype)
    D = batch.num_heads * batch.d_v
    return T * D * (3 * s + 4 + 4) + 8 * T


def bwd_attn_bytes(batch) -> int:
    """Backward attention kernel: read Q, K, V, dY (fp32) (+ timestamps, metadata, tables);
    write dQ, dK, dV and the table gradients."""
    T, H, s = batch.total_tokens, batch.num_heads, elem_size(batch.dtype)
    D = H * batch.d_v
    n = 2 * T * H * (2 * batch.d_qk + batch.d_v) * s     # Q, K, V read; dQ, dK, dV written
    n += 4 * T * D                                        # dY
    n += _ts_bytes(batch) + _meta_bytes(batch) + 4 * (batch.rel_bias_len + batch.time_bias_len)
    return n


# ------------------------------------------------------------------ visited tiles

def tiles_with_pairs_seq(L: int, c: int = 0, t: int = 0, W: int = 0, tile: int = 128,
                         flags: int = 0) -> int:
    """(query tile, key tile) pairs of one sequence that hold at least one valid pair: the
    tiles a kernel that skips empty tiles must visit.  Per query tile, the union of its
    rows' valid key ranges: the contextual prefix (every row), the history rows' causal
    (windowed) ranges, the candidate rows' history range and their own positions."""
    if L <= 0:
        return 0
    E = L - t
    nt = (L + tile - 1) // tile
    total = 0
    for qt in range(nt):
        i0, i1 = qt * tile, min(qt * tile + tile, L) - 1
        keys = set()

        def add(a, b):
            if a <= b:
                keys.update(range(a // tile, b // tile + 1))

        if c > 0:
            add(0, c - 1)                                     # contextual keys / prefix rows
            if flags & CTX_SEES_HISTORY and i0 < c:
                add(0, E - 1)                                 # contextual rows: the history
        ra, rb = max(i0, c), min(i1, E - 1)                   # history rows
        if ra <= rb:
            add(max(c, ra - W) if W > 0 else c, rb)
        ca, cb = max(i0, E), i1                               # candidate rows
        if ca <= cb:
            if E > 0:
                add(max(c, E - 1 - W) if W > 0 else c, E - 1)
            add(ca, cb)                                       # themselves
        total += len(keys)
    return total


def tiles_with_pairs(batch, tile: int = 128) -> int:
    L = np.diff(batch.seq_offsets)
    B = len(L)
    c = batch.num_contextuals if batch.num_contextuals is not None else np.zeros(B, np.int32)
    t = batch.num_targets if batch.num_targets is not None else np.zeros(B, np.int32)
    f = int(getattr(batch, "mask_flags", 0))
    return int(sum(tiles_with_pairs_seq(int(L[b]), int(c[b]), int(t[b]),
                                        int(batch.max_attn_len), tile, f) for b in range(B)))
