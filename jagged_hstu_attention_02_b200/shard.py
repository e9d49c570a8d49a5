"""Data-parallel sharding of a jagged batch by whole sequences.

Sequences are independent once N (the batch max_seqlen that scales A) is fixed, and the
LayerNorm is per token, so a batch splits across ranks by whole sequences with no exchange
in the forward ("Scaling HSTU: ragged execution, candidate amortization and content
features", "Variable length is a central systems issue": the cost of a sequence is its
pair work, which grows with the square of its length).  Every rank must run with the
GLOBAL N.  In the backward, dQ/dK/dV/dU of a token stay on the rank that owns the
token; the bias tables are shared parameters, so their gradients are summed across ranks
with one all-reduce.

plan()        longest-processing-time assignment of sequences to ranks by valid pairs
local_rows()  token rows and re-based offsets of a rank's sequences
shard()       a rank's slice of the jagged inputs (token tensors, per-sequence counts)
allreduce_table_grads()  the one collective of a sharded training step
"""
from __future__ import annotations

import heapq
from typing import Dict, List, Optional, Sequence

import numpy as np

from . import accounting

# per-token inputs, gathered by row; per-sequence inputs, gathered by sequence
TOKEN_KEYS = ("q", "k", "v", "u", "timestamps", "dout")
SEQ_KEYS = ("num_contextuals", "num_targets")


def sequence_work(seq_offsets, num_contextuals=None, num_targets=None, max_attn_len=0,
                  mask_flags=0):
    """Valid (unmasked) pairs per sequence, per head."""
    offs = np.asarray(seq_offsets, dtype=np.int64)
    B = len(offs) - 1
    ctx = np.zeros(B, np.int64) if num_contextuals is None else np.asarray(num_contextuals)
    tgt = np.zeros(B, np.int64) if num_targets is None else np.asarray(num_targets)
    return np.array([accounting.valid_pairs_seq(int(offs[b + 1] - offs[b]), int(ctx[b]),
                                                int(tgt[b]), int(max_attn_len),
                                                int(mask_flags))
                     for b in range(B)], dtype=np.int64)


def plan(seq_offsets, world: int, num_contextuals=None, num_targets=None,
         max_attn_len: int = 0) -> List[np.ndarray]:
    """Sequence indices per rank (ascending): greedy longest-processing-time on the pair
    work (ties broken by token count, then index), each sequence to the least-loaded rank."""
    if world < 1:
        raise ValueError("world must be >= 1")
    offs = np.asarray(seq_offsets, dtype=np.int64)
    work = sequence_work(offs, num_contextuals, num_targets, max_attn_len)
    tokens = np.diff(offs)
    order = sorted(range(len(work)), key=lambda b: (-int(work[b]), -int(tokens[b]), b))
    heap = [(0, 0, r) for r in range(world)]          # (pairs, tokens, rank)
    out: List[List[int]] = [[] for _ in range(world)]
    for b in order:
        w, t, r = heapq.heappop(heap)
        out[r].append(b)
        heapq.heappush(heap, (w + int(work[b]), t + int(tokens[b]), r))
    return [np.array(sorted(x), dtype=np.int64) for x in out]


def local_rows(seq_offsets, seqs: Sequence[int]):
    """(token rows of `seqs` in the global layout, re-based offsets of the local batch)."""
    offs = np.asarray(seq_offsets, dtype=np.int64)
    seqs = [int(s) for s in seqs]
    lengths = np.array([offs[s + 1] - offs[s] for s in seqs], dtype=np.int64)
    rows = (np.concatenate([np.arange(offs[s], offs[s + 1], dtype=np.int64) for s in seqs])
            if seqs else np.zeros(0, dtype=np.int64))
    new_offs = np.zeros(len(seqs) + 1, dtype=np.int64)
    new_offs[1:] = np.cumsum(lengths)
    return rows, new_offs


def shard(inputs: Dict[str, object], seqs: Sequence[int]) -> Dict[str, object]:
    """A rank's slice of jagged inputs given as numpy arrays or torch tensors: token tensors
    gathered by row, per-sequence counts by sequence, `seq_offsets` re-based, everything
    else (bias tables) shared unchanged."""
    rows, new_offs = local_rows(inputs["seq_offsets"], seqs)
    seq_idx = np.asarray(list(seqs), dtype=np.int64)
    out = dict(inputs)
    for key in TOKEN_KEYS + SEQ_KEYS:
        a = inputs.get(key)
        if a is None:
            continue
        idx = rows if key in TOKEN_KEYS else seq_idx
        out[key] = _take(a, idx)
    off = inputs["seq_offsets"]
    out["seq_offsets"] = _like(off, new_offs)
    return out


def allreduce_table_grads(d_rel, d_time, group=None):
    """Sums the bias-table gradients of all ranks in place with one all-reduce (the two
    tables travel in one buffer)."""
    import torch
    import torch.distributed as dist

    parts = [t for t in (d_rel, d_time) if t is not None]
    if not parts:
        return
    flat = torch.cat([t.reshape(-1) for t in parts])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    pos = 0
    for t in parts:
        n = t.numel()
        t.copy_(flat[pos:pos + n].view_as(t))
        pos += n


def _take(a, idx: np.ndarray):
    if isinstance(a, np.ndarray):
        return np.ascontiguousarray(a[idx])
    import torch
    return a.index_select(0, torch.as_tensor(idx, device=a.device)).contiguous()


def _like(ref, arr: np.ndarray):
    if isinstance(ref, np.ndarray):
        return arr.astype(ref.dtype)
    import torch
    return torch.as_tensor(arr, dtype=ref.dtype, device=ref.device)
