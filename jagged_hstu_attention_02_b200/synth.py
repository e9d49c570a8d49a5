"""Seeded synthetic jagged batches for jagged HSTU attention.

This module only draws inputs.  It holds none of the method's arithmetic, so the
oracle side and the CUDA side can both consume what it produces without sharing
any computation.

Value distributions and structure follow the workloads the HSTU pages describe:
 - "Scaling HSTU: ragged execution, candidate amortization and content features",
   section "Variable length is a central systems issue": lengths [10, 100, 1000];
 - "HSTU-MUSA: HSTU for Moore Threads (MUSA)", section "Accuracy Alignment":
   batch 128, hidden 128, 4 heads, bf16, at most 20 candidates, seed 1234.
MovieLens-20M itself is not available; Zipf history lengths and exponential
time gaps stand in for its length and inter-event-time distributions.

Every array is a numpy array.  Floating-point tensors are float32 arrays whose
values are exactly representable in the batch dtype ("bf16" values are rounded
to bfloat16 here, round-to-nearest-even, and kept as float32 so that both sides
read bit-identical numbers).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

BASE_SEED = 1234


@dataclasses.dataclass
class Batch:
    num_heads: int
    d_qk: int
    d_v: int
    dtype: str                      # "f32" or "bf16"
    seq_offsets: np.ndarray         # int64 [B+1]
    num_contextuals: Optional[np.ndarray]   # int32 [B] or None (= all zero)
    num_targets: Optional[np.ndarray]       # int32 [B] or None (= all zero)
    timestamps: Optional[np.ndarray]        # int64 [T] or None (no time bias)
    q: np.ndarray                   # float32 [T, H, d_qk]
    k: np.ndarray                   # float32 [T, H, d_qk]
    v: np.ndarray                   # float32 [T, H, d_v]
    u: np.ndarray                   # float32 [T, H*d_v]
    rel_bias: Optional[np.ndarray]  # float32 [R] or None
    time_bias: Optional[np.ndarray] # float32 [NB] or None
    alpha: float                    # exactly representable in float32
    max_attn_len: int               # <= 0: unlimited
    max_seqlen: int                 # N: the batch max of the sequence lengths
    time_bucket_div: float = 0.301
    ln_eps: float = float(np.float32(1e-5))
    dout: Optional[np.ndarray] = None       # float32 [T, H*d_v] (backward workloads)
    name: str = ""
    mask_flags: int = 0             # mask variants: 1 contextual rows see the history, 2 |rel|

    @property
    def batch(self) -> int:
        return int(self.seq_offsets.shape[0] - 1)

    @property
    def total_tokens(self) -> int:
        return int(self.seq_offsets[-1])

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.seq_offsets)

    @property
    def rel_bias_len(self) -> int:
        return 0 if self.rel_bias is None else int(self.rel_bias.shape[0])

    @property
    def time_bias_len(self) -> int:
        return 0 if self.time_bias is None else int(self.time_bias.shape[0])


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to `dtype` (RN-even) and return them as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype != "bf16":
        raise ValueError(dtype)
    bits = x.view(np.uint32).astype(np.uint64)
    # round-to-nearest-even on the upper 16 bits (inputs are finite normal draws)
    lsb = (bits >> 16) & 1
    bits = (bits + 0x7FFF + lsb) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32)


def f32(x: float) -> float:
    return float(np.float32(x))


def make_batch(rng: np.random.Generator, lengths: Sequence[int], num_heads: int, d_qk: int,
               d_v: int, dtype: str, *, contextuals=0, targets=0, max_attn_len: int = 0,
               rel_bias_len: int = 0, time_bias_len: int = 0, time_gap_mean: float = 3600.0,
               ts_base: int = 1_600_000_000, alpha: Optional[float] = None,
               max_seqlen: Optional[int] = None, bias_std: float = 0.1,
               with_dout: bool = False, name: str = "", mask_flags: int = 0) -> Batch:
    """Draw one jagged batch.  Draw order: timestamps, q, k, v, u, rel table, time table, dout.

    `contextuals` / `targets` are an int (same for every sequence) or a per-sequence list.
    """
    lengths = np.asarray(lengths, dtype=np.int64)
    B = int(lengths.shape[0])
    offsets = np.zeros(B + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(lengths)
    T = int(offsets[-1])
    H = num_heads

    def per_seq(val):
        if val is None:
            return None
        a = np.broadcast_to(np.asarray(val, dtype=np.int32), (B,)).copy()
        return a

    ctx = per_seq(contextuals)
    tgt = per_seq(targets)

    ts = None
    if time_bias_len > 0:
        ts = np.empty(T, dtype=np.int64)
        for b in range(B):
            L = int(lengths[b])
            gaps = rng.exponential(time_gap_mean, size=L)
            ts[offsets[b]:offsets[b + 1]] = ts_base + np.floor(np.cumsum(gaps)).astype(np.int64)

    q = round_to_dtype(rng.standard_normal((T, H, d_qk), dtype=np.float32), dtype)
    k = round_to_dtype(rng.standard_normal((T, H, d_qk), dtype=np.float32), dtype)
    v = round_to_dtype(rng.standard_normal((T, H, d_v), dtype=np.float32), dtype)
    u = round_to_dtype(rng.standard_normal((T, H * d_v), dtype=np.float32), dtype)
    rel = None
    if rel_bias_len > 0:
        rel = (rng.standard_normal(rel_bias_len) * bias_std).astype(np.float32)
    tb = None
    if time_bias_len > 0:
        tb = (rng.standard_normal(time_bias_len) * bias_std).astype(np.float32)
    dout = None
    if with_dout:
        dout = round_to_dtype(rng.standard_normal((T, H * d_v), dtype=np.float32), dtype)
    if alpha is None:
        alpha = 1.0 / math.sqrt(d_qk)
    if max_seqlen is None:
        max_seqlen = int(lengths.max()) if B > 0 else 0
    return Batch(num_heads=H, d_qk=d_qk, d_v=d_v, dtype=dtype, seq_offsets=offsets,
                 num_contextuals=ctx, num_targets=tgt, timestamps=ts, q=q, k=k, v=v, u=u,
                 rel_bias=rel, time_bias=tb, alpha=f32(alpha), max_attn_len=int(max_attn_len),
                 max_seqlen=int(max_seqlen), dout=dout, name=name, mask_flags=int(mask_flags))


# ------------------------------------------------------------------ the five workloads

WORKLOADS = {
    0: "tiny-fp32 B=3 L=[10,100,1000] H=2 d=32 causal rel-bias",
    1: "movielens-shaped B=128 H=4 d=128 bf16 zipf-history + 1 ctx + 1..20 targets",
    2: "long-history B=32 H=4 d=128 bf16 L~U[512,4096] 4 ctx 64 targets",
    3: "windowed B=8 H=8 d=64 bf16 L~U[4096,16384] 8 ctx 32 targets W=1024",
    4: "training-backward movielens-shaped B=128 H=4 d=128 bf16 + dO",
}


def make_config(cfg: int, seed: Optional[int] = None, batch: Optional[int] = None) -> Batch:
    """The five workloads, each drawn from default_rng(1234 + cfg) unless `seed` is given.
    `batch` changes the number of sequences of the MovieLens-shaped workloads (1 and 4),
    e.g. to draw the global batch of a data-parallel run (128 per GPU)."""
    if seed is None:
        seed = BASE_SEED + (1 if cfg == 4 else cfg)
    if batch is not None and cfg not in (1, 4):
        raise ValueError("only the MovieLens-shaped workloads take a batch size")
    rng = np.random.default_rng(seed)
    if cfg == 0:
        lengths = [10, 100, 1000]
        return make_batch(rng, lengths, 2, 32, 32, "f32", rel_bias_len=1001,
                          max_seqlen=1000, name=WORKLOADS[0])
    if cfg in (1, 4):
        B = 128 if batch is None else int(batch)
        hist = np.clip(rng.zipf(1.2, size=B), 8, 200).astype(np.int64)
        tgt = rng.integers(1, 21, size=B).astype(np.int32)
        lengths = 1 + hist + tgt
        N = int(lengths.max())
        return make_batch(rng, lengths, 4, 128, 128, "bf16", contextuals=1, targets=tgt,
                          rel_bias_len=N + 1, time_bias_len=128, with_dout=(cfg == 4),
                          name=WORKLOADS[cfg])
    if cfg == 2:
        lengths = rng.integers(512, 4097, size=32)
        N = int(lengths.max())
        return make_batch(rng, lengths, 4, 128, 128, "bf16", contextuals=4, targets=64,
                          rel_bias_len=N + 1, time_bias_len=128, name=WORKLOADS[2])
    if cfg == 3:
        lengths = rng.integers(4096, 16385, size=8)
        return make_batch(rng, lengths, 8, 64, 64, "bf16", contextuals=8, targets=32,
                          max_attn_len=1024, rel_bias_len=1025, time_bias_len=128,
                          name=WORKLOADS[3])
    raise ValueError("unknown workload %r" % cfg)


def sub_batch(b, seqs):
    """The sequences `seqs` of batch b as a batch of their own (same N, same tables)."""
    seqs = list(seqs)
    offs = b.seq_offsets
    rows = np.concatenate([np.arange(offs[s], offs[s + 1]) for s in seqs]) if seqs else \
        np.zeros(0, dtype=np.int64)
    lengths = np.array([offs[s + 1] - offs[s] for s in seqs], dtype=np.int64)
    new_offs = np.zeros(len(seqs) + 1, dtype=np.int64)
    new_offs[1:] = np.cumsum(lengths)

    def pick(a):
        return None if a is None else np.ascontiguousarray(a[rows])

    def pick_seq(a):
        return None if a is None else np.ascontiguousarray(a[seqs])

    return dataclasses.replace(
        b, seq_offsets=new_offs, num_contextuals=pick_seq(b.num_contextuals),
        num_targets=pick_seq(b.num_targets), timestamps=pick(b.timestamps), q=pick(b.q),
        k=pick(b.k), v=pick(b.v), u=pick(b.u), dout=pick(b.dout))


def draw_dout(batch: Batch, seed: int) -> np.ndarray:
    """An upstream gradient dO ~ N(0,1) in the batch dtype, from its own seed."""
    rng = np.random.default_rng(seed)
    T, D = batch.u.shape
    return round_to_dtype(rng.standard_normal((T, D), dtype=np.float32), batch.dtype)
