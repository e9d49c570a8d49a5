"""Plain reference implementations of the jagged-tensor operations around the attention:
Stochastic Length selection, row gathering and per-sequence concatenation.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline leg of the
benchmark may use this module; the product path never does.  Plain Python loops over
sequences and tokens, written from the definitions below; no code shared with the CUDA
library.

 - "Scaling HSTU: ragged execution, candidate amortization and content features", section
   "Variable length is a central systems issue": jagged storage is concatenated values plus
   offsets; Stochastic Length samples sequence lengths during training, changing the
   computation (not only the storage).  Reading used here (the page gives no formula):
   every sequence keeps its contextual prefix and its candidates, and of its h history
   tokens the min(h, budget) whose random keys are smallest (ties: the earlier position
   first), in their original order.  The random keys are inputs.
 - "HSTU-MUSA: HSTU for Moore Threads (MUSA)", section "Project Structure": jagged tensor
   concatenation (ops/jagged_concat.py): per sequence, the parts one after another.
"""
from __future__ import annotations

import numpy as np


def stochastic_length(offsets, num_contextuals, num_targets, keys, budget):
    """(kept global rows in output order, new offsets [B+1]) of Stochastic Length."""
    offsets = [int(x) for x in offsets]
    B = len(offsets) - 1
    rows, new_offs = [], [0]
    for b in range(B):
        a, e = offsets[b], offsets[b + 1]
        L = e - a
        c = 0 if num_contextuals is None else int(num_contextuals[b])
        t = 0 if num_targets is None else int(num_targets[b])
        E = L - t
        hist = list(range(c, E))
        if len(hist) > budget:
            ranked = sorted(hist, key=lambda j: (float(keys[a + j]), j))
            kept_hist = set(ranked[:budget])
        else:
            kept_hist = set(hist)
        for j in range(L):
            if j < c or j >= E or j in kept_hist:
                rows.append(a + j)
        new_offs.append(len(rows))
    return np.array(rows, dtype=np.int64), np.array(new_offs, dtype=np.int64)


def gather_rows(src, rows):
    """dst[i] = src[rows[i]]."""
    return np.stack([src[int(r)] for r in rows]) if len(rows) else src[:0].copy()


def jagged_concat(parts):
    """parts: list of (values [T_p, ...], offsets [B+1]).  Returns (values, offsets) with,
    for every sequence, the rows of part 0, then part 1, ... one after another."""
    B = len(parts[0][1]) - 1
    out, offs = [], [0]
    for b in range(B):
        for vals, o in parts:
            for r in range(int(o[b]), int(o[b + 1])):
                out.append(vals[r])
        offs.append(len(out))
    vals0 = parts[0][0]
    values = np.stack(out) if out else vals0[:0].copy()
    return values, np.array(offs, dtype=np.int64)
