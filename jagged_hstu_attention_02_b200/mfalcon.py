"""Candidate micro-batching with a cached history (M-FALCON), built from the library's calls.

"Scaling HSTU: ragged execution, candidate amortization and content features", section
"Many candidates make reuse valuable": scoring many candidates per user re-encodes the
history once per candidate unless candidate-independent work is reused, which is valid only
where the mask allows it.  Under target-group masking a candidate sees the history and
itself only, so:

 1. the history tokens (contextual prefix + history) run through the forward once, with no
    candidates: their outputs, and their K/V, are those of the full batch;
 2. the candidates run in micro-batches of at most `micro_batch` per user: each micro-batch
    is appended to its user's history (jagged concat on the device) and only the query
    tiles holding candidates are computed (HSTU_FLAG_CANDIDATES_ONLY);
 3. the candidates' rows are gathered and concatenated back in order.

Every step is a kernel of the library (forward attention, jagged concat, row gather); this
module only computes the micro-batch offsets from the host copy of the candidate counts.
Every call uses the batch's global max_seqlen, so the 1/N scale matches the full batch.
"""
from __future__ import annotations

import numpy as np
import torch

from . import ops


def _offsets(counts):
    o = np.zeros(len(counts) + 1, dtype=np.int64)
    o[1:] = np.cumsum(counts)
    return o


def mfalcon_fwd(hist, cand, *, micro_batch, max_seqlen, alpha, rel_bias=None, time_bias=None,
                max_attn_len=0, time_bucket_div=0.301, ln_eps=1e-5, mask_flags=0):
    """hist: dict(q, k, v, u, timestamps, seq_offsets, num_contextuals) of the contextual and
    history tokens of every user; cand: dict(q, k, v, u, seq_offsets) of the candidates
    (their timestamps are not used: a candidate takes its user's last history position).
    Returns (out of the history tokens [T_h, D], out of the candidates [T_c, D])."""
    if micro_batch < 1:
        raise ValueError("micro_batch must be >= 1")
    kw = dict(alpha=alpha, max_seqlen=max_seqlen, max_attn_len=max_attn_len,
              time_bucket_div=time_bucket_div, ln_eps=ln_eps)
    dev = hist["q"].device
    B = hist["seq_offsets"].numel() - 1
    # 1. the history, once
    out_h = ops.fwd(hist["q"], hist["k"], hist["v"], hist["u"], hist["seq_offsets"],
                    hist["num_contextuals"], None, hist.get("timestamps"), rel_bias, time_bias,
                    mask_flags=mask_flags, **kw)
    oc = cand["seq_offsets"].cpu().numpy()
    oh = hist["seq_offsets"].cpu().numpy()
    m = np.diff(oc)
    ts_h = hist.get("timestamps")
    D = hist["u"].shape[1]
    n_mb = int((m.max() + micro_batch - 1) // micro_batch) if B and m.max() > 0 else 0
    parts = []
    for k in range(n_mb):
        lo = np.minimum(m, k * micro_batch)
        hi = np.minimum(m, (k + 1) * micro_batch)
        cnt = hi - lo
        rows = np.concatenate([np.arange(oc[b] + lo[b], oc[b] + hi[b]) for b in range(B)])
        off_k = torch.from_numpy(_offsets(cnt)).to(dev)
        n_k = int(cnt.sum())
        rows_t = torch.from_numpy(rows.astype(np.int64)).to(dev)
        nk_t = off_k[-1:]
        # 2. the micro-batch after each user's history
        batch = {}
        for key in ("q", "k", "v", "u"):
            ck = ops.gather_rows(cand[key], rows_t, nk_t, n_k)
            batch[key], off_b = ops.jagged_concat([(hist[key], hist["seq_offsets"]), (ck, off_k)])
        if ts_h is not None:
            ts_c = torch.zeros(n_k, dtype=ts_h.dtype, device=dev)   # not read by the kernels
            batch["timestamps"], _ = ops.jagged_concat([(ts_h, hist["seq_offsets"]),
                                                        (ts_c, off_k)])
        else:
            batch["timestamps"] = None
        tgt = torch.from_numpy(cnt.astype(np.int32)).to(dev)
        out_k = ops.fwd(batch["q"], batch["k"], batch["v"], batch["u"], off_b,
                        hist["num_contextuals"], tgt, batch["timestamps"], rel_bias, time_bias,
                        mask_flags=mask_flags | ops.FLAG_CANDIDATES_ONLY, **kw)
        # 3. the candidates' rows of this micro-batch
        ob = _offsets(np.diff(oh) + cnt)
        crow = np.concatenate([np.arange(ob[b] + (oh[b + 1] - oh[b]), ob[b + 1])
                               for b in range(B)]).astype(np.int64)
        parts.append((ops.gather_rows(out_k, torch.from_numpy(crow).to(dev), nk_t, n_k), off_k))
    if not parts:
        return out_h, torch.empty((0, D), dtype=out_h.dtype, device=dev)
    out_c = parts[0][0]
    acc_off = parts[0][1]
    for start in range(1, len(parts), ops.MAX_CONCAT_PARTS - 1):
        chunk = [(out_c, acc_off)] + parts[start:start + ops.MAX_CONCAT_PARTS - 1]
        out_c, acc_off = ops.jagged_concat(chunk)
    return out_h, out_c
