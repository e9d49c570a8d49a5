"""Padded-dense fp64 formulation of jagged HSTU attention (numpy).

TEST INFRASTRUCTURE ONLY.  This is the second, independent formulation used to pin the
jagged C oracle: sequences are padded to [B, N] like the teaching code on
"HSTU tensor by tensor: SiLU aggregation, temporal bias and gating" (section
"Trace four projections": dense scores, SiLU, masked_fill after the nonlinearity,
then A @ V), with a key-padding mask, and the mask family is written as boolean
array algebra instead of the C oracle's per-pair branch cascade.

"Scaling HSTU: ragged execution, candidate amortization and content features",
section "Variable length is a central systems issue": jagged and padded storage
describe the same computation; this module checks that claim against the jagged oracle.
"""
from __future__ import annotations

import numpy as np


def _silu(x):
    return x / (1.0 + np.exp(-x))


CTX_SEES_HISTORY, REL_ABS = 1, 2   # mask variants, as in the jagged oracle


def _mask_dense(L, c, t, W, N, flags=0):
    """[N, N] bool mask of one sequence padded to N (rows = queries).  With CTX_SEES_HISTORY
    the contextual rows see every key before the candidates instead of the prefix only."""
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    E = L - t
    in_seq = (i < L) & (j < L)
    pi = np.where(i < E, i, E - 1) if E > 0 else i
    cand_key = j >= E
    ctx_row = i < c
    ctx_key = j < c
    window_ok = (pi - j <= W) if W > 0 else np.ones_like(cand_key)
    hist = (j <= pi) & window_ok
    ctx_row_keys = (j < E) if flags & CTX_SEES_HISTORY else ctx_key
    valid = np.where(cand_key, i == j, np.where(ctx_row, ctx_row_keys, ctx_key | hist))
    return valid & in_seq


def fwd(b):
    """Same outputs as the jagged oracle (out, y, mean, rstd), computed padded-dense."""
    B, H, dqk, dv = b.batch, b.num_heads, b.d_qk, b.d_v
    N = int(b.max_seqlen)
    D = H * dv
    T = b.total_tokens
    offs = b.seq_offsets
    q = np.zeros((B, N, H, dqk)); k = np.zeros((B, N, H, dqk)); v = np.zeros((B, N, H, dv))
    for s in range(B):
        L = offs[s + 1] - offs[s]
        q[s, :L] = b.q[offs[s]:offs[s + 1]]
        k[s, :L] = b.k[offs[s]:offs[s + 1]]
        v[s, :L] = b.v[offs[s]:offs[s + 1]]
    y_pad = np.zeros((B, N, H, dv))
    for s in range(B):
        L = int(offs[s + 1] - offs[s])
        c = 0 if b.num_contextuals is None else int(b.num_contextuals[s])
        t = 0 if b.num_targets is None else int(b.num_targets[s])
        E = L - t
        pos = np.arange(N)
        p = np.where(pos < E, pos, E - 1) if E > 0 else pos
        p = np.clip(p, 0, max(L - 1, 0))
        bias = np.zeros((N, N))
        flags = int(getattr(b, "mask_flags", 0))
        if b.rel_bias_len > 0:
            d = p[:, None] - p[None, :]
            r = np.clip(np.abs(d) if flags & REL_ABS else d, 0, b.rel_bias_len - 1)
            bias += np.asarray(b.rel_bias, np.float64)[r]
        if b.time_bias_len > 0 and L > 0:
            ts = np.zeros(N, dtype=np.int64)
            ts[:L] = b.timestamps[offs[s]:offs[s + 1]]
            dt = np.abs(ts[p][:, None] - ts[p][None, :]).astype(np.float64)
            bk = np.floor(np.log(dt + 1.0) / b.time_bucket_div)
            bk = np.clip(bk, 0, b.time_bias_len - 1).astype(np.int64)
            bias += np.asarray(b.time_bias, np.float64)[bk]
        m = _mask_dense(L, c, t, int(b.max_attn_len), N, flags)
        for h in range(H):
            scores = b.alpha * (q[s, :, h] @ k[s, :, h].T) + bias
            a = _silu(scores) / N
            a = np.where(m, a, 0.0)          # zero illegal coefficients after the SiLU
            y_pad[s, :, h] = a @ v[s, :, h]
    y = np.zeros((T, D))
    for s in range(B):
        L = offs[s + 1] - offs[s]
        y[offs[s]:offs[s + 1]] = y_pad[s, :L].reshape(L, D)
    mean = y.mean(axis=1)
    var = y.var(axis=1)
    rstd = 1.0 / np.sqrt(var + b.ln_eps)
    z = (y - mean[:, None]) * rstd[:, None]
    out = np.asarray(b.u, np.float64) * z
    return dict(out=out, y=y, mean=mean, rstd=rstd)
