"""fp64 reference of the HSTU layer around the attention: input LayerNorm, one fused U/V/Q/K
projection split into its four branches, the attention (the C oracle), the output
projection W_o and the residual.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline leg of the
benchmark may use this module; the product path never does.  numpy matmuls serve as steps;
nothing is shared with the CUDA library.

 - "HSTU tensor by tensor: SiLU aggregation, temporal bias and gating", section "Similar
   shape, different aggregation": o_i = W_o[U_i (.) Norm(sum_j A_ij V_j)] + x_i;
   section "Trace four projections": normalised inputs produce the U/V/Q/K projections, Q/K
   head dimensions may differ from U/V, a fused projection must be split to match the weight
   layout; "HSTU-MUSA: HSTU for Moore Threads (MUSA)", "Accuracy Alignment":
   add_uvqk_bias=True.
 - Readings (the pages give no more): the input normalisation is a LayerNorm over the model
   width without affine (eps as the attention's); the projection is linear plus bias, its
   columns ordered U | V | Q | K, each head-major (head h's d columns together); optionally
   (uvqk_silu) the SiLU of the original HSTU is applied to all four branches; W_o has a bias.
"""
from __future__ import annotations

import numpy as np

from . import oracle


def layer_norm(x, eps):
    x = np.asarray(x, np.float64)
    mu = x.mean(axis=1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def uvqk(xn, w, bias, H, d_qk, d_v, silu=False):
    """The fused projection and its split: (u [T, H*d_v], v [T,H,d_v], q [T,H,d_qk], k)."""
    y = np.asarray(xn, np.float64) @ np.asarray(w, np.float64)
    if bias is not None:
        y = y + np.asarray(bias, np.float64)
    if silu:
        y = y / (1.0 + np.exp(-y))
    T = y.shape[0]
    a, b_, c_ = H * d_v, 2 * H * d_v, 2 * H * d_v + H * d_qk
    return (y[:, :a], y[:, a:b_].reshape(T, H, d_v), y[:, b_:c_].reshape(T, H, d_qk),
            y[:, c_:].reshape(T, H, d_qk))


def out_proj(z, w_o, b_o, x):
    o = np.asarray(z, np.float64) @ np.asarray(w_o, np.float64)
    if b_o is not None:
        o = o + np.asarray(b_o, np.float64)
    if x is not None:
        o = o + np.asarray(x, np.float64)
    return o


def layer_fwd(batch, x, w_uvqk, b_uvqk, w_o, b_o, silu=False):
    """The layer on the jagged batch `batch` (its q/k/v/u are replaced by the projections of
    x; its offsets, counts, stamps, tables and scalars are used).  Returns dict(xn, u, v, q,
    k, attn (the attention output), o)."""
    import dataclasses
    H, dqk, dv = batch.num_heads, batch.d_qk, batch.d_v
    xn = layer_norm(x, batch.ln_eps)
    u, v, q, k = uvqk(xn, w_uvqk, b_uvqk, H, dqk, dv, silu)
    b = dataclasses.replace(batch, q=q, k=k, v=v, u=u)
    attn = oracle.fwd(b)["out"]
    return dict(xn=xn, u=u, v=v, q=q, k=k, attn=attn, o=out_proj(attn, w_o, b_o, x))
