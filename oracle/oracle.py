"""ctypes front end of the fp64 CPU oracle (hstu_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline leg of
the benchmark may import this module; the product path never does.  It shares no code
with the CUDA library: it reads the seeded inputs and nothing else.

What the oracle computes is written out at the top of hstu_oracle.c, with the page and
section each step follows ("HSTU tensor by tensor: SiLU aggregation, temporal bias and
gating", "HSTU-MUSA: HSTU for Moore Threads (MUSA)").
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_lib = None

_P_I64 = ctypes.POINTER(ctypes.c_int64)
_P_I32 = ctypes.POINTER(ctypes.c_int32)
_P_F64 = ctypes.POINTER(ctypes.c_double)
_P_U8 = ctypes.POINTER(ctypes.c_uint8)
_I64 = ctypes.c_int64
_F64 = ctypes.c_double


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.hstu_oracle_time_bucket.restype = _I64
        L.hstu_oracle_time_bucket.argtypes = [_I64, _F64, _I64]
        L.hstu_oracle_mask.restype = _I64
        L.hstu_oracle_mask.argtypes = [_I64, _I64, _I64, _I64, _P_U8]
        L.hstu_oracle_mask_flags.restype = _I64
        L.hstu_oracle_mask_flags.argtypes = [_I64] * 5 + [_P_U8]
        common = [_I64, _I64, _I64, _I64, _P_I64, _P_I32, _P_I32, _P_I64, _P_F64, _P_F64,
                  _P_F64, _P_F64, _P_F64, _I64, _P_F64, _I64, _F64, _F64, _I64, _I64, _F64, _I64]
        L.hstu_oracle_mask_rows.restype = _I64
        L.hstu_oracle_mask_rows.argtypes = [_I64] * 8 + [_P_U8]
        L.hstu_oracle_fwd.restype = ctypes.c_int
        L.hstu_oracle_fwd.argtypes = common + [_P_F64] * 4
        L.hstu_oracle_bwd.restype = ctypes.c_int
        L.hstu_oracle_bwd.argtypes = common + [_P_F64] * 7
        L.hstu_oracle_num_threads.restype = ctypes.c_int
        L.hstu_oracle_num_threads.argtypes = []
        _lib = L
    return _lib


def _ptr(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def time_bucket(dt: int, div: float = 0.301, nb: int = 128) -> int:
    return int(lib().hstu_oracle_time_bucket(int(dt), float(div), int(nb)))


# mask variants (flags): contextual rows see the whole history; rel index |p(i) - p(j)|
CTX_SEES_HISTORY, REL_ABS = 1, 2


def mask(L: int, c: int = 0, t: int = 0, W: int = 0, flags: int = 0):
    """(L x L uint8 mask, valid-pair count) of one sequence; row = query position."""
    m = np.zeros((max(L, 1), max(L, 1)), dtype=np.uint8)[:L, :L].copy()
    if flags:
        n = lib().hstu_oracle_mask_flags(L, c, t, W, flags, _ptr(m, ctypes.c_uint8))
    else:
        n = lib().hstu_oracle_mask(L, c, t, W, _ptr(m, ctypes.c_uint8))
    return m, int(n)


def mask_rows(L: int, c: int, t: int, W: int, r0: int, nrows: int, ncols: int, flags: int = 0):
    """Rows [r0, r0+nrows) x keys [0, ncols) of the mask of one sequence (positions >= L
    invalid), as a uint8 matrix."""
    m = np.zeros((nrows, ncols), dtype=np.uint8)
    lib().hstu_oracle_mask_rows(L, c, t, W, flags, r0, nrows, ncols, _ptr(m, ctypes.c_uint8))
    return m


def num_threads() -> int:
    return int(lib().hstu_oracle_num_threads())


def _common_args(b, keep):
    offs = np.ascontiguousarray(b.seq_offsets, dtype=np.int64)
    ctx = None if b.num_contextuals is None else np.ascontiguousarray(b.num_contextuals, np.int32)
    tgt = None if b.num_targets is None else np.ascontiguousarray(b.num_targets, np.int32)
    ts = None if b.timestamps is None else np.ascontiguousarray(b.timestamps, np.int64)
    q, k, v, u = _f64(b.q), _f64(b.k), _f64(b.v), _f64(b.u)
    rel, tb = _f64(b.rel_bias), _f64(b.time_bias)
    keep.extend([offs, ctx, tgt, ts, q, k, v, u, rel, tb])
    return [b.batch, b.num_heads, b.d_qk, b.d_v, _ptr(offs, ctypes.c_int64),
            _ptr(ctx, ctypes.c_int32), _ptr(tgt, ctypes.c_int32), _ptr(ts, ctypes.c_int64),
            _ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double), _ptr(v, ctypes.c_double),
            _ptr(u, ctypes.c_double), _ptr(rel, ctypes.c_double), b.rel_bias_len,
            _ptr(tb, ctypes.c_double), b.time_bias_len, float(b.time_bucket_div),
            float(b.alpha), int(b.max_attn_len), int(b.max_seqlen), float(b.ln_eps),
            int(getattr(b, "mask_flags", 0))]


def fwd(b):
    """fp64 forward: dict(out [T,D], y [T,D], mean [T], rstd [T])."""
    keep = []
    T, D = b.total_tokens, b.num_heads * b.d_v
    out = np.zeros((T, D)); y = np.zeros((T, D)); mean = np.zeros(T); rstd = np.zeros(T)
    rc = lib().hstu_oracle_fwd(*_common_args(b, keep), _ptr(out, ctypes.c_double),
                               _ptr(y, ctypes.c_double), _ptr(mean, ctypes.c_double),
                               _ptr(rstd, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle rejected the batch (bad offsets / contextual / target counts)")
    return dict(out=out, y=y, mean=mean, rstd=rstd)


def bwd(b, dout=None):
    """fp64 backward of sum(dout * O): dict(dq, dk, dv, du, drel, dtb)."""
    keep = []
    if dout is None:
        dout = b.dout
    T, H = b.total_tokens, b.num_heads
    dout = _f64(dout)
    dq = np.zeros((T, H, b.d_qk)); dk = np.zeros((T, H, b.d_qk)); dv = np.zeros((T, H, b.d_v))
    du = np.zeros((T, H * b.d_v))
    drel = np.zeros(max(b.rel_bias_len, 1)); dtb = np.zeros(max(b.time_bias_len, 1))
    rc = lib().hstu_oracle_bwd(*_common_args(b, keep), _ptr(dout, ctypes.c_double),
                               _ptr(dq, ctypes.c_double), _ptr(dk, ctypes.c_double),
                               _ptr(dv, ctypes.c_double), _ptr(du, ctypes.c_double),
                               _ptr(drel, ctypes.c_double), _ptr(dtb, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle rejected the batch")
    return dict(dq=dq, dk=dk, dv=dv, du=du, drel=drel[:b.rel_bias_len],
                dtb=dtb[:b.time_bias_len])
