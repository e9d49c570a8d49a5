"""Thin ctypes binding of libhstu_attn.so (C ABI in include/hstu_attn.h).

Argument marshalling only: tensors become raw device pointers plus the current CUDA
stream; every step of the computation runs in the library's kernels.  There is no CPU
path: without the built library, or with tensors not on a CUDA device, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhstu_attn.so")

HSTU_F32, HSTU_BF16 = 0, 1
STATUS_NAMES = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "workspace too small",
                4: "CUDA error", 5: "invalid device data"}
DEV_BAD_OFFSETS, DEV_BAD_COUNTS, DEV_SEQ_TOO_LONG, DEV_WAIT_TIMEOUT = 0x1, 0x2, 0x4, 0x8

EXPORTED = ["hstu_attn_fwd_workspace_size", "hstu_attn_fwd", "hstu_attn_bwd_workspace_size",
            "hstu_attn_bwd", "hstu_attn_read_device_status", "hstu_attn_debug_mask",
            "hstu_attn_debug_kernel_mask", "hstu_attn_set_wait_test",
            "hstu_stochastic_length", "hstu_gather_rows", "hstu_jagged_concat",
            "hstu_layer_norm_rows", "hstu_uvqk_proj", "hstu_out_proj",
            "hstu_attn_time_thresholds", "hstu_attn_set_stage_events", "hstu_status_string",
            "hstu_attn_version"]
STAGES = {"fwd_attn": 0, "fwd_norm": 1, "bwd_norm": 2, "bwd_attn": 3}


class HstuError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__("%s failed: %s (status %d)" % (what, STATUS_NAMES.get(status, "?"), status))
        self.status = status


class Params(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("max_seqlen", ctypes.c_int32), ("max_attn_len", ctypes.c_int32),
                ("total_tokens", ctypes.c_int64), ("alpha", ctypes.c_float),
                ("ln_eps", ctypes.c_float), ("rel_bias_len", ctypes.c_int32),
                ("time_bias_len", ctypes.c_int32), ("time_bucket_div", ctypes.c_double),
                ("dtype", ctypes.c_int32), ("flags", ctypes.c_int32)]

# mask variants (Params.flags)
FLAG_CTX_SEES_HISTORY, FLAG_REL_ABS, FLAG_CANDIDATES_ONLY = 0x1, 0x2, 0x4


_lib = None
_VP = ctypes.c_void_p


def lib():
    """Load libhstu_attn.so (build it with `python -m jagged_hstu_attention_02_b200.build`)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libhstu_attn.so is not built (%s); run "
                               "`python -m jagged_hstu_attention_02_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(Params)
        sz = ctypes.POINTER(ctypes.c_size_t)
        L.hstu_attn_fwd_workspace_size.argtypes = [P, sz]
        L.hstu_attn_bwd_workspace_size.argtypes = [P, sz]
        L.hstu_attn_fwd.argtypes = [P] + [_VP] * 15 + [ctypes.c_size_t, _VP]
        L.hstu_attn_bwd.argtypes = [P] + [_VP] * 21 + [ctypes.c_size_t, _VP]
        L.hstu_attn_read_device_status.argtypes = [_VP, _VP, ctypes.POINTER(ctypes.c_int32)]
        L.hstu_attn_debug_mask.argtypes = [P, _VP, _VP, _VP, ctypes.c_int32, ctypes.c_int32, _VP,
                                           _VP]
        L.hstu_attn_debug_kernel_mask.argtypes = [P, _VP, _VP, _VP] + [ctypes.c_int32] * 5 + [
            _VP, _VP]
        L.hstu_attn_time_thresholds.argtypes = [ctypes.c_double, ctypes.c_int32,
                                                ctypes.POINTER(ctypes.c_uint64)]
        L.hstu_attn_set_stage_events.argtypes = [ctypes.c_int32, _VP, _VP]
        L.hstu_attn_set_wait_test.argtypes = [ctypes.c_int64, ctypes.c_int32]
        L.hstu_stochastic_length.argtypes = [_VP, _VP, _VP, ctypes.c_int32, ctypes.c_int64, _VP,
                                             ctypes.c_int32, _VP, _VP, _VP, _VP]
        L.hstu_layer_norm_rows.argtypes = [_VP, _VP, ctypes.c_int64, ctypes.c_int32,
                                           ctypes.c_float, _VP]
        L.hstu_uvqk_proj.argtypes = [_VP, _VP, _VP, ctypes.c_int64] + [ctypes.c_int32] * 5 + \
            [_VP] * 6
        L.hstu_out_proj.argtypes = [_VP, _VP, _VP, _VP, ctypes.c_int64, ctypes.c_int32,
                                    ctypes.c_int32, _VP, _VP, _VP]
        L.hstu_gather_rows.argtypes = [_VP, ctypes.c_int64, _VP, _VP, ctypes.c_int64, _VP, _VP]
        L.hstu_jagged_concat.argtypes = [ctypes.c_int32, ctypes.POINTER(_VP),
                                         ctypes.POINTER(_VP), ctypes.c_int32, ctypes.c_int64,
                                         _VP, _VP, _VP]
        L.hstu_status_string.restype = ctypes.c_char_p
        L.hstu_status_string.argtypes = [ctypes.c_int]
        L.hstu_attn_version.restype = ctypes.c_int32
        for name in EXPORTED:
            f = getattr(L, name)
            if name not in ("hstu_status_string", "hstu_attn_version"):
                f.restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int, what: str):
    if status != 0:
        raise HstuError(status, what)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return HSTU_F32
    if t.dtype == torch.bfloat16:
        return HSTU_BF16
    raise ValueError("unsupported dtype %s" % t.dtype)


def make_params(q, v, seq_offsets, *, alpha, max_seqlen, max_attn_len=0, rel_bias=None,
                time_bias=None, time_bucket_div=0.301, ln_eps=1e-5, mask_flags=0) -> Params:
    T, H, dqk = q.shape
    return Params(batch=seq_offsets.numel() - 1, num_heads=H, d_qk=dqk, d_v=v.shape[2],
                  max_seqlen=int(max_seqlen), max_attn_len=int(max_attn_len), total_tokens=T,
                  alpha=float(alpha), ln_eps=float(ln_eps),
                  rel_bias_len=0 if rel_bias is None else rel_bias.numel(),
                  time_bias_len=0 if time_bias is None else time_bias.numel(),
                  time_bucket_div=float(time_bucket_div), dtype=dtype_code(q),
                  flags=int(mask_flags))


def fwd_workspace_size(params: Params) -> int:
    n = ctypes.c_size_t()
    _check(lib().hstu_attn_fwd_workspace_size(ctypes.byref(params), ctypes.byref(n)),
           "hstu_attn_fwd_workspace_size")
    return n.value


def bwd_workspace_size(params: Params) -> int:
    n = ctypes.c_size_t()
    _check(lib().hstu_attn_bwd_workspace_size(ctypes.byref(params), ctypes.byref(n)),
           "hstu_attn_bwd_workspace_size")
    return n.value


@dataclass
class Saved:
    y: torch.Tensor
    mean: torch.Tensor
    rstd: torch.Tensor


def fwd(q, k, v, u, seq_offsets, num_contextuals=None, num_targets=None, timestamps=None,
        rel_bias=None, time_bias=None, *, alpha, max_seqlen, max_attn_len=0,
        time_bucket_div=0.301, ln_eps=1e-5, mask_flags=0, training=False, out=None,
        workspace=None, saved: Optional[Saved] = None, stream=None):
    """out [T, H*d_v] (and Saved(y, mean, rstd) when training)."""
    p = make_params(q, v, seq_offsets, alpha=alpha, max_seqlen=max_seqlen,
                    max_attn_len=max_attn_len, rel_bias=rel_bias, time_bias=time_bias,
                    time_bucket_div=time_bucket_div, ln_eps=ln_eps, mask_flags=mask_flags)
    T, H, dv = v.shape
    dev = q.device
    if out is None:
        out = torch.empty((T, H * dv), dtype=q.dtype, device=dev)
    if training and saved is None:
        saved = Saved(torch.empty((T, H * dv), dtype=torch.float32, device=dev),
                      torch.empty(T, dtype=torch.float32, device=dev),
                      torch.empty(T, dtype=torch.float32, device=dev))
    if workspace is None:
        workspace = torch.empty(fwd_workspace_size(p), dtype=torch.uint8, device=dev)
    st = lib().hstu_attn_fwd(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(seq_offsets),
        _ptr(num_contextuals), _ptr(num_targets), _ptr(timestamps), _ptr(rel_bias),
        _ptr(time_bias), _ptr(out), _ptr(saved.y if training else None),
        _ptr(saved.mean if training else None), _ptr(saved.rstd if training else None),
        _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "hstu_attn_fwd")
    fwd.last_workspace = workspace
    return (out, saved) if training else out


def bwd(dout, q, k, v, u, seq_offsets, num_contextuals=None, num_targets=None, timestamps=None,
        rel_bias=None, time_bias=None, *, saved: Saved, alpha, max_seqlen, max_attn_len=0,
        time_bucket_div=0.301, ln_eps=1e-5, mask_flags=0, grads=None, workspace=None,
        stream=None):
    """(dq, dk, dv, du, d_rel_bias or None, d_time_bias or None)."""
    p = make_params(q, v, seq_offsets, alpha=alpha, max_seqlen=max_seqlen,
                    max_attn_len=max_attn_len, rel_bias=rel_bias, time_bias=time_bias,
                    time_bucket_div=time_bucket_div, ln_eps=ln_eps, mask_flags=mask_flags)
    dev = q.device
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                 torch.empty_like(u),
                 None if rel_bias is None else torch.empty_like(rel_bias),
                 None if time_bias is None else torch.empty_like(time_bias))
    dq, dk, dv, du, drel, dtb = grads
    if workspace is None:
        workspace = torch.empty(bwd_workspace_size(p), dtype=torch.uint8, device=dev)
    st = lib().hstu_attn_bwd(
        ctypes.byref(p), _ptr(dout), _ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(seq_offsets),
        _ptr(num_contextuals), _ptr(num_targets), _ptr(timestamps), _ptr(rel_bias),
        _ptr(time_bias), _ptr(saved.y), _ptr(saved.mean), _ptr(saved.rstd), _ptr(dq), _ptr(dk),
        _ptr(dv), _ptr(du), _ptr(drel), _ptr(dtb), _ptr(workspace), workspace.numel(),
        _stream(stream))
    _check(st, "hstu_attn_bwd")
    bwd.last_workspace = workspace
    return grads


def read_device_status(workspace: torch.Tensor, stream=None) -> int:
    code = ctypes.c_int32(0)
    st = lib().hstu_attn_read_device_status(_ptr(workspace), _stream(stream), ctypes.byref(code))
    if st not in (0, 5):
        _check(st, "hstu_attn_read_device_status")
    return code.value


def debug_mask(params: Params, seq_offsets, num_contextuals, num_targets, seq: int, seq_len: int,
               stream=None) -> torch.Tensor:
    """[seq_len, seq_len] bool mask of sequence `seq` as the device predicate evaluates it."""
    words = (seq_len * seq_len + 31) // 32
    bits = torch.zeros(max(words, 1), dtype=torch.int32, device=seq_offsets.device)
    _check(lib().hstu_attn_debug_mask(ctypes.byref(params), _ptr(seq_offsets),
                                      _ptr(num_contextuals), _ptr(num_targets), seq, seq_len,
                                      _ptr(bits), _stream(stream)), "hstu_attn_debug_mask")
    b = bits.cpu().numpy().view("uint32")
    import numpy as np
    flat = ((b[:, None] >> np.arange(32, dtype=np.uint32)[None, :]) & 1).astype(bool).reshape(-1)
    return torch.from_numpy(flat[:seq_len * seq_len].reshape(seq_len, seq_len).copy())


def debug_kernel_mask(params: Params, seq_offsets, num_contextuals, num_targets, seq: int,
                      kernel: str, row_begin: int, row_count: int, key_count: int,
                      stream=None):
    """[row_count, key_count] bool mask of sequence `seq` as the tensor-core forward
    (kernel "fwd") or backward ("bwd") decides it, rows from row_begin."""
    import numpy as np
    words = row_count * key_count // 32
    bits = torch.zeros(max(words, 1), dtype=torch.int32, device=seq_offsets.device)
    _check(lib().hstu_attn_debug_kernel_mask(
        ctypes.byref(params), _ptr(seq_offsets), _ptr(num_contextuals), _ptr(num_targets), seq,
        {"fwd": 0, "bwd": 1}[kernel], row_begin, row_count, key_count, _ptr(bits),
        _stream(stream)), "hstu_attn_debug_kernel_mask")
    b = bits.cpu().numpy().view("uint32")[:words]
    flat = ((b[:, None] >> np.arange(32, dtype=np.uint32)[None, :]) & 1).astype(bool).reshape(-1)
    return torch.from_numpy(flat.reshape(row_count, key_count).copy())


def time_thresholds(div: float, nb: int):
    """Host-side threshold table the device compares |dt| against (uint64, nb-1 entries)."""
    arr = (ctypes.c_uint64 * max(nb - 1, 1))()
    _check(lib().hstu_attn_time_thresholds(float(div), int(nb), arr), "hstu_attn_time_thresholds")
    return [int(arr[i]) for i in range(nb - 1)]


def set_stage_events(stage: str, start=None, stop=None):
    """Record torch.cuda.Event `start`/`stop` around the kernels of `stage` in every later
    fwd/bwd call (None clears).  The events must stay alive while set."""
    sp = None if start is None else ctypes.c_void_p(start.cuda_event)
    ep = None if stop is None else ctypes.c_void_p(stop.cuda_event)
    _check(lib().hstu_attn_set_stage_events(STAGES[stage], sp, ep), "hstu_attn_set_stage_events")


def set_wait_test(limit_cycles: int = 0, stall: bool = False):
    """Test hook: shorten the kernels' pipeline waits and make one of them run out."""
    _check(lib().hstu_attn_set_wait_test(int(limit_cycles), 1 if stall else 0),
           "hstu_attn_set_wait_test")


# ------------------------------------------------------------------ jagged operations

MAX_CONCAT_PARTS = 16

def stochastic_length(seq_offsets, num_contextuals, num_targets, keys, budget: int,
                      status=None, stream=None):
    """(kept rows [T] int64 (first new_offsets[-1] valid), new offsets [B+1] int64)."""
    T = int(keys.numel())
    B = seq_offsets.numel() - 1
    rows = torch.empty(max(T, 1), dtype=torch.int64, device=seq_offsets.device)
    offs = torch.empty(B + 1, dtype=torch.int64, device=seq_offsets.device)
    _check(lib().hstu_stochastic_length(_ptr(seq_offsets), _ptr(num_contextuals),
                                        _ptr(num_targets), B, T, _ptr(keys), int(budget),
                                        _ptr(rows), _ptr(offs), _ptr(status), _stream(stream)),
           "hstu_stochastic_length")
    return rows, offs


def gather_rows(src, rows, n_rows, max_rows: int, out=None, stream=None):
    """out[r] = src[rows[r]] for r < n_rows (a device scalar tensor), up to max_rows rows."""
    if out is None:
        out = torch.empty((max_rows,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    row_bytes = src[0].numel() * src.element_size() if src.numel() else 1
    _check(lib().hstu_gather_rows(_ptr(src), row_bytes, _ptr(rows), _ptr(n_rows), int(max_rows),
                                  _ptr(out), _stream(stream)), "hstu_gather_rows")
    return out


def jagged_concat(parts, out=None, stream=None):
    """parts: list of (values [T_q, ...], offsets [B+1]); (values, offsets) of the per-sequence
    concatenation."""
    vals0, offs0 = parts[0]
    B = offs0.numel() - 1
    total = sum(int(v.shape[0]) for v, _ in parts)
    if out is None:
        out = torch.empty((total,) + tuple(vals0.shape[1:]), dtype=vals0.dtype,
                          device=vals0.device)
    out_offs = torch.empty(B + 1, dtype=torch.int64, device=offs0.device)
    n = len(parts)
    V = (_VP * n)(*[_ptr(v) for v, _ in parts])
    O = (_VP * n)(*[_ptr(o) for _, o in parts])
    row_bytes = vals0[0].numel() * vals0.element_size() if vals0.numel() else \
        int(np.prod(vals0.shape[1:])) * vals0.element_size()
    _check(lib().hstu_jagged_concat(n, V, O, B, row_bytes, _ptr(out), _ptr(out_offs),
                                    _stream(stream)), "hstu_jagged_concat")
    return out, out_offs


# ------------------------------------------------------------------ the layer around the path

def layer_norm_rows(x, eps=1e-5, out=None, stream=None):
    """LayerNorm (no affine) of every row of the bf16 matrix x."""
    if out is None:
        out = torch.empty_like(x)
    _check(lib().hstu_layer_norm_rows(_ptr(x), _ptr(out), x.shape[0], x.shape[1], float(eps),
                                      _stream(stream)), "hstu_layer_norm_rows")
    return out


def uvqk_proj(x, w, bias, num_heads, d_qk, d_v, silu=False, status=None, stream=None):
    """(u [T, H*d_v], v [T,H,d_v], q [T,H,d_qk], k [T,H,d_qk]) of the fused projection."""
    T = x.shape[0]
    dev, dt = x.device, x.dtype
    u = torch.empty((T, num_heads * d_v), dtype=dt, device=dev)
    v = torch.empty((T, num_heads, d_v), dtype=dt, device=dev)
    q = torch.empty((T, num_heads, d_qk), dtype=dt, device=dev)
    k = torch.empty((T, num_heads, d_qk), dtype=dt, device=dev)
    _check(lib().hstu_uvqk_proj(_ptr(x), _ptr(w), _ptr(bias), T, x.shape[1], num_heads, d_qk,
                                d_v, 1 if silu else 0, _ptr(u), _ptr(v), _ptr(q), _ptr(k),
                                _ptr(status), _stream(stream)), "hstu_uvqk_proj")
    return u, v, q, k


def out_proj(z, w_o, bias=None, x=None, status=None, stream=None):
    """z [T, d_in] w_o [d_in, d_model] (+ bias) (+ x): the output projection and residual."""
    T, d_model = z.shape[0], w_o.shape[1]
    out = torch.empty((T, d_model), dtype=z.dtype, device=z.device)
    _check(lib().hstu_out_proj(_ptr(z), _ptr(w_o), _ptr(bias), _ptr(x), T, z.shape[1], d_model,
                               _ptr(out), _ptr(status), _stream(stream)), "hstu_out_proj")
    return out


def layer_fwd(x, seq_offsets, num_contextuals, num_targets, timestamps, rel_bias, time_bias,
              w_uvqk, b_uvqk, w_o, b_o, *, num_heads, d_qk, d_v, alpha, max_seqlen,
              max_attn_len=0, time_bucket_div=0.301, ln_eps=1e-5, mask_flags=0,
              uvqk_silu=False, stream=None):
    """One HSTU layer on jagged tokens x [T, d_model] (bf16): input LayerNorm, fused U/V/Q/K
    projection, attention with LayerNorm and U gating, output projection with bias and the
    residual.  Returns dict(xn, u, v, q, k, attn, o)."""
    xn = layer_norm_rows(x, ln_eps, stream=stream)
    u, v, q, k = uvqk_proj(xn, w_uvqk, b_uvqk, num_heads, d_qk, d_v, silu=uvqk_silu,
                           stream=stream)
    attn = fwd(q, k, v, u, seq_offsets, num_contextuals, num_targets, timestamps, rel_bias,
               time_bias, alpha=alpha, max_seqlen=max_seqlen, max_attn_len=max_attn_len,
               time_bucket_div=time_bucket_div, ln_eps=ln_eps, mask_flags=mask_flags,
               stream=stream)
    o = out_proj(attn, w_o, b_o, x, stream=stream)
    return dict(xn=xn, u=u, v=v, q=q, k=k, attn=attn, o=o)


def version() -> int:
    return int(lib().hstu_attn_version())


# ------------------------------------------------------------------ batch helpers

def batch_to_device(b, device="cuda"):
    """Device tensors of a synth.Batch (values already exact in the batch dtype)."""
    dt = torch.float32 if b.dtype == "f32" else torch.bfloat16

    def T(a, dtype=None):
        if a is None:
            return None
        t = torch.from_numpy(a)
        if dtype is not None:
            t = t.to(dtype)
        return t.to(device).contiguous()

    return dict(q=T(b.q, dt), k=T(b.k, dt), v=T(b.v, dt), u=T(b.u, dt),
                seq_offsets=T(b.seq_offsets), num_contextuals=T(b.num_contextuals),
                num_targets=T(b.num_targets), timestamps=T(b.timestamps),
                rel_bias=T(b.rel_bias), time_bias=T(b.time_bias),
                dout=T(b.dout, dt) if b.dout is not None else None)


def batch_kwargs(b):
    return dict(alpha=b.alpha, max_seqlen=b.max_seqlen, max_attn_len=b.max_attn_len,
                time_bucket_div=b.time_bucket_div, ln_eps=b.ln_eps,
                mask_flags=int(getattr(b, "mask_flags", 0)))


def run_fwd(b, dev_tensors=None, training=False, **kw):
    t = batch_to_device(b) if dev_tensors is None else dev_tensors
    args = batch_kwargs(b)
    args.update(kw)
    return fwd(t["q"], t["k"], t["v"], t["u"], t["seq_offsets"], t["num_contextuals"],
               t["num_targets"], t["timestamps"], t["rel_bias"], t["time_bias"],
               training=training, **args)


def run_bwd(b, saved, dout=None, dev_tensors=None, **kw):
    t = batch_to_device(b) if dev_tensors is None else dev_tensors
    if dout is None:
        dout = t["dout"]
    args = batch_kwargs(b)
    args.update(kw)
    return bwd(dout, t["q"], t["k"], t["v"], t["u"], t["seq_offsets"], t["num_contextuals"],
               t["num_targets"], t["timestamps"], t["rel_bias"], t["time_bias"], saved=saved,
               **args)
