"""Host-side checks of the CUDA library that need no GPU: it loads, exports every symbol
declared in include/*.h, validates arguments, and its fp64 time-bucket threshold table
agrees with the oracle's fp64 bucket decision at every boundary."""
import ctypes
import glob
import os
import re

import pytest

from jagged_hstu_attention_02_b200 import ops
from oracle import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(hstu_\w+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    lib = ops.lib()
    names = _declared_symbols()
    assert len(names) >= 9
    for name in names:
        assert hasattr(lib, name), name
    assert set(ops.EXPORTED) <= set(names)


def test_status_strings_and_version():
    lib = ops.lib()
    for code in range(6):
        assert lib.hstu_status_string(code)
    assert ops.version() == 100


def _params(**kw):
    base = dict(batch=2, num_heads=2, d_qk=32, d_v=32, max_seqlen=16, max_attn_len=0,
                total_tokens=20, alpha=0.5, ln_eps=1e-5, rel_bias_len=17, time_bias_len=128,
                time_bucket_div=0.301, dtype=ops.HSTU_BF16, flags=0)
    base.update(kw)
    return ops.Params(**base)


def test_workspace_size_and_validation():
    p = _params()
    n = ops.fwd_workspace_size(p)
    assert n >= 256 + 20 * 64 * 4
    assert ops.bwd_workspace_size(p) >= 256 + 20 * 64 * 4 + 20 * 64 * 4
    for bad in [dict(num_heads=0), dict(d_qk=0), dict(d_v=300), dict(max_seqlen=0),
                dict(time_bias_len=-1), dict(dtype=7), dict(flags=8),
                dict(time_bucket_div=0.0), dict(batch=-1)]:
        with pytest.raises(ops.HstuError) as e:
            ops.fwd_workspace_size(_params(**bad))
        assert e.value.status in (1, 2)


def test_fwd_rejects_bad_pointers_before_launch():
    """Host-checkable problems return a status and enqueue nothing (no GPU touched)."""
    lib = ops.lib()
    p = _params()
    args = [ctypes.byref(p)] + [None] * 15 + [0, None]
    assert lib.hstu_attn_fwd(*args) == 1            # NULL pointers
    fake = ctypes.c_void_p(0x1000)
    mis = ctypes.c_void_p(0x1008)
    #       params          q     k     v     u     offs  ctx   tgt   ts    rel   tb    out
    args = [ctypes.byref(p), fake, fake, fake, fake, fake, None, None, fake, fake, fake, fake,
            None, None, None, fake, 10, None]   # saved_y, mean, rstd, workspace, bytes, stream
    assert lib.hstu_attn_fwd(*args) == 3            # workspace too small
    args[1] = mis
    assert lib.hstu_attn_fwd(*args) == 1            # misaligned q
    args[1] = fake
    args[12] = fake                                 # saved_y without mean / rstd
    assert lib.hstu_attn_fwd(*args) == 1


@pytest.mark.parametrize("div,nb", [(0.301, 128), (0.301, 256), (1.0, 16), (0.05, 256),
                                    (7.5, 8)])
def test_time_thresholds_match_oracle_fp64_decision(div, nb):
    thr = ops.time_thresholds(div, nb)
    assert len(thr) == nb - 1
    assert thr == sorted(thr)
    for kk, t in enumerate(thr, start=1):
        if t >= 2 ** 63:      # beyond the |dt| < 2^63 the interface admits
            continue
        # first |dt| of bucket >= kk: the oracle (fp64) agrees on both sides of the boundary
        assert oracle.time_bucket(t, div, nb) >= kk
        if t > 0:
            assert oracle.time_bucket(t - 1, div, nb) < kk


def test_test_hooks_validate_their_arguments():
    lib = ops.lib()
    assert lib.hstu_attn_set_wait_test(-1, 0) == 1
    assert lib.hstu_attn_set_wait_test(1000, 2) == 1
    assert lib.hstu_attn_set_wait_test(0, 0) == 0
    p = _params()
    fake = ctypes.c_void_p(16)   # never dereferenced: every call below fails validation first
    for args in [(0, 2, 0, 4, 128), (0, 0, -1, 4, 128), (0, 0, 0, -4, 128), (0, 0, 0, 4, 100),
                 (5, 0, 0, 4, 128), (-1, 1, 0, 4, 128)]:
        seq, kernel, r0, nrows, nkeys = args
        st = lib.hstu_attn_debug_kernel_mask(ctypes.byref(p), fake, None, None, seq, kernel, r0,
                                             nrows, nkeys, fake, None)
        assert st == 1, args
