"""The forward entry point for callers that cannot allocate device memory.

hstu_attn_fwd_noalloc takes its scratch from a fixed array inside the library instead of a
caller workspace, for callers such as framework plugins that own no allocator or serving
loops that must not call cudaMalloc.  Through the C ABI, two calls in a row must match the
regular hstu_attn_fwd within the bf16 tolerance, and a request larger than the fixed
scratch must be refused before anything runs.  Both calls run the same kernels, so the
comparison is bitwise: a difference would mean that state left in the shared scratch by an
earlier call leaked into a later one.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from jagged_hstu_attention_02_b200 import ops, synth
from tests.helpers import assert_close

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    lib = ops.lib()
    fn = lib.hstu_attn_fwd_noalloc
    fn.argtypes = [ctypes.POINTER(ops.Params)] + [ctypes.c_void_p] * 12
    fn.restype = ctypes.c_int
    return fn


def _call_noalloc(fn, params, t, out):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(ctypes.byref(params), ops._ptr(t["q"]), ops._ptr(t["k"]), ops._ptr(t["v"]),
              ops._ptr(t["u"]), ops._ptr(t["seq_offsets"]), ops._ptr(t["num_contextuals"]),
              ops._ptr(t["num_targets"]), ops._ptr(t["timestamps"]), ops._ptr(t["rel_bias"]),
              ops._ptr(t["time_bias"]), ops._ptr(out), stream)


def test_noalloc_forward_matches_regular_forward_twice():
    b = synth.make_batch(np.random.default_rng(2024), [5, 200, 77, 260, 129], 4, 128, 128,
                         "bf16", contextuals=[1, 4, 0, 8, 3], targets=[2, 20, 5, 0, 64],
                         rel_bias_len=261, time_bias_len=128)
    t = ops.batch_to_device(b)
    ref = ops.run_fwd(b, t).float().cpu().numpy()
    params = ops.make_params(t["q"], t["v"], t["seq_offsets"], alpha=b.alpha,
                             max_seqlen=b.max_seqlen, max_attn_len=b.max_attn_len,
                             rel_bias=t["rel_bias"], time_bias=t["time_bias"],
                             time_bucket_div=b.time_bucket_div, ln_eps=b.ln_eps)
    fn = _noalloc_fn()
    ref_t = ops.run_fwd(b, t)
    for _ in range(2):
        out = torch.full_like(t["u"], float("nan"))
        assert _call_noalloc(fn, params, t, out) == 0
        torch.cuda.synchronize()
        assert torch.equal(out, ref_t), "no-alloc forward differs from hstu_attn_fwd"
        assert_close(out.float().cpu().numpy(), ref, "bf16", "no-alloc forward vs hstu_attn_fwd")


def _params_of(b, t):
    return ops.make_params(t["q"], t["v"], t["seq_offsets"], alpha=b.alpha,
                           max_seqlen=b.max_seqlen, max_attn_len=b.max_attn_len,
                           rel_bias=t["rel_bias"], time_bias=t["time_bias"],
                           time_bucket_div=b.time_bucket_div, ln_eps=b.ln_eps)


def test_noalloc_large_batch_then_small_batch():
    """A large call fills the shared scratch; a smaller call afterwards must not see any of
    it, also when its offsets end short of its token count (rows no sequence covers)."""
    fn = _noalloc_fn()
    big = synth.make_batch(np.random.default_rng(31), [900, 1500, 2000], 4, 128, 128, "bf16",
                           contextuals=2, targets=[10, 30, 5], rel_bias_len=2001,
                           time_bias_len=128)
    tb = ops.batch_to_device(big)
    out_big = torch.empty_like(tb["u"])
    assert _call_noalloc(fn, _params_of(big, tb), tb, out_big) == 0
    small = synth.make_batch(np.random.default_rng(32), [40, 130, 77], 4, 128, 128, "bf16",
                             contextuals=1, targets=[3, 9, 1], rel_bias_len=131,
                             time_bias_len=128)
    ts = ops.batch_to_device(small)
    out = torch.empty_like(ts["u"])
    assert _call_noalloc(fn, _params_of(small, ts), ts, out) == 0
    torch.cuda.synchronize()
    assert torch.equal(out, ops.run_fwd(small, ts))
    # offsets that end 20 rows short of T: the uncovered rows come out as zeros, flagged
    short = dict(ts)
    offs = small.seq_offsets.copy()
    offs[-1] -= 20
    short["seq_offsets"] = torch.from_numpy(offs).cuda()
    out = torch.full_like(ts["u"], float("nan"))
    assert _call_noalloc(fn, _params_of(small, ts), short, out) == 0
    torch.cuda.synchronize()
    last = int(offs[-2])
    assert torch.equal(out[:last], ops.run_fwd(small, ts)[:last])
    assert bool((out[last:] == 0).all()), "rows of the skipped sequence are not zero"


def test_noalloc_forward_refuses_requests_above_its_scratch():
    fn = _noalloc_fn()
    b = synth.make_batch(np.random.default_rng(1), [4], 4, 128, 128, "bf16", rel_bias_len=5)
    t = ops.batch_to_device(b)
    params = ops.make_params(t["q"], t["v"], t["seq_offsets"], alpha=b.alpha,
                             max_seqlen=b.max_seqlen, rel_bias=t["rel_bias"])
    params.total_tokens = 20000            # 256 + 4 * 20000 * 512 bytes > 32 MiB
    out = torch.empty_like(t["u"])
    assert _call_noalloc(fn, params, t, out) == 3   # HSTU_ERR_WORKSPACE_TOO_SMALL
