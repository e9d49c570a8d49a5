"""The HSTU layer around the attention on the GPU against its fp64 oracle: input LayerNorm,
the fused U/V/Q/K projection (tcgen05 GEMM, split epilogue), the output projection with bias
and residual, and the whole layer ("HSTU tensor by tensor: SiLU aggregation, temporal bias
and gating", "Similar shape, different aggregation" and "Trace four projections")."""
import numpy as np
import pytest
import torch

from jagged_hstu_attention_02_b200 import ops, synth
from oracle import layer
from tests.helpers import assert_close

pytestmark = pytest.mark.gpu


def _bf16(a):
    return synth.round_to_dtype(np.asarray(a, np.float32), "bf16")


def _t(a, dt=torch.bfloat16):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda().to(dt)


def _np(t):
    return t.float().cpu().numpy()


@pytest.mark.parametrize("T", [1, 127, 129, 1000, 10923])
@pytest.mark.parametrize("shape", [(128, 4, 128, 128, True, False), (256, 2, 64, 128, False, True),
                                   (128, 3, 64, 64, True, True)])
def test_uvqk_projection(T, shape):
    d_model, H, dqk, dv, with_bias, silu = shape
    rng = np.random.default_rng(T + H)
    N = 2 * H * (dv + dqk)
    x = _bf16(rng.standard_normal((T, d_model)))
    w = _bf16(rng.standard_normal((d_model, N)) / np.sqrt(d_model))
    b = (rng.standard_normal(N) * 0.1).astype(np.float32) if with_bias else None
    u, v, q, k = ops.uvqk_proj(_t(x), _t(w), None if b is None else _t(b, torch.float32),
                               H, dqk, dv, silu=silu)
    torch.cuda.synchronize()
    ru, rv, rq, rk = layer.uvqk(x, w, b, H, dqk, dv, silu)
    for got, ref, name in ((u, ru, "u"), (v, rv, "v"), (q, rq, "q"), (k, rk, "k")):
        assert tuple(got.shape) == ref.shape, name
        assert_close(_np(got), ref, "bf16", "uvqk %s T=%d" % (name, T))


@pytest.mark.parametrize("T", [5, 128, 3001])
@pytest.mark.parametrize("dims", [(512, 128), (128, 256)])
def test_output_projection_with_residual(T, dims):
    d_in, d_model = dims
    rng = np.random.default_rng(T)
    z = _bf16(rng.standard_normal((T, d_in)))
    w = _bf16(rng.standard_normal((d_in, d_model)) / np.sqrt(d_in))
    b = (rng.standard_normal(d_model) * 0.1).astype(np.float32)
    x = _bf16(rng.standard_normal((T, d_model)))
    for bias, res in ((b, x), (None, None), (b, None)):
        got = ops.out_proj(_t(z), _t(w), None if bias is None else _t(bias, torch.float32),
                           None if res is None else _t(res))
        torch.cuda.synchronize()
        assert_close(_np(got), layer.out_proj(z, w, bias, res), "bf16", "out_proj T=%d" % T)


def test_input_layer_norm():
    rng = np.random.default_rng(3)
    for width in (32, 128, 1024):
        x = _bf16(rng.standard_normal((777, width)) * 3 + 1)
        got = ops.layer_norm_rows(_t(x), 1e-5)
        torch.cuda.synchronize()
        assert_close(_np(got), layer.layer_norm(x, 1e-5), "bf16", "input norm %d" % width)


@pytest.mark.parametrize("silu", [False, True])
def test_whole_layer_movielens_shaped(silu):
    """MovieLens-shaped batch, d_model 128, 4 heads of 128: the layer's output (and its
    attention step) against the fp64 oracle."""
    b = synth.make_config(1)
    rng = np.random.default_rng(77)
    d_model, H, d = 128, b.num_heads, b.d_qk
    x = _bf16(rng.standard_normal((b.total_tokens, d_model)))
    w = _bf16(rng.standard_normal((d_model, 4 * H * d)) / np.sqrt(d_model))
    bw = (rng.standard_normal(4 * H * d) * 0.1).astype(np.float32)
    wo = _bf16(rng.standard_normal((H * d, d_model)) / np.sqrt(H * d))
    bo = (rng.standard_normal(d_model) * 0.1).astype(np.float32)
    dev = ops.batch_to_device(b)
    r = ops.layer_fwd(_t(x), dev["seq_offsets"], dev["num_contextuals"], dev["num_targets"],
                      dev["timestamps"], dev["rel_bias"], dev["time_bias"], _t(w),
                      _t(bw, torch.float32), _t(wo), _t(bo, torch.float32), num_heads=H,
                      d_qk=d, d_v=d, alpha=b.alpha, max_seqlen=b.max_seqlen,
                      ln_eps=b.ln_eps, uvqk_silu=silu)
    torch.cuda.synchronize()
    ref = layer.layer_fwd(b, x, w, bw, wo, bo, silu=silu)
    assert_close(_np(r["xn"]), ref["xn"], "bf16", "input norm")
    assert_close(_np(r["q"]), ref["q"], "bf16", "q")
    assert_close(_np(r["attn"]), ref["attn"], "bf16", "attention output")
    assert_close(_np(r["o"]), ref["o"], "bf16", "layer output")
