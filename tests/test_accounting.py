"""The algorithmic byte and FLOP counts behind the bench's roofline figures, restated from
their definitions for the MovieLens-shaped workload (H = 4, d_qk = d_v = 128, bf16, with
timestamps): the forward attention reads Q, K, V (3 x 1024 B per token) and writes Y in
fp32 (2048 B); the backward attention reads Q, K, V and dY in fp32 and writes dQ, dK, dV
(8192 B); each reads the int64 timestamps (8 B); the per-sequence offsets and counts and
the two bias tables are counted once per launch."""
from jagged_hstu_attention_02_b200 import accounting, synth


def _meta(b):
    return 8 * (b.batch + 1) + 8 * b.batch + 4 * (b.rel_bias_len + b.time_bias_len)


def test_per_token_bytes_of_the_attention_kernels():
    b = synth.make_config(4)
    T = b.total_tokens
    assert accounting.fwd_attn_bytes(b) == T * (3 * 1024 + 2048 + 8) + _meta(b)
    # the backward also writes the table gradients (one value per table entry)
    assert accounting.bwd_attn_bytes(b) == (T * (2 * 3 * 1024 + 2048 + 8) + _meta(b)
                                            + 4 * (b.rel_bias_len + b.time_bias_len))
    # LayerNorm + gating: Y (fp32) and U in, O out (+ mean and rstd when training)
    assert accounting.fwd_norm_bytes(b) == T * 512 * (4 + 2 + 2)
    assert accounting.fwd_norm_bytes(b, training=True) == T * 512 * 8 + 8 * T
    # its backward: dO, U, Y, mean, rstd in; dU and dY (fp32) out
    assert accounting.bwd_norm_bytes(b) == T * 512 * (2 + 2 + 4 + 2 + 4) + 8 * T


def test_flops_count_valid_pairs_only():
    b = synth.make_config(4)
    P = accounting.valid_pairs(b)
    assert accounting.fwd_flops(b, P) == P * 4 * 2 * (128 + 128)
    assert accounting.bwd_flops(b, P) == P * 4 * 2 * (2 * 128 + 2 * 128)
    assert accounting.bwd_flops_recompute(b, P) > accounting.bwd_flops(b, P)
