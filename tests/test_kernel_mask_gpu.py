"""The masked-pair structure of the tensor-core kernels, bit for bit against the oracle.

hstu_attn_debug_kernel_mask exports the validity decisions the tcgen05 forward and backward
take (visited 128 x 128 tiles, then the 32-wide block masks), through the same device
functions the kernels call.  For every sequence of the sweep, and both kernels, the exported
bits over the sequence's own rows and keys must equal the oracle's mask ("HSTU-MUSA: HSTU
for Moore Threads (MUSA)", section "Mathematical Equivalence"), and no pair that reaches
past the sequence's end (the padding rows and keys of its last tile) may be marked for a
row the forward stores or a key the backward stores.
"""
import numpy as np
import pytest
import torch

from jagged_hstu_attention_02_b200 import ops
from oracle import oracle

pytestmark = pytest.mark.gpu

# (L, c, t): lengths around the 32- and 128-wide block edges, contextual prefixes and
# candidate groups that straddle them, E = 0 (all candidates), c + t = L, L = 1
SEQS = [(1, 0, 0), (1, 1, 0), (1, 0, 1), (5, 2, 3), (31, 0, 0), (32, 32, 0), (33, 0, 33),
        (64, 0, 64), (100, 40, 60), (128, 31, 33), (129, 32, 32), (130, 127, 1),
        (160, 33, 95), (257, 129, 127), (300, 33, 96), (383, 1, 20), (400, 3, 5),
        (513, 0, 0), (700, 8, 128), (1000, 100, 200)]
WINDOWS = [0, 1, 5, 31, 32, 33, 127, 128, 129, 1024]


def _params(lengths, W):
    return ops.Params(batch=len(lengths), num_heads=1, d_qk=64, d_v=64, max_seqlen=max(lengths),
                      max_attn_len=W, total_tokens=int(sum(lengths)), alpha=1.0, ln_eps=1e-5,
                      rel_bias_len=0, time_bias_len=0, time_bucket_div=0.301,
                      dtype=ops.HSTU_BF16, flags=0)


def _device_batch(seqs):
    lengths = [s[0] for s in seqs]
    offs = np.zeros(len(seqs) + 1, np.int64)
    offs[1:] = np.cumsum(lengths)
    ctx = np.array([s[1] for s in seqs], np.int32)
    tgt = np.array([s[2] for s in seqs], np.int32)
    return (lengths, torch.from_numpy(offs).cuda(), torch.from_numpy(ctx).cuda(),
            torch.from_numpy(tgt).cuda())


def _check_rows(p, d, seq, L, c, t, W, r0, nrows):
    pad = (L + 127) // 128 * 128
    ref = oracle.mask_rows(L, c, t, W, r0, nrows, pad).astype(bool)
    for kernel in ("fwd", "bwd"):
        got = ops.debug_kernel_mask(p, d[1], d[2], d[3], seq, kernel, r0, nrows, pad).numpy()
        rows_in = min(nrows, max(L - r0, 0))
        # the pairs of the sequence itself: bit-exact
        assert np.array_equal(got[:rows_in, :L], ref[:rows_in, :L]), (kernel, L, c, t, W, r0)
        if kernel == "fwd":
            # the forward stores rows < L: none of their keys past the end may be valid
            assert not got[:rows_in, L:].any(), ("fwd padding keys", L, c, t, W)
        else:
            # the backward stores keys < L: no query row past the end may reach them
            assert not got[rows_in:, :L].any(), ("bwd padding rows", L, c, t, W)


@pytest.mark.parametrize("W", WINDOWS)
def test_kernel_mask_bit_exact(W):
    d = _device_batch(SEQS)
    p = _params(d[0], W)
    for s, (L, c, t) in enumerate(SEQS):
        pad = (L + 127) // 128 * 128
        _check_rows(p, d, s, L, c, t, W, 0, pad)


def test_kernel_mask_past_255_tiles():
    """A sequence of 33,000 tokens (258 tiles; the kernels' tile-count cache saturates at
    255): rows at the start, across the 255-tile mark and at the end, windowed and not."""
    seqs = [(33000, 5, 40), (17, 2, 3)]
    d = _device_batch(seqs)
    for W in (0, 64, 1024):
        p = _params(d[0], W)
        for r0, n in ((0, 160), (255 * 128 - 64, 192), (33000 - 200, 328)):
            _check_rows(p, d, 0, 33000, 5, 40, W, r0, n)
        _check_rows(p, d, 1, 17, 2, 3, W, 0, 128)
