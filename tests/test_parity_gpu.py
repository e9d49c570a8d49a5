"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, element by element.

Tolerances: max|err| <= 1e-2*max|ref| + 1e-3 for bf16 inputs, <= 1e-5*max|ref| for fp32
inputs, per output tensor; the masked-pair structure bit-exact.
"""
import numpy as np
import pytest
import torch

from jagged_hstu_attention_02_b200 import ops, synth
from oracle import oracle
from tests.helpers import assert_close, rows_of, sub_batch

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().float().cpu().numpy()


def _fwd_check(b, training=True, what=""):
    dev = ops.batch_to_device(b)
    if training:
        out, saved = ops.run_fwd(b, dev, training=True)
    else:
        out = ops.run_fwd(b, dev)
    torch.cuda.synchronize()
    ref = oracle.fwd(b)
    assert_close(_np(out), ref["out"], b.dtype, what + " out")
    if training:
        assert_close(_np(saved.y), ref["y"], b.dtype, what + " y")
        assert_close(_np(saved.mean), ref["mean"], b.dtype, what + " mean")
        # rstd is large where Y is tiny; compare it relative to itself
        assert_close(_np(saved.rstd), ref["rstd"], b.dtype, what + " rstd")
    assert ops.read_device_status(ops.fwd.last_workspace) == 0
    return dev, out


SMALL_CASES = [
    # name, lengths, H, dqk, dv, dtype, ctx, tgt, W, R, NB
    ("f32-causal", [1, 37, 129, 300, 0, 513], 2, 32, 32, "f32", 0, 0, 0, 514, 0),
    ("f32-full-family", [5, 200, 77, 260], 2, 48, 80, "f32", [1, 4, 0, 8], [2, 20, 5, 0], 0,
     261, 128),
    ("f32-window", [300, 130, 2], 1, 32, 32, "f32", [3, 3, 1], [7, 0, 1], 17, 40, 64),
    ("bf16-causal", [1, 37, 129, 300, 0, 513], 2, 64, 64, "bf16", 0, 0, 0, 514, 128),
    ("bf16-family", [5, 200, 77, 260, 129], 4, 128, 128, "bf16", [1, 4, 0, 8, 3],
     [2, 20, 5, 0, 64], 0, 261, 128),
    ("bf16-window", [700, 130, 2, 256], 2, 64, 64, "bf16", [8, 8, 1, 8], [32, 0, 1, 248], 100,
     101, 128),
    ("bf16-small-window", [400], 2, 32, 32, "bf16", 2, 10, 5, 8, 128),
    ("bf16-all-targets", [64, 150], 2, 64, 64, "bf16", 0, [64, 150], 0, 10, 128),
    ("bf16-all-context", [64, 150], 2, 64, 64, "bf16", [64, 150], 0, 0, 151, 128),
    ("bf16-dqk-ne-dv", [90, 300], 2, 128, 64, "bf16", 1, 3, 0, 301, 128),
    # head dims the tensor-core forward runs zero-padded to 64 / 128
    ("bf16-d96-d48", [33, 260, 129], 2, 96, 48, "bf16", [1, 4, 0], [2, 9, 1], 0, 261, 128),
    ("bf16-d16-d112", [150, 7, 300], 3, 16, 112, "bf16", 2, [3, 0, 30], 60, 61, 128),
    # the widest rows (H * d_v = 2048) and the largest time table (256 buckets)
    ("bf16-max-width", [70, 300], 16, 128, 128, "bf16", [2, 0], [5, 17], 0, 301, 256),
]


@pytest.mark.parametrize("case", SMALL_CASES, ids=[c[0] for c in SMALL_CASES])
def test_fwd_parity_small(case):
    name, lengths, H, dqk, dv, dtype, ctx, tgt, W, R, NB = case
    b = synth.make_batch(np.random.default_rng(100), lengths, H, dqk, dv, dtype,
                         contextuals=ctx, targets=tgt, max_attn_len=W, rel_bias_len=R,
                         time_bias_len=NB)
    _fwd_check(b, what=name)


BF16_CASES = [c for c in SMALL_CASES if c[5] == "bf16"]


@pytest.mark.parametrize("case", BF16_CASES, ids=[c[0] for c in BF16_CASES])
def test_fwd_parity_small_inference(case):
    """The inference forward (bf16 pair arithmetic in the epilogue) on the small shapes."""
    name, lengths, H, dqk, dv, dtype, ctx, tgt, W, R, NB = case
    b = synth.make_batch(np.random.default_rng(102), lengths, H, dqk, dv, dtype,
                         contextuals=ctx, targets=tgt, max_attn_len=W, rel_bias_len=R,
                         time_bias_len=NB)
    _fwd_check(b, training=False, what=name + " inference")


@pytest.mark.parametrize("case", SMALL_CASES, ids=[c[0] for c in SMALL_CASES])
def test_bwd_parity_small(case):
    name, lengths, H, dqk, dv, dtype, ctx, tgt, W, R, NB = case
    b = synth.make_batch(np.random.default_rng(101), lengths, H, dqk, dv, dtype,
                         contextuals=ctx, targets=tgt, max_attn_len=W, rel_bias_len=R,
                         time_bias_len=NB, with_dout=True)
    dev = ops.batch_to_device(b)
    out, saved = ops.run_fwd(b, dev, training=True)
    dq, dk, dv_, du, drel, dtb = ops.run_bwd(b, saved, dev_tensors=dev)
    torch.cuda.synchronize()
    assert ops.read_device_status(ops.bwd.last_workspace) == 0
    ref = oracle.bwd(b)
    assert_close(_np(dq), ref["dq"], dtype, name + " dq")
    assert_close(_np(dk), ref["dk"], dtype, name + " dk")
    assert_close(_np(dv_), ref["dv"], dtype, name + " dv")
    assert_close(_np(du), ref["du"], dtype, name + " du")
    if R > 0:
        assert_close(_np(drel), ref["drel"], dtype, name + " drel")
    if NB > 0:
        assert_close(_np(dtb), ref["dtb"], dtype, name + " dtb")


# ------------------------------------------------------------------ the five workloads

def test_fwd_parity_tiny_fp32_workload():
    _fwd_check(synth.make_config(0), what="tiny fp32")


def test_fwd_parity_movielens_workload():
    _fwd_check(synth.make_config(1), what="movielens-shaped")


@pytest.mark.parametrize("cfg", [2, 3])
def test_fwd_parity_long_workloads_sampled(cfg):
    """Full-size batch on the GPU; the oracle checks whole sequences sampled from it
    (shortest, longest and one in between), which are independent given N."""
    b = synth.make_config(cfg)
    dev = ops.batch_to_device(b)
    out = ops.run_fwd(b, dev)
    torch.cuda.synchronize()
    assert ops.read_device_status(ops.fwd.last_workspace) == 0
    L = b.lengths
    seqs = sorted({int(np.argmin(L)), int(np.argmax(L)), int(np.argsort(L)[len(L) // 2])})
    ref = oracle.fwd(sub_batch(b, seqs))
    got = _np(out)[rows_of(b, seqs)]
    assert_close(got, ref["out"], b.dtype, "workload %d sampled out" % cfg)


def test_bwd_parity_tiny_fp32_workload():
    b = synth.make_config(0)
    b.dout = synth.draw_dout(b, 777)
    dev = ops.batch_to_device(b)
    _, saved = ops.run_fwd(b, dev, training=True)
    g = ops.run_bwd(b, saved, dev_tensors=dev)
    ref = oracle.bwd(b)
    for got, key in zip(g, ["dq", "dk", "dv", "du", "drel"]):
        assert_close(_np(got), ref[key], "f32", "tiny fp32 " + key)


def test_bwd_parity_training_workload():
    b = synth.make_config(4)
    dev = ops.batch_to_device(b)
    _, saved = ops.run_fwd(b, dev, training=True)
    g = ops.run_bwd(b, saved, dev_tensors=dev)
    torch.cuda.synchronize()
    assert ops.read_device_status(ops.bwd.last_workspace) == 0
    ref = oracle.bwd(b)
    for got, key in zip(g, ["dq", "dk", "dv", "du", "drel", "dtb"]):
        assert_close(_np(got), ref[key], "bf16", "training workload " + key)


# ------------------------------------------------------------------ mask structure

MASK_CASES = [(1, 0, 0, 0), (5, 2, 3, 0), (130, 4, 64, 0), (300, 8, 32, 50), (257, 0, 0, 0),
              (64, 64, 0, 0), (20, 0, 20, 0), (129, 1, 20, 1), (400, 3, 5, 127), (0, 0, 0, 0)]


@pytest.mark.parametrize("W", [0, 50])
def test_debug_mask_bit_exact(W):
    lengths = [c[0] for c in MASK_CASES]
    ctx = np.array([c[1] for c in MASK_CASES], np.int32)
    tgt = np.array([c[2] for c in MASK_CASES], np.int32)
    offs = np.zeros(len(lengths) + 1, np.int64)
    offs[1:] = np.cumsum(lengths)
    d_offs = torch.from_numpy(offs).cuda()
    d_ctx = torch.from_numpy(ctx).cuda()
    d_tgt = torch.from_numpy(tgt).cuda()
    p = ops.Params(batch=len(lengths), num_heads=1, d_qk=16, d_v=16, max_seqlen=max(lengths),
                   max_attn_len=W, total_tokens=int(offs[-1]), alpha=1.0, ln_eps=1e-5,
                   rel_bias_len=0, time_bias_len=0, time_bucket_div=0.301, dtype=ops.HSTU_BF16,
                   flags=0)
    for s, L in enumerate(lengths):
        got = ops.debug_mask(p, d_offs, d_ctx, d_tgt, s, L).numpy()
        ref, _ = oracle.mask(L, int(ctx[s]), int(tgt[s]), W)
        assert np.array_equal(got, ref.astype(bool)), (s, L, W)


# ------------------------------------------------------------------ page example on the GPU

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_page_signed_aggregation_on_gpu(dtype):
    """q_1 = e0, k_0 = -e0, k_1 = e0, V_0 = e0, V_1 = e1, zero biases: N*Y_1 = [SiLU(-1), SiLU(1)]
    ~ [-0.269, 0.731] as printed on the HSTU tensor-by-tensor page."""
    b = synth.make_batch(np.random.default_rng(0), [2], 1, 32, 32, dtype, rel_bias_len=0,
                         alpha=1.0)
    for a in (b.q, b.k, b.v):
        a[...] = 0.0
    b.u[...] = 1.0
    b.q[1, 0, 0] = 1.0
    b.k[0, 0, 0] = -1.0
    b.k[1, 0, 0] = 1.0
    b.v[0, 0, 0] = 1.0
    b.v[1, 0, 1] = 1.0
    _, saved = ops.run_fwd(b, training=True)
    y = _np(saved.y) * b.max_seqlen
    tol = 1e-5 if dtype == "f32" else 4e-3
    assert abs(y[1, 0] - (-0.269)) < 5e-4 + tol and abs(y[1, 1] - 0.731) < 5e-4 + tol
    assert np.all(y[0] == 0.0)


# ------------------------------------------------------------------ invariants

def test_changing_future_inputs_leaves_earlier_outputs_bitwise_unchanged():
    b = synth.make_batch(np.random.default_rng(5), [700, 300], 2, 64, 64, "bf16", contextuals=4,
                         targets=[16, 8], rel_bias_len=701, time_bias_len=128)
    out0 = _np(ops.run_fwd(b))
    for cut in [130, 400]:
        b2 = synth.make_batch(np.random.default_rng(5), [700, 300], 2, 64, 64, "bf16",
                              contextuals=4, targets=[16, 8], rel_bias_len=701, time_bias_len=128)
        rng = np.random.default_rng(cut)
        for name in ("q", "k", "v", "u"):
            a = getattr(b2, name)
            a[cut + 1:700] = synth.round_to_dtype(
                rng.standard_normal(a[cut + 1:700].shape).astype(np.float32), "bf16")
        b2.timestamps[cut + 1:700] += 1000
        out1 = _np(ops.run_fwd(b2))
        assert np.array_equal(out0[:cut + 1], out1[:cut + 1]), cut
        assert np.array_equal(out0[700:], out1[700:])        # other sequence untouched


def test_candidate_isolation_bitwise():
    b = synth.make_batch(np.random.default_rng(6), [300], 2, 64, 64, "bf16", contextuals=2,
                         targets=20, rel_bias_len=301, time_bias_len=128)
    out0 = _np(ops.run_fwd(b))
    m = 290
    for name in ("q", "k", "v", "u"):
        getattr(b, name)[m] *= -1.0
    out1 = _np(ops.run_fwd(b))
    others = [i for i in range(300) if i != m]
    assert np.array_equal(out0[others], out1[others])


def test_forward_is_deterministic():
    b = synth.make_config(1)
    dev = ops.batch_to_device(b)
    a = ops.run_fwd(b, dev).clone()
    c = ops.run_fwd(b, dev)
    assert torch.equal(a, c)


# ------------------------------------------------------------------ edge cases and faults

def test_empty_batch_and_zero_length_sequences():
    b = synth.make_batch(np.random.default_rng(8), [0, 0, 3, 0], 2, 64, 64, "bf16",
                         rel_bias_len=4, time_bias_len=128)
    _fwd_check(b, what="zero-length")
    dev = ops.batch_to_device(b)
    e = synth.make_batch(np.random.default_rng(8), [], 2, 64, 64, "bf16", rel_bias_len=4,
                         max_seqlen=1)
    out = ops.run_fwd(e)
    assert out.shape == (0, 128)
    del dev


def test_bad_device_data_is_reported_and_the_context_stays_usable():
    b = synth.make_batch(np.random.default_rng(9), [10, 20, 30], 2, 64, 64, "bf16",
                         contextuals=[1, 2, 3], targets=[1, 2, 3], rel_bias_len=31,
                         time_bias_len=128)
    dev = ops.batch_to_device(b)
    bad = dict(dev)
    bad["num_targets"] = torch.tensor([1, 25, 3], dtype=torch.int32, device="cuda")   # c+t > L
    ops.run_fwd(b, bad)
    assert ops.read_device_status(ops.fwd.last_workspace) & ops.DEV_BAD_COUNTS
    bad = dict(dev)
    bad["seq_offsets"] = torch.tensor([0, 10, 5, 60], dtype=torch.int64, device="cuda")
    ops.run_fwd(b, bad)
    assert ops.read_device_status(ops.fwd.last_workspace) & ops.DEV_BAD_OFFSETS
    short = dict(alpha=b.alpha, max_seqlen=20, max_attn_len=0)
    ops.fwd(dev["q"], dev["k"], dev["v"], dev["u"], dev["seq_offsets"], dev["num_contextuals"],
            dev["num_targets"], dev["timestamps"], dev["rel_bias"], dev["time_bias"], **short)
    assert ops.read_device_status(ops.fwd.last_workspace) & ops.DEV_SEQ_TOO_LONG
    # a valid call afterwards still matches the oracle
    _fwd_check(b, what="after bad data")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_uncovered_rows_are_zero_and_flagged(dtype):
    """Offsets that start after row 0 or end before row T, and a sequence skipped for bad
    counts: the status word says so, the rows no valid sequence covers come out as zeros in
    out, saved Y, dK and dV, and the other sequences still match the oracle."""
    lengths = [30, 150, 60, 40]
    b = synth.make_batch(np.random.default_rng(12), lengths, 2, 64, 64, dtype,
                         contextuals=[1, 2, 3, 1], targets=[2, 5, 3, 1], rel_bias_len=151,
                         time_bias_len=128, with_dout=True)
    dev = ops.batch_to_device(b)
    offs = b.seq_offsets.copy()
    offs[0] = 5                   # rows 0..4 uncovered; sequence 0 skipped (does not start at 0)
    offs[-1] -= 7                 # last sequence ends 7 rows short of T: skipped
    bad = dict(dev)
    bad["seq_offsets"] = torch.from_numpy(offs).cuda()
    bad["num_targets"] = torch.tensor([2, 500, 3, 1], dtype=torch.int32, device="cuda")
    T = b.total_tokens
    out, saved = ops.run_fwd(b, bad, training=True)
    code = ops.read_device_status(ops.fwd.last_workspace)
    assert code & ops.DEV_BAD_OFFSETS and code & ops.DEV_BAD_COUNTS
    g = ops.run_bwd(b, saved, dev_tensors=bad)
    torch.cuda.synchronize()
    dead = np.zeros(T, bool)
    dead[:offs[1]] = True                        # rows 0..4 and sequence 0
    dead[offs[1]:offs[2]] = True                 # sequence 1 (c + t > L)
    dead[offs[3]:] = True                        # sequence 3 and the 7 rows after it
    for t_, name in ((out, "out"), (saved.y, "y"), (g[1], "dk"), (g[2], "dv"), (g[0], "dq"),
                     (g[3], "du")):
        a = _np(t_).reshape(T, -1)
        assert np.all(a[dead] == 0), name + ": an uncovered row is not zero"
    # sequence 2 alone is intact
    ref = oracle.fwd(sub_batch(b, [2]))
    rows = rows_of(b, [2])
    assert_close(_np(out)[rows], ref["out"], dtype, "intact sequence out")


# ------------------------------------------------------------------ timestamp orders and ranges
#
# The workloads draw ascending timestamps; the kernels exploit ascending order only for
# speed (runs of equal buckets, one-boundary blocks).  Any order and any range is an input
# the library must get right: shuffled stamps inside each sequence, and gaps beyond 2^31
# that force the 64-bit bucket search.

def _stamped(seed, stamps, dqk=128, dv=128):
    lengths = [130, 300, 77, 256]
    b = synth.make_batch(np.random.default_rng(seed), lengths, 2, dqk, dv, "bf16",
                         contextuals=[1, 4, 0, 3], targets=[5, 40, 2, 0], rel_bias_len=301,
                         time_bias_len=128, with_dout=True)
    rng = np.random.default_rng(seed + 1)
    ts = b.timestamps.copy()
    for s in range(b.batch):
        a, e = int(b.seq_offsets[s]), int(b.seq_offsets[s + 1])
        if stamps == "shuffled":
            ts[a:e] = rng.permutation(ts[a:e])
        elif stamps == "huge-gaps":
            gaps = rng.choice([1, 3600, 1 << 33, 7 << 40], size=e - a, p=[0.3, 0.4, 0.2, 0.1])
            ts[a:e] = 1_000_000_000 + np.cumsum(gaps)
    import dataclasses
    return dataclasses.replace(b, timestamps=ts)


@pytest.mark.parametrize("stamps", ["shuffled", "huge-gaps"])
@pytest.mark.parametrize("dims", [(128, 128), (64, 64)])
def test_fwd_bwd_parity_any_timestamp_order(stamps, dims):
    b = _stamped(300, stamps, *dims)
    name = "%s d=%s" % (stamps, dims)
    _fwd_check(b, training=False, what=name + " inference")
    dev = ops.batch_to_device(b)
    out, saved = ops.run_fwd(b, dev, training=True)
    dq, dk, dv_, du, drel, dtb = ops.run_bwd(b, saved, dev_tensors=dev)
    torch.cuda.synchronize()
    assert ops.read_device_status(ops.bwd.last_workspace) == 0
    ref = oracle.bwd(b)
    for got, key in ((dq, "dq"), (dk, "dk"), (dv_, "dv"), (du, "du"), (drel, "drel"),
                     (dtb, "dtb")):
        assert_close(_np(got), ref[key], "bf16", name + " " + key)


# ------------------------------------------------------------------ work-unit hand-out

def _fwd_bwd_check(b, name, seqs=None):
    """Inference and training forward, then backward, against the oracle; with `seqs` the
    per-token outputs are compared on those sequences only (the table gradients need all)."""
    dev = ops.batch_to_device(b)
    out_inf = ops.run_fwd(b, dev)
    out, saved = ops.run_fwd(b, dev, training=True)
    g = ops.run_bwd(b, saved, dev_tensors=dev)
    torch.cuda.synchronize()
    assert ops.read_device_status(ops.fwd.last_workspace) == 0
    assert ops.read_device_status(ops.bwd.last_workspace) == 0
    ref_f = oracle.fwd(b if seqs is None else sub_batch(b, seqs))
    ref_b = oracle.bwd(b)
    rows = slice(None) if seqs is None else rows_of(b, seqs)
    assert_close(_np(out_inf)[rows], ref_f["out"], b.dtype, name + " inference out")
    assert_close(_np(out)[rows], ref_f["out"], b.dtype, name + " training out")
    for got, key in zip(g, ["dq", "dk", "dv", "du", "drel", "dtb"]):
        assert_close(_np(got), ref_b[key], b.dtype, name + " " + key)


def test_more_sequences_than_the_tile_cache():
    """2100 sequences (the per-CTA cache of tile counts holds 2048): every unit is drawn
    and checked against its sequence; empty sequences and two-tile ones among them."""
    rng = np.random.default_rng(2100)
    lengths = rng.integers(0, 41, size=2100)
    lengths[[5, 700, 2099]] = [129, 200, 150]
    lengths[[6, 7, 1500]] = 0
    tgt = np.minimum(rng.integers(0, 4, size=2100), lengths)
    b = synth.make_batch(rng, lengths, 2, 64, 64, "bf16", contextuals=0, targets=tgt,
                         rel_bias_len=int(lengths.max()) + 1, time_bias_len=128,
                         with_dout=True)
    _fwd_bwd_check(b, "2100 sequences")


def test_tile_count_past_the_cache_range():
    """A sequence of 33,000 tokens has more 128-row tiles than the cache counts (255): its
    units past that count are checked against the sequence itself.  Windowed, so the
    oracle stays quick."""
    rng = np.random.default_rng(33000)
    lengths = [33000, 17, 300]
    b = synth.make_batch(rng, lengths, 1, 64, 64, "bf16", contextuals=[2, 0, 1],
                         targets=[8, 3, 20], max_attn_len=64, rel_bias_len=65,
                         time_bias_len=128, with_dout=True)
    _fwd_bwd_check(b, "33000-token sequence")


# ------------------------------------------------------------------ table-size branches
#
# The backward keeps the rel table in shared memory up to 2048 entries and the forward up
# to 4352; longer tables are read (and the backward's gradient added) in global memory.
# Sequences of config-2-like lengths with R = N + 1 reach those branches; a window keeps the
# oracle quick while contextual keys far back still use the high table indices.

def _long_table_batch(seed, lengths, W, H=2):
    N = int(max(lengths))
    return synth.make_batch(np.random.default_rng(seed), lengths, H, 128, 128, "bf16",
                            contextuals=4, targets=64, max_attn_len=W, rel_bias_len=N + 1,
                            time_bias_len=128, with_dout=True)


def test_bwd_parity_rel_table_in_global_memory():
    b = _long_table_batch(2049, [3100, 4096, 700], W=256)
    assert b.rel_bias_len > 2048
    _fwd_bwd_check(b, "R=%d backward" % b.rel_bias_len)


def test_fwd_parity_rel_table_in_global_memory():
    b = _long_table_batch(4353, [4500, 1300], W=300)
    assert b.rel_bias_len > 4352
    _fwd_bwd_check(b, "R=%d forward" % b.rel_bias_len)


@pytest.mark.parametrize("cfg", [2, 3])
def test_training_forward_long_workloads_sampled(cfg):
    """The training forward (A carried as a bf16 hi + lo pair) on the full long-history and
    windowed batches; out, Y, mean and rstd checked on sampled whole sequences."""
    b = synth.make_config(cfg)
    dev = ops.batch_to_device(b)
    out, saved = ops.run_fwd(b, dev, training=True)
    torch.cuda.synchronize()
    assert ops.read_device_status(ops.fwd.last_workspace) == 0
    L = b.lengths
    seqs = sorted({int(np.argmin(L)), int(np.argmax(L))})
    ref = oracle.fwd(sub_batch(b, seqs))
    rows = rows_of(b, seqs)
    for got, key in ((out, "out"), (saved.y, "y"), (saved.mean, "mean"), (saved.rstd, "rstd")):
        assert_close(_np(got)[rows], ref[key], b.dtype, "workload %d training %s" % (cfg, key))


# ------------------------------------------------------------------ guard bands
#
# Every output (and the workspace) sits inside a larger buffer whose bytes before and after
# it hold NaN (or 0xFF bytes); after the calls those bands must be untouched: no kernel
# writes outside the buffers it was given.

_PAD = 4096


class _Guarded:
    def __init__(self):
        self.bufs = []

    def alloc(self, shape, dtype):
        n = int(np.prod(shape)) if len(shape) else 1
        if dtype == torch.uint8:
            whole = torch.full((2 * _PAD + n,), 0xFF, dtype=dtype, device="cuda")
        else:
            whole = torch.full((2 * _PAD + n,), float("nan"), dtype=dtype, device="cuda")
        self.bufs.append((whole, n))
        return whole[_PAD:_PAD + n].view(*shape)

    def check(self, what):
        torch.cuda.synchronize()
        for whole, n in self.bufs:
            for band in (whole[:_PAD], whole[_PAD + n:]):
                if whole.dtype == torch.uint8:
                    assert bool((band == 0xFF).all()), what + ": a guard band was written"
                else:
                    assert bool(torch.isnan(band.float()).all()), what + ": a guard band was written"


@pytest.mark.parametrize("case", [c for c in SMALL_CASES if c[0] in
                                  ("bf16-family", "bf16-window", "f32-full-family",
                                   "bf16-dqk-ne-dv")], ids=lambda c: c[0])
def test_outputs_stay_inside_their_buffers(case):
    name, lengths, H, dqk, dv, dtype, ctx, tgt, W, R, NB = case
    b = synth.make_batch(np.random.default_rng(77), lengths, H, dqk, dv, dtype,
                         contextuals=ctx, targets=tgt, max_attn_len=W, rel_bias_len=R,
                         time_bias_len=NB, with_dout=True)
    dev = ops.batch_to_device(b)
    kw = ops.batch_kwargs(b)
    tdt = dev["q"].dtype
    T, D = b.u.shape
    g = _Guarded()
    p = ops.make_params(dev["q"], dev["v"], dev["seq_offsets"], alpha=b.alpha,
                        max_seqlen=b.max_seqlen, max_attn_len=b.max_attn_len,
                        rel_bias=dev["rel_bias"], time_bias=dev["time_bias"])
    out = g.alloc((T, D), tdt)
    saved = ops.Saved(g.alloc((T, D), torch.float32), g.alloc((T,), torch.float32),
                      g.alloc((T,), torch.float32))
    ws_f = g.alloc((ops.fwd_workspace_size(p),), torch.uint8)
    args = (dev["q"], dev["k"], dev["v"], dev["u"], dev["seq_offsets"], dev["num_contextuals"],
            dev["num_targets"], dev["timestamps"], dev["rel_bias"], dev["time_bias"])
    ops.fwd(*args, out=out, workspace=ws_f, **kw)
    g.check(name + " inference forward")
    ops.fwd(*args, training=True, out=out, saved=saved, workspace=ws_f, **kw)
    g.check(name + " training forward")
    grads = (g.alloc(tuple(b.q.shape), tdt), g.alloc(tuple(b.k.shape), tdt),
             g.alloc(tuple(b.v.shape), tdt), g.alloc((T, D), tdt),
             g.alloc((R,), torch.float32) if R else None,
             g.alloc((NB,), torch.float32) if NB else None)
    ws_b = g.alloc((ops.bwd_workspace_size(p),), torch.uint8)
    ops.bwd(dev["dout"], *args, saved=saved, grads=grads, workspace=ws_b, **kw)
    g.check(name + " backward")
    ref = oracle.bwd(b)
    assert_close(_np(out), oracle.fwd(b)["out"], dtype, name + " guarded out")
    assert_close(_np(grads[0]), ref["dq"], dtype, name + " guarded dq")


# ------------------------------------------------------------------ bounded waits

def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    """The MMA issuer of both tensor-core kernels waits on a barrier nothing completes, with
    a limit of 2e7 cycles (about 10 ms): the wait runs out, HSTU_DEV_WAIT_TIMEOUT is set,
    every role unwinds, and the next normal calls still match the oracle."""
    b = synth.make_batch(np.random.default_rng(15), [70, 300, 129], 2, 128, 128, "bf16",
                         contextuals=[1, 2, 3], targets=[2, 20, 1], rel_bias_len=301,
                         time_bias_len=128, with_dout=True)
    dev = ops.batch_to_device(b)
    try:
        ops.set_wait_test(20_000_000, stall=True)
        out, saved = ops.run_fwd(b, dev, training=True)
        assert ops.read_device_status(ops.fwd.last_workspace) & ops.DEV_WAIT_TIMEOUT
        ops.run_bwd(b, saved, dev_tensors=dev)
        assert ops.read_device_status(ops.bwd.last_workspace) & ops.DEV_WAIT_TIMEOUT
    finally:
        ops.set_wait_test(0, stall=False)
    _fwd_bwd_check(b, "after the stall test")


# ------------------------------------------------------------------ mask variants
#
# Contextual rows that see the whole history (flag 1) and the rel index |p(i) - p(j)| (flag 2),
# through both tensor-core kernels and the CUDA-core path: values against the oracle, and
# the tensor-core kernels' masked-pair structure bit for bit.

VARIANT_CASES = [
    # name, lengths, H, dqk, dv, dtype, ctx, tgt, W, R, NB
    ("bf16-family", [5, 200, 77, 260, 129], 2, 128, 128, "bf16", [1, 4, 0, 8, 3],
     [2, 20, 5, 0, 64], 0, 261, 128),
    ("bf16-window", [700, 130, 2, 256], 2, 64, 64, "bf16", [8, 40, 1, 130], [32, 0, 1, 60], 100,
     101, 128),
    ("bf16-all-targets", [64, 150], 2, 64, 64, "bf16", [0, 3], [64, 100], 0, 10, 128),
    ("f32-family", [5, 200, 77], 2, 32, 48, "f32", [1, 4, 3], [2, 20, 5], 9, 40, 64),
]


@pytest.mark.parametrize("flags", [1, 2, 3])
@pytest.mark.parametrize("case", VARIANT_CASES, ids=[c[0] for c in VARIANT_CASES])
def test_mask_variants_fwd_bwd_parity(case, flags):
    name, lengths, H, dqk, dv, dtype, ctx, tgt, W, R, NB = case
    b = synth.make_batch(np.random.default_rng(90 + flags), lengths, H, dqk, dv, dtype,
                         contextuals=ctx, targets=tgt, max_attn_len=W, rel_bias_len=R,
                         time_bias_len=NB, with_dout=True, mask_flags=flags)
    _fwd_bwd_check(b, "%s flags=%d" % (name, flags))


@pytest.mark.parametrize("flags", [1, 3])
def test_mask_variants_kernel_mask_bit_exact(flags):
    seqs = [(1, 1, 0), (33, 5, 3), (129, 40, 32), (300, 130, 60), (257, 129, 127), (70, 0, 70)]
    lengths = [q[0] for q in seqs]
    offs = np.zeros(len(seqs) + 1, np.int64)
    offs[1:] = np.cumsum(lengths)
    d_offs = torch.from_numpy(offs).cuda()
    d_ctx = torch.tensor([q[1] for q in seqs], dtype=torch.int32, device="cuda")
    d_tgt = torch.tensor([q[2] for q in seqs], dtype=torch.int32, device="cuda")
    for W in (0, 33):
        p = ops.Params(batch=len(seqs), num_heads=1, d_qk=64, d_v=64, max_seqlen=max(lengths),
                       max_attn_len=W, total_tokens=int(offs[-1]), alpha=1.0, ln_eps=1e-5,
                       rel_bias_len=0, time_bias_len=0, time_bucket_div=0.301,
                       dtype=ops.HSTU_BF16, flags=flags)
        for s, (L, c, t) in enumerate(seqs):
            pad = (L + 127) // 128 * 128
            ref = oracle.mask_rows(L, c, t, W, 0, pad, pad, flags).astype(bool)
            for kernel in ("fwd", "bwd"):
                got = ops.debug_kernel_mask(p, d_offs, d_ctx, d_tgt, s, kernel, 0, pad,
                                            pad).numpy()
                assert np.array_equal(got[:L, :L], ref[:L, :L]), (kernel, L, c, t, W, flags)
                if kernel == "fwd":
                    assert not got[:L, L:].any()
                else:
                    assert not got[L:, :L].any()
