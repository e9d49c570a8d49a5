"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each test pins one part of the oracle to something other than itself: values the pages
print, hand-derived masks, closed forms, a second (padded-dense) formulation, special
cases that reduce to prefix sums, high-precision evaluation of the bucket boundaries,
and central finite differences for the backward.
"""
import math
from decimal import Decimal, getcontext

import numpy as np
import pytest

from jagged_hstu_attention_02_b200 import accounting, synth
from oracle import dense, oracle

E_CONST = math.e


def _read_kv(path):
    out = {}
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        key, *vals = line.split()
        out[key] = [float(x) for x in vals]
    return out


def _empty_batch(lengths, H, d_qk, d_v, *, ctx=0, tgt=0, W=0, R=0, NB=0, alpha=1.0, N=None):
    rng = np.random.default_rng(0)
    b = synth.make_batch(rng, lengths, H, d_qk, d_v, "f32", contextuals=ctx, targets=tgt,
                         max_attn_len=W, rel_bias_len=R, time_bias_len=NB, alpha=alpha,
                         max_seqlen=N)
    for name in ("q", "k", "v", "u"):
        getattr(b, name)[...] = 0.0
    if b.rel_bias is not None:
        b.rel_bias[...] = 0.0
    if b.time_bias is not None:
        b.time_bias[...] = 0.0
    b.u[...] = 1.0
    return b


# ---------------------------------------------------------------- page values

def test_silu_values_and_signed_aggregation(golden_dir):
    """q_1 = e0, k_0 = -e0, k_1 = e0, V_0 = e0, V_1 = e1: N*Y_1 = SiLU(-1) V_0 + SiLU(1) V_1."""
    g = _read_kv(f"{golden_dir}/page_silu_values.txt")
    b = _empty_batch([2], 1, 32, 32, R=0, NB=0, alpha=1.0)
    b.q[1, 0, 0] = 1.0
    b.k[0, 0, 0] = -1.0
    b.k[1, 0, 0] = 1.0
    b.v[0, 0, 0] = 1.0
    b.v[1, 0, 1] = 1.0
    r = oracle.fwd(b)
    N = b.max_seqlen
    agg = N * r["y"][1, :2]
    # the page's printed three-decimal values
    assert abs(agg[0] - g["aggregate_0"][0]) < 5e-4
    assert abs(agg[1] - g["aggregate_1"][0]) < 5e-4
    assert abs(agg[0] - g["silu_at_minus_1"][0]) < 5e-4
    assert abs(agg[1] - g["silu_at_1"][0]) < 5e-4
    # closed forms: SiLU(-1) = -1/(1+e), SiLU(1) = 1/(1+1/e)
    assert abs(agg[0] - (-1.0 / (1.0 + E_CONST))) < 1e-15
    assert abs(agg[1] - (1.0 / (1.0 + 1.0 / E_CONST))) < 1e-15
    # the aggregate lies outside the segment between [1,0] and [0,1] (coefficients sum != 1)
    assert agg[0] < 0 and abs(agg.sum() - 1.0) > 0.5
    # row 0: q_0 = 0, so s_00 = 0 and SiLU(0) = 0 -> Y_0 = 0 exactly, and O_0 = 0
    assert np.all(r["y"][0] == 0.0) and g["silu_at_0"][0] == 0.0
    assert np.all(r["out"][0] == 0.0)
    assert np.all(r["y"][1, 2:] == 0.0)


def test_row_sums_are_not_one():
    """With V = 1 the row sums N*Y_i = sum_j SiLU(s_ij) are not 1 (no softmax)."""
    b = synth.make_batch(np.random.default_rng(7), [4, 9], 1, 8, 8, "f32", rel_bias_len=10)
    b.v[...] = 1.0
    r = oracle.fwd(b)
    sums = b.max_seqlen * r["y"][:, 0]
    assert np.all(np.abs(sums - 1.0) > 1e-3)
    # every column of a head carries the same row sum when V = 1
    assert np.allclose(r["y"], r["y"][:, :1], rtol=0, atol=1e-15)


def test_padding_arithmetic(golden_dir):
    g = _read_kv(f"{golden_dir}/page_padding_arithmetic.txt")
    lengths = [int(x) for x in g["lengths"]]
    padded, ragged, ratio = accounting.padding_stats(lengths)
    assert padded == g["padded"][0] and ragged == g["ragged"][0]
    assert ratio == g["pair_work_dense"][0] / g["pair_work_ragged"][0] or \
        float(ratio) == pytest.approx(g["pair_work_dense"][0] / g["pair_work_ragged"][0], rel=1e-15)
    assert round(float(ratio), 3) == 2.970
    # the per-sequence causal pair work equals the oracle's valid-pair count
    n = sum(oracle.mask(L)[1] for L in lengths)
    assert n == sum(L * (L + 1) // 2 for L in lengths) == 505605


# ---------------------------------------------------------------- mask

def _golden_masks(golden_dir):
    lines = [ln.split("#")[0].strip() for ln in open(f"{golden_dir}/mask_examples.txt")]
    lines = [ln for ln in lines if ln]
    out, i = [], 0
    while i < len(lines):
        _, L, c, t, W, n = lines[i].split()
        L, c, t, W, n = int(L), int(c), int(t), int(W), int(n)
        rows = lines[i + 1:i + 1 + L]
        m = np.array([[int(ch) for ch in row] for row in rows], dtype=np.uint8)
        out.append((L, c, t, W, n, m))
        i += 1 + L
    return out


def test_mask_hand_examples(golden_dir):
    for L, c, t, W, n, m in _golden_masks(golden_dir):
        got, cnt = oracle.mask(L, c, t, W)
        assert np.array_equal(got, m), (L, c, t, W)
        assert cnt == n == int(m.sum())
        assert accounting.valid_pairs_seq(L, c, t, W) == n
        assert np.array_equal(dense._mask_dense(L, c, t, W, L).astype(np.uint8), m)


@pytest.mark.parametrize("W", [0, 1, 3, 50])
def test_mask_counts_closed_form(W):
    for L in [0, 1, 2, 5, 17, 40]:
        for c in range(0, min(L, 4) + 1):
            for t in range(0, L - c + 1, max(1, (L - c) // 3 or 1)):
                m, cnt = oracle.mask(L, c, t, W)
                assert cnt == accounting.valid_pairs_seq(L, c, t, W), (L, c, t, W)
                dm = dense._mask_dense(L, c, t, W, L)
                assert np.array_equal(m.astype(bool), dm), (L, c, t, W)


def test_mask_structure_invariants():
    for L, c, t, W in [(30, 3, 5, 0), (30, 0, 0, 4), (25, 2, 25 - 2, 0), (40, 5, 7, 6)]:
        m, _ = oracle.mask(L, c, t, W)
        E = L - t
        # no history or contextual row sees a candidate key
        assert m[:E, E:].sum() == 0
        # a candidate key is seen only by itself
        for j in range(E, L):
            assert m[:, j].sum() == 1 and m[j, j] == 1
        # the contextual block is all ones and contextual rows see nothing else
        assert m[:c, :c].all() and m[:c, c:].sum() == 0
        # every non-contextual row sees its own position when it is history
        for i in range(c, E):
            assert m[i, i] == 1 and m[i, i + 1:].sum() == 0


# ---------------------------------------------------------------- time buckets

def _bucket_exact(dt, div="0.301", nb=128):
    getcontext().prec = 60
    x = (Decimal(abs(dt)) + 1).ln() / Decimal(div)
    return min(int(x), nb - 1)


def test_time_bucket_values():
    for dt in [0, 1, 2, 3, 10, 59, 60, 3600, 86400, 2592000, 31536000, -3600, 10 ** 12,
               10 ** 17, -(2 ** 63) + 1]:
        assert oracle.time_bucket(dt, 0.301, 128) == _bucket_exact(dt), dt
    assert oracle.time_bucket(1, 0.301, 128) == 2          # ln 2 / 0.301 = 2.30
    assert oracle.time_bucket(3600, 0.301, 128) == 27      # ln 3601 / 0.301 = 27.2
    assert oracle.time_bucket(5, 0.301, 4) == 3            # clamped to NB - 1


def test_time_bucket_boundaries():
    """T_k = ceil(exp(0.301 k) - 1), the first |dt| of bucket k, evaluated in 60 digits.

    The oracle evaluates floor(log(|dt|+1)/0.301) in fp64.  At |dt| = T_k - 1 and T_k the
    fp64 decision must equal the exact one, except where the exact quotient lies within
    1e-13 (relative) of the integer k: there fp64 rounding decides, and the device takes the
    same fp64 decision (its threshold table is derived from the same fp64 evaluation).
    """
    getcontext().prec = 60
    thr = []
    for kk in range(1, 128):
        x = (Decimal("0.301") * kk).exp() - 1
        thr.append(int(x.to_integral_value(rounding="ROUND_CEILING")))
    rounding_decided = []
    for kk, T in enumerate(thr, start=1):
        for dt in ([T - 1, T] if T >= 1 else [T]):
            expect = sum(1 for tt in thr if tt <= dt)
            got = oracle.time_bucket(dt, 0.301, 128)
            if got == expect:
                continue
            xq = (Decimal(dt) + 1).ln() / Decimal("0.301")
            near = abs(xq - xq.to_integral_value()) < Decimal("1e-13") * xq
            assert near and abs(got - expect) == 1, (kk, dt, got, expect)
            rounding_decided.append((kk, dt, got))
    # fp64 rounding decides only where one unit of |dt| moves the quotient by a few ulps:
    # |dt| above 1e13 (over 300,000 years in seconds); below that fp64 equals exact math.
    assert all(dt > 10 ** 13 for _, dt, _ in rounding_decided), rounding_decided
    assert oracle.time_bucket(53195770115074, 0.301, 128) == 105   # exact value: 104


# ---------------------------------------------------------------- bias structure

def test_rel_bias_one_hot_direction_and_clamp():
    """Q = K = 0 and a one-hot rel table at r: N*Y_i = SiLU(1) * sum_{valid j, idx(i,j)=r} V_j."""
    silu1 = 1.0 / (1.0 + 1.0 / E_CONST)
    L, R = 12, 5
    for r in [0, 2, R - 1]:
        b = _empty_batch([L], 1, 16, 4, R=R)
        b.rel_bias[r] = 1.0
        b.v[:, 0, :] = np.random.default_rng(r).standard_normal((L, 4))
        y = oracle.fwd(b)["y"] * b.max_seqlen
        V = b.v[:, 0, :].astype(np.float64)
        for i in range(L):
            if r < R - 1:
                expect = silu1 * V[i - r] if i - r >= 0 else np.zeros(4)
            else:   # clamped index: every key at distance >= R-1
                expect = silu1 * V[: i - r + 1].sum(axis=0) if i - r >= 0 else np.zeros(4)
            assert np.allclose(y[i], expect, atol=1e-14), (r, i)


def test_rel_bias_negative_distance_clamps_to_zero():
    """Contextual rows see later contextual keys (p(i) < p(j)); that index clamps to 0."""
    silu1 = 1.0 / (1.0 + 1.0 / E_CONST)
    b = _empty_batch([6], 1, 16, 4, ctx=3, R=4)
    b.rel_bias[0] = 1.0
    b.v[:, 0, :] = np.random.default_rng(1).standard_normal((6, 4))
    y = oracle.fwd(b)["y"] * b.max_seqlen
    V = b.v[:, 0, :].astype(np.float64)
    # row 0 (contextual) sees keys 0, 1, 2 with distances 0, -1, -2 -> all index 0
    assert np.allclose(y[0], silu1 * V[:3].sum(0), atol=1e-14)
    # row 1 sees 0 (distance 1 -> zero bias), 1 and 2 (index 0)
    assert np.allclose(y[1], silu1 * V[1:3].sum(0), atol=1e-14)


def test_time_bias_one_hot_and_candidate_clamping():
    """Q = K = 0, one-hot time table: only pairs whose bucket matches contribute SiLU(1)*V_j.
    Candidates use the clamped position's timestamp (their own timestamp is unused)."""
    silu1 = 1.0 / (1.0 + 1.0 / E_CONST)
    L, t = 8, 2
    b = _empty_batch([L], 1, 16, 4, tgt=t, NB=128)
    ts = np.array([0, 1, 3600, 3601, 90000, 90001, 10 ** 9, 5], dtype=np.int64) + 10 ** 9
    b.timestamps = ts
    b.v[:, 0, :] = np.random.default_rng(3).standard_normal((L, 4))
    V = b.v[:, 0, :].astype(np.float64)
    E = L - t
    p = [i if i < E else E - 1 for i in range(L)]
    for k in [0, 2, 27, 37]:
        b.time_bias[...] = 0.0
        b.time_bias[k] = 1.0
        y = oracle.fwd(b)["y"] * b.max_seqlen
        m, _ = oracle.mask(L, 0, t, 0)
        for i in range(L):
            expect = np.zeros(4)
            for j in range(L):
                if m[i, j] and _bucket_exact(int(ts[p[i]] - ts[p[j]])) == k:
                    expect += silu1 * V[j]
            assert np.allclose(y[i], expect, atol=1e-14), (k, i)
    # perturbing the candidates' own timestamps changes nothing
    b.time_bias[...] = np.random.default_rng(4).standard_normal(128) * 0.1
    r0 = oracle.fwd(b)
    b.timestamps = ts.copy()
    b.timestamps[E:] += 123456789
    r1 = oracle.fwd(b)
    assert np.array_equal(r0["out"], r1["out"])


def test_constant_bias_reduces_to_prefix_sums():
    """Q = K = 0 and a constant rel table beta = 1: N*Y_i = SiLU(1) * sum_{j<=i} V_j (causal)."""
    silu1 = 1.0 / (1.0 + 1.0 / E_CONST)
    L = 37
    b = _empty_batch([L, 5], 2, 8, 8, R=64)
    b.rel_bias[...] = 1.0
    b.v[...] = np.random.default_rng(5).standard_normal(b.v.shape)
    y = oracle.fwd(b)["y"] * b.max_seqlen
    for s, (lo, hi) in enumerate([(0, L), (L, L + 5)]):
        for h in range(2):
            pref = np.cumsum(b.v[lo:hi, h, :].astype(np.float64), axis=0) * silu1
            assert np.allclose(y[lo:hi, h * 8:(h + 1) * 8], pref, atol=1e-13)


# ---------------------------------------------------------------- layer norm + gating

def test_layernorm_properties():
    b = synth.make_batch(np.random.default_rng(11), [7, 30], 2, 8, 16, "f32", rel_bias_len=31,
                         time_bias_len=16, contextuals=[1, 2], targets=[2, 3])
    r = oracle.fwd(b)
    z = r["out"] / b.u
    var = r["y"].var(axis=1)
    assert np.allclose(z.mean(axis=1), 0.0, atol=1e-12)
    assert np.allclose(z.var(axis=1), var / (var + b.ln_eps), rtol=1e-12)
    assert np.allclose(r["mean"], r["y"].mean(axis=1), atol=1e-15)
    # V = 0 gives Y = 0 and O = 0
    b.v[...] = 0.0
    r = oracle.fwd(b)
    assert np.all(r["y"] == 0.0) and np.all(r["out"] == 0.0)


# ---------------------------------------------------------------- jagged == padded dense

@pytest.mark.parametrize("case", [
    dict(lengths=[10, 100, 1000][:2] + [57], H=2, d=32, ctx=0, tgt=0, W=0, R=101, NB=0),
    dict(lengths=[1, 9, 33, 64, 2], H=2, d=16, ctx=[0, 2, 4, 1, 0], tgt=[1, 3, 5, 0, 2], W=0,
         R=65, NB=32),
    dict(lengths=[40, 25, 3], H=3, d=8, ctx=2, tgt=[4, 4, 1], W=5, R=7, NB=128),
    dict(lengths=[0, 12, 0, 20], H=1, d=8, ctx=[0, 3, 0, 0], tgt=[0, 9, 0, 20], W=0, R=30,
         NB=8),
])
def test_jagged_equals_padded_dense(case):
    b = synth.make_batch(np.random.default_rng(21), case["lengths"], case["H"], case["d"],
                         case["d"], "f32", contextuals=case["ctx"], targets=case["tgt"],
                         max_attn_len=case["W"], rel_bias_len=case["R"],
                         time_bias_len=case["NB"])
    a = oracle.fwd(b)
    d = dense.fwd(b)
    for key in ("y", "out", "mean", "rstd"):
        ref = np.abs(d[key]).max() if d[key].size else 1.0
        assert np.abs(a[key] - d[key]).max(initial=0.0) <= 1e-12 * max(ref, 1.0), key


# ---------------------------------------------------------------- causality

def test_changing_future_inputs_leaves_earlier_outputs_unchanged():
    b = synth.make_batch(np.random.default_rng(31), [50], 2, 16, 16, "f32", contextuals=3,
                         targets=6, rel_bias_len=51, time_bias_len=64)
    r0 = oracle.fwd(b)
    E = 50 - 6
    for cut in [10, 25, E - 1]:
        b2 = synth.make_batch(np.random.default_rng(31), [50], 2, 16, 16, "f32", contextuals=3,
                              targets=6, rel_bias_len=51, time_bias_len=64)
        rng = np.random.default_rng(cut)
        for name in ("q", "k", "v", "u"):
            arr = getattr(b2, name)
            arr[cut + 1:] = rng.standard_normal(arr[cut + 1:].shape)
        b2.timestamps[cut + 1:] += rng.integers(1, 10 ** 6, size=50 - cut - 1)
        r1 = oracle.fwd(b2)
        assert np.array_equal(r0["out"][:cut + 1], r1["out"][:cut + 1]), cut
        assert not np.array_equal(r0["out"][cut + 1:], r1["out"][cut + 1:])
    # candidate isolation: perturbing candidate m leaves every other row unchanged
    for m in range(E, 50):
        b3 = synth.make_batch(np.random.default_rng(31), [50], 2, 16, 16, "f32", contextuals=3,
                              targets=6, rel_bias_len=51, time_bias_len=64)
        for name in ("q", "k", "v", "u"):
            getattr(b3, name)[m] += 1.0
        r3 = oracle.fwd(b3)
        others = [i for i in range(50) if i != m]
        assert np.array_equal(r0["out"][others], r3["out"][others])


# ---------------------------------------------------------------- backward

def _loss(b, dout):
    return float((oracle.fwd(b)["out"] * dout).sum())


def _fd_check(b, dout, samples, h=1e-6, rtol=1e-6, seed=0):
    g = oracle.bwd(b, dout)
    rng = np.random.default_rng(seed)
    names = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("u", "du"), ("rel_bias", "drel"),
             ("time_bias", "dtb")]
    for name, gname in names:
        arr = getattr(b, name)
        if arr is None:
            continue
        flat = arr.reshape(-1)
        gflat = g[gname].reshape(-1)
        scale = np.abs(gflat).max()
        for idx in rng.choice(flat.size, size=min(samples, flat.size), replace=False):
            orig = float(flat[idx])
            arr64 = arr.astype(np.float64)
            setattr(b, name, arr64)
            f64 = arr64.reshape(-1)
            f64[idx] = orig + h
            lp = _loss(b, dout)
            f64[idx] = orig - h
            lm = _loss(b, dout)
            setattr(b, name, arr)
            num = (lp - lm) / (2 * h)
            assert abs(num - gflat[idx]) <= rtol * max(scale, 1e-30) + 1e-9, \
                (name, idx, num, gflat[idx])


def test_backward_finite_differences_full_mask_family():
    b = synth.make_batch(np.random.default_rng(41), [9, 17, 3], 2, 8, 8, "f32",
                         contextuals=[2, 3, 0], targets=[3, 2, 1], max_attn_len=4,
                         rel_bias_len=12, time_bias_len=32)
    dout = np.random.default_rng(42).standard_normal(b.u.shape)
    _fd_check(b, dout, samples=12)


def test_backward_finite_differences_tiny_workload_shapes():
    """Central differences on the tiny fp32 workload shapes (lengths 10, 100, 1000; H=2; d=32)."""
    b = synth.make_config(0)
    dout = np.random.default_rng(43).standard_normal(b.u.shape)
    _fd_check(b, dout, samples=3)


def test_mask_rows_is_the_mask_with_padding_invalid():
    """The row-range mask equals rows of the full mask, with every position past the end
    invalid (pinned through the full mask, itself pinned by the golden examples)."""
    for L, c, t, W in [(300, 4, 20, 50), (129, 32, 32, 0), (7, 0, 7, 0), (1, 1, 0, 3)]:
        full, _ = oracle.mask(L, c, t, W)
        pad = (L + 127) // 128 * 128
        for r0, n in [(0, L), (L // 2, pad - L // 2), (max(L - 3, 0), 10)]:
            m = oracle.mask_rows(L, c, t, W, r0, n, pad)
            rows_in = max(min(n, L - r0), 0)
            assert np.array_equal(m[:rows_in, :L], full[r0:r0 + rows_in])
            assert not m[rows_in:].any() and not m[:, L:].any()


@pytest.mark.parametrize("L,c,t,W", [(300, 4, 20, 50), (129, 32, 32, 0), (7, 0, 7, 0),
                                     (1, 1, 0, 3), (1000, 100, 200, 129), (513, 0, 0, 0),
                                     (700, 8, 128, 1024), (260, 1, 5, 1), (64, 0, 64, 0)])
def test_visited_tile_count_is_the_tiles_holding_a_valid_pair(L, c, t, W):
    """The accounting's tile count (used for the tile-skip efficiency) equals a brute-force
    count of the 128 x 128 tiles of the oracle mask that hold a valid pair."""
    m, _ = oracle.mask(L, c, t, W)
    nt = (L + 127) // 128
    brute = sum(1 for a in range(nt) for b in range(nt)
                if m[a * 128:(a + 1) * 128, b * 128:(b + 1) * 128].any())
    assert accounting.tiles_with_pairs_seq(L, c, t, W) == brute


# ---------------------------------------------------------------- mask variants (flags)

def test_mask_variant_hand_examples(golden_dir):
    """The two variants of the mask family against hand-derived masks; the dense
    formulation and the closed-form count agree."""
    lines = [ln.split("#")[0].strip() for ln in open(f"{golden_dir}/mask_examples_variants.txt")]
    lines = [ln for ln in lines if ln]
    i = 0
    while i < len(lines):
        _, L, c, t, W, f, n = lines[i].split()
        L, c, t, W, f, n = int(L), int(c), int(t), int(W), int(f), int(n)
        m = np.array([[int(ch) for ch in row] for row in lines[i + 1:i + 1 + L]], np.uint8)
        got, cnt = oracle.mask(L, c, t, W, f)
        assert np.array_equal(got, m), (L, c, t, W, f)
        assert cnt == n == int(m.sum())
        assert accounting.valid_pairs_seq(L, c, t, W, f) == n
        assert np.array_equal(dense._mask_dense(L, c, t, W, L, f).astype(np.uint8), m)
        i += 1 + L


@pytest.mark.parametrize("W", [0, 2, 7])
def test_mask_variant_counts_and_structure(W):
    """Contextual rows see every key before the candidates and nothing after; every other
    row keeps the default mask; counts follow the closed form."""
    for L in [1, 2, 9, 23]:
        for c in range(0, min(L, 4) + 1):
            for t in range(0, L - c + 1, max(1, (L - c) // 3 or 1)):
                base, _ = oracle.mask(L, c, t, W)
                m, cnt = oracle.mask(L, c, t, W, oracle.CTX_SEES_HISTORY)
                E = L - t
                assert m[:c, :E].all() and not m[:c, E:].any()
                assert np.array_equal(m[c:], base[c:])
                assert cnt == accounting.valid_pairs_seq(L, c, t, W, 1)
                assert np.array_equal(oracle.mask(L, c, t, W, oracle.REL_ABS)[0], base)


def test_rel_abs_indexes_bidirectional_pairs_by_distance():
    """Q = K = 0, one-hot rel table at r: contextual rows see later keys at p(j) - p(i) > 0.
    Default: that index clamps to 0.  With the |p(i) - p(j)| variant it is the distance."""
    silu1 = 1.0 / (1.0 + 1.0 / E_CONST)
    for flags in (oracle.REL_ABS, oracle.REL_ABS | oracle.CTX_SEES_HISTORY):
        for r in (1, 2):
            b = _empty_batch([6], 1, 16, 4, ctx=3, R=4)
            b.mask_flags = flags
            b.rel_bias[r] = 1.0
            b.v[:, 0, :] = np.random.default_rng(r).standard_normal((6, 4))
            y = oracle.fwd(b)["y"] * b.max_seqlen
            V = b.v[:, 0, :].astype(np.float64)
            see = 6 if flags & oracle.CTX_SEES_HISTORY else 3   # keys of the contextual rows
            for i in range(3):
                expect = sum(V[j] for j in range(see) if abs(i - j) == r)
                assert np.allclose(y[i], silu1 * expect if np.ndim(expect) else 0 * V[0],
                                   atol=1e-14), (flags, r, i)
            for i in range(3, 6):   # history rows: causal, the distance is i - j >= 0
                expect = sum(V[j] for j in range(0, i + 1) if i - j == r)
                assert np.allclose(y[i], silu1 * expect, atol=1e-14), (flags, r, i)


@pytest.mark.parametrize("flags", [1, 2, 3])
def test_mask_variants_jagged_equals_dense(flags):
    b = synth.make_batch(np.random.default_rng(60 + flags), [9, 30, 1, 14], 2, 8, 8, "f32",
                         contextuals=[2, 4, 0, 3], targets=[3, 5, 1, 0], max_attn_len=5,
                         rel_bias_len=12, time_bias_len=32, mask_flags=flags)
    a, d = oracle.fwd(b), dense.fwd(b)
    for key in ("out", "y", "mean", "rstd"):
        assert np.allclose(a[key], d[key], rtol=1e-12, atol=1e-12), key


@pytest.mark.parametrize("flags", [1, 2, 3])
def test_mask_variants_backward_finite_differences(flags):
    b = synth.make_batch(np.random.default_rng(70 + flags), [9, 17, 3], 2, 8, 8, "f32",
                         contextuals=[2, 3, 0], targets=[3, 2, 1], max_attn_len=4,
                         rel_bias_len=12, time_bias_len=32, mask_flags=flags)
    dout = np.random.default_rng(80 + flags).standard_normal(b.u.shape)
    _fd_check(b, dout, samples=8)


# ---------------------------------------------------------------- jagged operations

def _read_sl_golden(path):
    g = {}
    for ln in open(path):
        ln = ln.split("#")[0].strip()
        if ln:
            k, *v = ln.split()
            g[k] = v
    return g


def test_stochastic_length_hand_example(golden_dir):
    from oracle import jagged
    g = _read_sl_golden(f"{golden_dir}/stochastic_length_example.txt")
    lengths = [int(x) for x in g["lengths"]]
    offs = np.concatenate([[0], np.cumsum(lengths)])
    rows, new = jagged.stochastic_length(offs, [int(x) for x in g["contextuals"]],
                                         [int(x) for x in g["targets"]],
                                         [float(x) for x in g["keys"]], int(g["budget"][0]))
    assert rows.tolist() == [int(x) for x in g["rows"]]
    assert new.tolist() == [int(x) for x in g["offsets"]]


def test_stochastic_length_invariants():
    """Kept counts, order, what is always kept, and that the kept history keys are the
    smallest ones; a budget at least the history keeps everything."""
    from oracle import jagged
    rng = np.random.default_rng(5)
    L = rng.integers(0, 60, size=40)
    c = np.minimum(rng.integers(0, 4, size=40), L)
    t = np.minimum(rng.integers(0, 6, size=40), L - c)
    offs = np.concatenate([[0], np.cumsum(L)])
    keys = rng.integers(0, 8, size=int(offs[-1])) / 8.0          # many ties
    for budget in (0, 5, 17, 1000):
        rows, new = jagged.stochastic_length(offs, c, t, keys, budget)
        for b in range(40):
            a, e = offs[b], offs[b + 1]
            E = e - t[b]
            mine = rows[new[b]:new[b + 1]] - a
            assert np.all(np.diff(mine) > 0)                        # original order
            h = E - a - c[b]
            assert len(mine) == c[b] + t[b] + min(h, budget)
            assert set(range(c[b])) <= set(mine) and set(range(E - a, e - a)) <= set(mine)
            kept = [j for j in mine if c[b] <= j < E - a]
            dropped = [j for j in range(c[b], E - a) if j not in set(mine)]
            if kept and dropped:   # every kept (key, pos) precedes every dropped one
                assert max((keys[a + j], j) for j in kept) < min((keys[a + j], j) for j in dropped)
        if budget == 1000:
            assert rows.tolist() == list(range(int(offs[-1])))


def test_jagged_concat_and_gather_examples():
    from oracle import jagged
    a = np.arange(6).reshape(3, 2); oa = np.array([0, 1, 1, 3])
    b = 10 + np.arange(8).reshape(4, 2); ob = np.array([0, 2, 3, 4])
    v, o = jagged.jagged_concat([(a, oa), (b, ob)])
    assert o.tolist() == [0, 3, 4, 7]
    assert v[:, 0].tolist() == [0, 10, 12, 14, 2, 4, 16]
    g = jagged.gather_rows(b, [3, 0, 0])
    assert g[:, 0].tolist() == [16, 10, 10]


def test_candidate_outputs_do_not_depend_on_the_other_candidates():
    """The property M-FALCON rests on ("Scaling HSTU", "Many candidates make reuse valuable"):
    under target-group masking a candidate's output, computed with the history plus only
    some of the candidates (same N), equals its output in the full batch, and the history
    rows equal those of the history alone.  Exact in fp64: the same terms in the same order."""
    import dataclasses
    rng = np.random.default_rng(31)
    H, d = 2, 8
    hist_len = [12, 30, 5]
    ncand = [7, 3, 4]
    full = synth.make_batch(rng, [h + c for h, c in zip(hist_len, ncand)], H, d, d, "f32",
                            contextuals=[2, 3, 1], targets=ncand, max_attn_len=6,
                            rel_bias_len=40, time_bias_len=32)
    ref = oracle.fwd(full)
    N = full.max_seqlen
    offs = full.seq_offsets

    def sub(keep_cands):
        rows, lens, tg = [], [], []
        for s in range(3):
            a = offs[s]
            rows += list(range(a, a + hist_len[s]))
            sel = [a + hist_len[s] + j for j in keep_cands[s]]
            rows += sel
            lens.append(hist_len[s] + len(sel))
            tg.append(len(sel))
        rows = np.array(rows)
        o = np.concatenate([[0], np.cumsum(lens)])
        return rows, dataclasses.replace(
            full, seq_offsets=o, num_targets=np.array(tg, np.int32), q=full.q[rows],
            k=full.k[rows], v=full.v[rows], u=full.u[rows], timestamps=full.timestamps[rows],
            max_seqlen=N)

    for keep in ([[], [], []], [[0, 2], [1], [3]], [[6], [0, 1, 2], []]):
        rows, b = sub(keep)
        got = oracle.fwd(b)["out"]
        assert np.array_equal(got, ref["out"][rows])


# ---------------------------------------------------------------- the layer around the path

def test_fused_projection_splits_into_four_projections():
    """One projection with columns U | V | Q | K (head-major) equals four separate
    projections, with d_qk != d_v; the SiLU variant applies to every branch."""
    from oracle import layer
    rng = np.random.default_rng(7)
    T, dm, H, dqk, dv = 9, 16, 3, 4, 6
    x = rng.standard_normal((T, dm))
    Wu, Wv = rng.standard_normal((dm, H * dv)), rng.standard_normal((dm, H * dv))
    Wq, Wk = rng.standard_normal((dm, H * dqk)), rng.standard_normal((dm, H * dqk))
    bu, bv, bq, bk = (rng.standard_normal(w.shape[1]) for w in (Wu, Wv, Wq, Wk))
    W = np.concatenate([Wu, Wv, Wq, Wk], axis=1)
    bias = np.concatenate([bu, bv, bq, bk])
    silu = lambda a: a / (1 + np.exp(-a))
    for act, f in ((False, lambda a: a), (True, silu)):
        u, v, q, k = layer.uvqk(x, W, bias, H, dqk, dv, silu=act)
        assert np.allclose(u, f(x @ Wu + bu))
        assert np.allclose(v[:, 2, :], f(x @ Wv + bv)[:, 2 * dv:3 * dv])
        assert np.allclose(q[:, 1, :], f(x @ Wq + bq)[:, dqk:2 * dqk])
        assert np.allclose(k.reshape(T, -1), f(x @ Wk + bk))


def test_layer_output_projection_and_residual():
    """W_o = 0 and no bias: the layer returns its input (the residual).  W_o the identity
    (d_model = H * d_v), no residual: it returns the attention output."""
    from oracle import layer
    b = synth.make_batch(np.random.default_rng(8), [7, 12], 2, 4, 4, "f32", contextuals=1,
                         targets=[2, 3], rel_bias_len=13, time_bias_len=16)
    dm = 8
    rng = np.random.default_rng(9)
    x = rng.standard_normal((b.total_tokens, dm))
    W = rng.standard_normal((dm, 2 * 2 * 4 + 2 * 2 * 4)) * 0.3
    r0 = layer.layer_fwd(b, x, W, None, np.zeros((dm, dm)), None)
    assert np.array_equal(r0["o"], x)
    r1 = layer.out_proj(r0["attn"], np.eye(dm), None, None)
    assert np.allclose(r1, r0["attn"])
    # the input normalisation: mean 0 and variance var/(var + eps) per token
    xn = layer.layer_norm(x, 1e-5)
    assert np.allclose(xn.mean(1), 0, atol=1e-12)
    v = x.var(1)
    assert np.allclose(xn.var(1), v / (v + 1e-5))
