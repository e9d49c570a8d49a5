"""Shared test helpers: tolerances and row selection (data handling only)."""
import os

import numpy as np

from jagged_hstu_attention_02_b200.synth import sub_batch  # noqa: F401

# max|err| <= 1e-2 * max|ref| + 1e-3 for bf16 inputs; <= 1e-5 * max|ref| for fp32 inputs
TOL = {"bf16": (1e-2, 1e-3), "f32": (1e-5, 0.0)}


def max_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0, 0.0
    return float(np.abs(got - ref).max()), float(np.abs(ref).max())


def assert_close(got, ref, dtype, what=""):
    err, scale = max_err(got, ref)
    rel, ab = TOL[dtype]
    tol = rel * scale + ab
    log = os.environ.get("HSTU_PARITY_LOG")
    if log:   # margin record: what, max|err|, tolerance, their ratio
        with open(log, "a") as f:
            f.write("%s\t%.4e\t%.4e\t%.4f\n" % (what, err, tol, err / tol if tol else 0.0))
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), what + ": non-finite values"
    assert err <= tol, "%s: max|err| %.3e > tol %.3e (max|ref| %.3e)" % (what, err, tol, scale)
    return err, scale


def rows_of(b, seqs):
    offs = b.seq_offsets
    return np.concatenate([np.arange(offs[s], offs[s + 1]) for s in seqs])
