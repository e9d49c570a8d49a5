"""Jagged operations on the GPU against the oracle: Stochastic Length selection (bit-exact:
it is index work), row gathering and per-sequence concatenation, and a Stochastic-Length
batch fed through the attention kernels ("Scaling HSTU: ragged execution, candidate
amortization and content features", "Variable length is a central systems issue";
"HSTU-MUSA: HSTU for Moore Threads (MUSA)", "Project Structure")."""
import numpy as np
import pytest
import torch

from jagged_hstu_attention_02_b200 import ops, synth
from oracle import jagged as ojag
from oracle import oracle
from tests.helpers import assert_close

pytestmark = pytest.mark.gpu


def _batch(rng, B, maxlen):
    L = rng.integers(0, maxlen, size=B)
    L[:4] = [0, 1, 7, maxlen]
    c = np.minimum(rng.integers(0, 5, size=B), L)
    t = np.minimum(rng.integers(0, 9, size=B), L - c)
    c[5], t[5] = 0, L[5]              # all candidates
    c[6], t[6] = L[6], 0              # all contextual
    offs = np.concatenate([[0], np.cumsum(L)]).astype(np.int64)
    return L, c.astype(np.int32), t.astype(np.int32), offs


@pytest.mark.parametrize("budget", [0, 5, 100, 1 << 30])
def test_stochastic_length_matches_oracle_bit_exact(budget):
    rng = np.random.default_rng(budget % 997)
    L, c, t, offs = _batch(rng, 300, 400)
    T = int(offs[-1])
    keys = (rng.integers(0, 64, size=T) / 64.0).astype(np.float32)   # ties on purpose
    keys[::7] = -keys[::7]                                          # negative keys too
    d = lambda a: torch.from_numpy(a).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rows, new = ops.stochastic_length(d(offs), d(c), d(t), d(keys), budget, status=status)
    ref_rows, ref_new = ojag.stochastic_length(offs, c, t, keys, budget)
    assert new.cpu().numpy().tolist() == ref_new.tolist()
    n = int(ref_new[-1])
    assert rows[:n].cpu().numpy().tolist() == ref_rows.tolist()
    assert int(status.item()) == 0


def test_stochastic_length_long_sequence_and_bad_counts():
    rng = np.random.default_rng(3)
    L = np.array([20000, 50, 40], np.int64)
    c = np.array([3, 2, 1], np.int32)
    t = np.array([30, 100, 2], np.int32)          # sequence 1: c + t > L
    offs = np.concatenate([[0], np.cumsum(L)])
    keys = rng.random(int(offs[-1])).astype(np.float32)
    d = lambda a: torch.from_numpy(a).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rows, new = ops.stochastic_length(d(offs), d(c), d(t), d(keys), 1000, status=status)
    assert int(status.item()) & ops.DEV_BAD_COUNTS
    ok = [0, 2]
    ref_rows, ref_new = ojag.stochastic_length(offs[[0, 1]], c[:1], t[:1], keys, 1000)
    got = new.cpu().numpy()
    assert got[1] - got[0] == 3 + 30 + 1000 and got[2] == got[1]   # bad sequence keeps nothing
    assert rows[:got[1]].cpu().numpy().tolist() == ref_rows.tolist()
    del ok


def test_gather_rows_and_jagged_concat():
    rng = np.random.default_rng(11)
    B = 50
    parts = []
    for q, (lo, hi, w) in enumerate([(0, 3, 24), (0, 300, 24), (1, 21, 24)]):
        L = rng.integers(lo, hi, size=B)
        offs = np.concatenate([[0], np.cumsum(L)]).astype(np.int64)
        vals = rng.standard_normal((int(offs[-1]), w)).astype(np.float32)
        parts.append((vals, offs))
    tparts = [(torch.from_numpy(v).cuda(), torch.from_numpy(o).cuda()) for v, o in parts]
    got, got_offs = ops.jagged_concat(tparts)
    ref, ref_offs = ojag.jagged_concat(parts)
    assert got_offs.cpu().numpy().tolist() == ref_offs.tolist()
    assert np.array_equal(got.cpu().numpy(), ref)
    # bf16 rows of 6 bytes (no 16-byte vectors) and fp32 rows of 96 bytes
    src = torch.randn(1000, 3, device="cuda").to(torch.bfloat16)
    idx = torch.from_numpy(rng.integers(0, 1000, size=700)).cuda()
    n = torch.tensor([650], dtype=torch.int64, device="cuda")
    out = ops.gather_rows(src, idx, n, 700)
    assert torch.equal(out[:650], src[idx[:650]])
    src2 = torch.from_numpy(parts[1][0]).cuda()
    idx2 = torch.from_numpy(rng.integers(0, src2.shape[0], size=500)).cuda()
    out2 = ops.gather_rows(src2, idx2, torch.tensor([500], device="cuda"), 500)
    assert torch.equal(out2, src2[idx2])


def test_stochastic_length_batch_through_the_attention():
    """Training with Stochastic Length: the sampled batch (rows gathered on the GPU) runs
    through the forward and backward kernels and matches the oracle on the same sample."""
    b = synth.make_batch(np.random.default_rng(21), [300, 90, 700, 5], 2, 64, 64, "bf16",
                         contextuals=[2, 1, 4, 0], targets=[10, 3, 20, 1], rel_bias_len=701,
                         time_bias_len=128, with_dout=True)
    dev = ops.batch_to_device(b)
    keys = torch.from_numpy(np.random.default_rng(22).random(b.total_tokens).astype(np.float32)).cuda()
    rows, new = ops.stochastic_length(dev["seq_offsets"], dev["num_contextuals"],
                                      dev["num_targets"], keys, 128)
    n = new[-1:]
    T2 = int(n.item())
    sampled = dict(dev)
    for key in ("q", "k", "v", "u", "timestamps", "dout"):
        sampled[key] = ops.gather_rows(dev[key], rows, n, T2)
    sampled["seq_offsets"] = new
    rr = rows[:T2].cpu().numpy()
    import dataclasses
    sb = dataclasses.replace(b, seq_offsets=new.cpu().numpy(), q=b.q[rr], k=b.k[rr], v=b.v[rr],
                             u=b.u[rr], timestamps=b.timestamps[rr], dout=b.dout[rr])
    out, saved = ops.run_fwd(sb, sampled, training=True)
    g = ops.run_bwd(sb, saved, dev_tensors=sampled)
    torch.cuda.synchronize()
    assert ops.read_device_status(ops.fwd.last_workspace) == 0
    ref_f = oracle.fwd(sb)
    ref_b = oracle.bwd(sb)
    assert_close(out.float().cpu().numpy(), ref_f["out"], "bf16", "sampled out")
    for got, key in zip(g, ["dq", "dk", "dv", "du", "drel", "dtb"]):
        assert_close(got.float().cpu().numpy(), ref_b[key], "bf16", "sampled " + key)
