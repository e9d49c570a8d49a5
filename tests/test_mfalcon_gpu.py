"""Candidate micro-batching with a cached history (M-FALCON) on the GPU: the history runs
once, the candidates in micro-batches appended to it with only their query tiles computed;
every output must match the oracle's full batch ("Scaling HSTU: ragged execution, candidate
amortization and content features", "Many candidates make reuse valuable")."""
import numpy as np
import pytest
import torch

from jagged_hstu_attention_02_b200 import mfalcon, ops, synth
from oracle import oracle
from tests.helpers import assert_close

pytestmark = pytest.mark.gpu


def _split(b):
    """The history (contextual + history tokens) and candidate parts of a batch."""
    offs = b.seq_offsets
    t = b.num_targets
    hrows, crows, hl, cl = [], [], [], []
    for s in range(b.batch):
        E = offs[s + 1] - t[s]
        hrows += list(range(offs[s], E))
        crows += list(range(E, offs[s + 1]))
        hl.append(E - offs[s])
        cl.append(t[s])
    hrows, crows = np.array(hrows, np.int64), np.array(crows, np.int64)
    d = lambda a, dt=None: torch.from_numpy(np.ascontiguousarray(a if dt is None else a.astype(dt))).cuda()
    tdt = torch.bfloat16 if b.dtype == "bf16" else torch.float32
    cast = lambda a: d(a).to(tdt)
    hist = dict(q=cast(b.q[hrows]), k=cast(b.k[hrows]), v=cast(b.v[hrows]), u=cast(b.u[hrows]),
                timestamps=d(b.timestamps[hrows]) if b.timestamps is not None else None,
                seq_offsets=d(np.concatenate([[0], np.cumsum(hl)]), np.int64),
                num_contextuals=d(b.num_contextuals, np.int32))
    cand = dict(q=cast(b.q[crows]), k=cast(b.k[crows]), v=cast(b.v[crows]), u=cast(b.u[crows]),
                seq_offsets=d(np.concatenate([[0], np.cumsum(cl)]), np.int64))
    return hist, cand, hrows, crows


@pytest.mark.parametrize("micro_batch", [1, 7, 64])
@pytest.mark.parametrize("dims", [(128, 128, "bf16"), (64, 64, "bf16"), (32, 32, "f32")])
def test_mfalcon_matches_the_full_batch(micro_batch, dims):
    dqk, dv, dtype = dims
    rng = np.random.default_rng(500 + micro_batch)
    B = 12
    hist = rng.integers(8, 260, size=B)
    tg = rng.integers(1, 40, size=B)
    tg[0] = 33 if micro_batch == 1 else tg[0]     # > 16 micro-batches: concat chaining
    b = synth.make_batch(rng, 1 + hist + tg, 2, dqk, dv, dtype, contextuals=1, targets=tg,
                         rel_bias_len=int((1 + hist + tg).max()) + 1, time_bias_len=128,
                         max_attn_len=0)
    h, c, hrows, crows = _split(b)
    out_h, out_c = mfalcon.mfalcon_fwd(
        h, c, micro_batch=micro_batch, max_seqlen=b.max_seqlen, alpha=b.alpha,
        rel_bias=torch.from_numpy(b.rel_bias).cuda(), time_bias=torch.from_numpy(b.time_bias).cuda())
    torch.cuda.synchronize()
    ref = oracle.fwd(b)["out"]
    assert_close(out_h.float().cpu().numpy(), ref[hrows], dtype, "history rows")
    assert_close(out_c.float().cpu().numpy(), ref[crows], dtype, "candidate rows")


def test_candidates_only_flag_is_forward_inference_only():
    b = synth.make_batch(np.random.default_rng(1), [40], 1, 64, 64, "bf16", targets=5,
                         rel_bias_len=41, with_dout=True)
    dev = ops.batch_to_device(b)
    with pytest.raises(ops.HstuError):
        ops.run_fwd(b, dev, training=True, mask_flags=ops.FLAG_CANDIDATES_ONLY)
    out, saved = ops.run_fwd(b, dev, training=True)
    with pytest.raises(ops.HstuError):
        ops.run_bwd(b, saved, dev_tensors=dev, mask_flags=ops.FLAG_CANDIDATES_ONLY)
