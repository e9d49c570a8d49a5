"""Sharding a jagged batch by whole sequences across ranks (CPU, gloo).

The plan must cover every sequence exactly once and balance the pair work; a rank's slice
must equal the sequences it owns; and a two-rank backward (each rank on its own slice,
with the global N) followed by the one all-reduce of the bias-table gradients must give
the full batch's gradients: per-token gradients on the owning rank, table gradients on
every rank.  The per-rank compute here is the fp64 oracle (no GPU on this host); the
library kernels take the same slices.
"""
import dataclasses
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from jagged_hstu_attention_02_b200 import accounting, shard, synth


def _batch():
    rng = np.random.default_rng(77)
    lengths = [12, 40, 7, 33, 25, 3, 18, 29]
    return synth.make_batch(rng, lengths, 2, 8, 8, "f32", contextuals=[1, 3, 0, 2, 4, 0, 1, 2],
                            targets=[2, 5, 1, 0, 6, 1, 3, 4], max_attn_len=16,
                            rel_bias_len=30, time_bias_len=32, with_dout=True)


def _local(b, seqs):
    d = shard.shard(dataclasses.asdict(b), seqs)
    return dataclasses.replace(b, **{k: d[k] for k in ("seq_offsets", "num_contextuals",
                                                        "num_targets", "q", "k", "v", "u",
                                                        "timestamps", "dout")})


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_plan_covers_every_sequence_once_and_balances_pairs(world):
    rng = np.random.default_rng(world)
    lengths = rng.integers(1, 300, size=41)
    offs = np.concatenate([[0], np.cumsum(lengths)])
    ctx = rng.integers(0, 3, size=41)
    tgt = np.minimum(rng.integers(0, 10, size=41), lengths - ctx)
    parts = shard.plan(offs, world, ctx, tgt, max_attn_len=64)
    assert len(parts) == world
    flat = np.sort(np.concatenate(parts))
    assert np.array_equal(flat, np.arange(41))
    work = shard.sequence_work(offs, ctx, tgt, 64)
    loads = np.array([work[p].sum() for p in parts])
    # longest-processing-time bound: no rank exceeds the mean by more than one sequence
    assert loads.max() <= work.sum() / world + work.max()
    for b in range(41):
        assert work[b] == accounting.valid_pairs_seq(int(lengths[b]), int(ctx[b]),
                                                     int(tgt[b]), 64)


def test_shard_slices_match_sub_batches():
    b = _batch()
    for seqs in ([0, 3, 5], [1], [2, 4, 6, 7], []):
        loc = _local(b, seqs)
        ref = synth.sub_batch(b, seqs)
        for key in ("seq_offsets", "num_contextuals", "num_targets", "q", "k", "v", "u",
                    "timestamps", "dout"):
            assert np.array_equal(getattr(loc, key), getattr(ref, key)), key


def test_shard_works_on_torch_tensors():
    b = _batch()
    t = {k: (torch.from_numpy(v) if isinstance(v, np.ndarray) else v)
         for k, v in dataclasses.asdict(b).items()}
    d = shard.shard(t, [4, 1])
    ref = synth.sub_batch(b, [4, 1])
    assert torch.equal(d["q"], torch.from_numpy(ref.q))
    assert torch.equal(d["seq_offsets"], torch.from_numpy(ref.seq_offsets))
    assert torch.equal(d["num_targets"], torch.from_numpy(ref.num_targets))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    import torch.distributed as dist
    from oracle import oracle

    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        b = _batch()
        parts = shard.plan(b.seq_offsets, world, b.num_contextuals, b.num_targets,
                           b.max_attn_len)
        loc = _local(b, parts[rank])
        g = oracle.bwd(loc)
        drel = torch.from_numpy(g["drel"].copy())
        dtb = torch.from_numpy(g["dtb"].copy())
        shard.allreduce_table_grads(drel, dtb)
        np.savez(os.path.join(outdir, "rank%d.npz" % rank), seqs=parts[rank], dq=g["dq"],
                 dk=g["dk"], dv=g["dv"], du=g["du"], drel=drel.numpy(), dtb=dtb.numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_backward_with_table_allreduce_matches_full_batch(tmp_path):
    from oracle import oracle

    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    b = _batch()
    full = oracle.bwd(b)
    scale_rel = np.abs(full["drel"]).max()
    scale_tb = np.abs(full["dtb"]).max()
    owned = []
    for r in range(world):
        d = np.load(os.path.join(tmp_path, "rank%d.npz" % r))
        rows, _ = shard.local_rows(b.seq_offsets, d["seqs"])
        owned.append(rows)
        for key in ("dq", "dk", "dv", "du"):
            np.testing.assert_allclose(d[key], full[key][rows], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(d["drel"], full["drel"], rtol=0, atol=1e-12 * scale_rel)
        np.testing.assert_allclose(d["dtb"], full["dtb"], rtol=0, atol=1e-12 * scale_tb)
    assert np.array_equal(np.sort(np.concatenate(owned)), np.arange(b.total_tokens))
