"""Benchmark of jagged HSTU attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline: the training step on the MovieLens-shaped workload (B=128 per GPU, H=4, d=128,
bf16, Zipf history + 1 contextual + 1..20 candidate tokens, time and rel-pos bias,
dO ~ N(0,1)): forward with saved activations, then backward.  One step = one pass of the
whole path over one batch.  Throughput counts valid (unmasked) pairs only:
fwd P*H*2*(d_qk+d_v) + bwd P*H*2*(2d_qk+2d_v).

Under torchrun the global batch holds N*128 sequences; shard.plan deals them to the ranks
by longest-processing-time on their pair work, every rank runs with the global max_seqlen,
and the bias-table gradients are summed with one all-reduce per step ("scaling": "weak":
the work per GPU stays fixed as N grows).  Timing is the max over ranks.

On one GPU the line also carries one block per inference-forward workload (long history,
windowed, MovieLens-shaped), each timed over >= 50 L2-flushed calls with its own roofline,
clocks and CPU baseline.  Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from jagged_hstu_attention_02_b200 import accounting, synth  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
WORKLOAD_CFG = 4          # MovieLens-shaped inputs + upstream gradient
METRIC = "jagged HSTU attn fwd+bwd TFLOP/s (valid pairs) on 1 B200"
# inference-forward blocks: workload -> (block name, roofline that bounds its attention kernel)
FWD_BLOCKS = {2: ("long_history_fwd", "tensor"), 3: ("windowed_fwd", "tensor"),
              1: ("movielens_fwd", "hbm")}


# DRAM traffic per launch of a kernel, from an ncu capture summarised under profiles/; used
# only while the kernel's sources hash to the value recorded with the capture.
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
KERNEL_SOURCES = {
    "bwd_attn": ["bwd_sm100.cu", "bias.cuh", "common.cuh", "sm100.cuh", "tiles.cuh",
                 "units.cuh"],
    "fwd_attn": ["fwd_sm100.cu", "bias.cuh", "common.cuh", "sm100.cuh", "tiles.cuh",
                 "units.cuh"],
}


def sources_sha(stage):
    """Hash of a stage's kernel sources with comments and blank lines left out, so that an
    edit of the comments alone keeps a recorded capture valid."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(stage, []):
        with open(os.path.join(ROOT, "jagged_hstu_attention_02_b200", "csrc", f)) as fh:
            for line in fh:
                code = re.sub(r"//.*$", "", line).rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def recorded_traffic(stage, workload):
    """(bytes per launch, note) when profiles/traffic.json holds a capture of this stage's
    kernel on this workload whose sources match the current ones, else (None, why)."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, "no capture recorded"
    with open(TRAFFIC_FILE) as f:
        rec = json.load(f).get("%s@%d" % (stage, workload))
    if not rec:
        return None, "no capture of this workload"
    if rec.get("sources_sha") != sources_sha(stage):
        return None, "kernel changed since the capture"
    return rec["bytes_per_launch"], rec.get("capture", "")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons polled through NVML every few ms while
    the timed region runs (read-only queries)."""
    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, gpu_index, period_s=0.002):
        self.gpu = gpu_index
        self.bus_id = None
        try:
            import torch
            pr = torch.cuda.get_device_properties(gpu_index)
            self.bus_id = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
        except Exception:
            pass
        self.period = period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.err = None

    def _run(self):
        import pynvml
        try:
            pynvml.nvmlInit()
            hd = (pynvml.nvmlDeviceGetHandleByPciBusId(self.bus_id) if self.bus_id
                  else pynvml.nvmlDeviceGetHandleByIndex(self.gpu))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(hd, pynvml.NVML_CLOCK_SM)
            masks = {k: getattr(pynvml, v, 0) for k, v in self.REASONS.items()}
            while not self.stop_flag.is_set():
                self.samples.append(pynvml.nvmlDeviceGetClockInfo(hd, pynvml.NVML_CLOCK_SM))
                r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(hd)
                for k, m in masks.items():
                    if m and (r & m):
                        self.reasons.add(k)
                time.sleep(self.period)
            pynvml.nvmlShutdown()
        except Exception as e:  # NVML unavailable: report it instead of clocks
            self.err = repr(e)

    def start(self):
        import threading
        self.stop_flag = threading.Event()
        self.th = threading.Thread(target=self._run, daemon=True)
        self.th.start()
        time.sleep(0.02)

    def stop(self):
        self.stop_flag.set()
        self.th.join(timeout=5)
        if self.err or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz,
                    "reasons": ["nvml unavailable: %s" % self.err] if self.err else [],
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def stage_timer(ops, torch, stages):
    """Per-stage CUDA events recorded by the library around its kernels."""
    evs = {}
    for st in stages:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        b.record()
        ops.set_stage_events(st, a, b)
        evs[st] = (a, b)
    return evs


def headline_batch(world, rank):
    """This rank's share of the global training batch: N*128 MovieLens-shaped sequences dealt
    by shard.plan, all with the global max_seqlen (and rel table of N+1 entries)."""
    from jagged_hstu_attention_02_b200 import shard

    g = synth.make_config(WORKLOAD_CFG, batch=128 * world)
    if world == 1:
        return g, g
    seqs = shard.plan(g.seq_offsets, world, g.num_contextuals, g.num_targets,
                      g.max_attn_len)[rank]
    return synth.sub_batch(g, seqs), g


def run_ours(args, world, rank, local):
    import torch
    from jagged_hstu_attention_02_b200 import ops

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    peaks, peak_kind = load_peaks()

    b, gb = headline_batch(world, rank)
    P = accounting.valid_pairs(b)
    flops = accounting.fwd_flops(b, P) + accounting.bwd_flops(b, P)
    P_all = accounting.valid_pairs(gb)
    flops_all = accounting.fwd_flops(gb, P_all) + accounting.bwd_flops(gb, P_all)
    tokens = b.total_tokens
    dev = ops.batch_to_device(b)
    kw = ops.batch_kwargs(b)
    out, saved = ops.run_fwd(b, dev, training=True)
    # the bias-table gradients live in one buffer: a sharded step sums them across ranks
    # with one all-reduce (jagged_hstu_attention_02_b200.shard), the only exchange it has
    R, NB = b.rel_bias_len, b.time_bias_len
    table_grads = torch.zeros(R + NB, dtype=torch.float32, device="cuda")
    grads = (torch.empty_like(dev["q"]), torch.empty_like(dev["k"]), torch.empty_like(dev["v"]),
             torch.empty_like(dev["u"]), table_grads[:R], table_grads[R:])
    ops.run_bwd(b, saved, dev_tensors=dev, grads=grads)
    ws_f = ops.fwd.last_workspace
    ws_b = ops.bwd.last_workspace
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    def step(collective=True):
        ops.fwd(dev["q"], dev["k"], dev["v"], dev["u"], dev["seq_offsets"],
                dev["num_contextuals"], dev["num_targets"], dev["timestamps"], dev["rel_bias"],
                dev["time_bias"], training=True, out=out, saved=saved, workspace=ws_f, **kw)
        ops.bwd(dev["dout"], dev["q"], dev["k"], dev["v"], dev["u"], dev["seq_offsets"],
                dev["num_contextuals"], dev["num_targets"], dev["timestamps"], dev["rel_bias"],
                dev["time_bias"], saved=saved, grads=grads, workspace=ws_b, **kw)
        if world > 1 and collective:
            torch.distributed.all_reduce(table_grads)

    stages = ["fwd_attn", "fwd_norm", "bwd_norm", "bwd_attn"]
    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    # per-stage times of eager steps (events between every kernel, so each includes its
    # launch gap); they pick the dominant kernel, the one timed inside the measured steps
    evs = stage_timer(ops, torch, stages)
    stage_ms = {s: [] for s in stages}
    for _ in range(max(3, args.warmup)):
        flush.fill_(1.0)
        step()
        torch.cuda.synchronize()
        for s in stages:
            stage_ms[s].append(evs[s][0].elapsed_time(evs[s][1]))
    for s in stages:
        ops.set_stage_events(s)
    avg = {s: sum(v) / len(v) for s, v in stage_ms.items()}
    dom = max(avg, key=avg.get)
    if world > 1:   # every rank times the same stage (the graph below depends on it)
        t = torch.tensor([stages.index(dom)], device="cuda")
        torch.distributed.broadcast(t, 0)
        dom = stages[int(t.item())]

    # the measured steps replay one CUDA graph of the step's library calls (the table-grad
    # all-reduce of a sharded step stays outside it), with no events between its kernels:
    # an event would hold back the kernel behind it, which otherwise starts its set-up while
    # the kernel ahead finishes
    def capture():
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            with torch.cuda.graph(g, stream=cap):
                step(collective=False)
        torch.cuda.current_stream().wait_stream(cap)
        torch.cuda.synchronize()
        return g

    graph = capture()
    for _ in range(args.warmup):
        flush.fill_(1.0)
        graph.replay()
        if world > 1:
            torch.distributed.all_reduce(table_grads)
    torch.cuda.synchronize()

    step_ms = []
    clocks = ClockSampler(local)
    clocks.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_region = time.perf_counter()
    for _ in range(args.steps):
        flush.fill_(1.0)                       # evict the previous step's data from L2
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        if world > 1:
            torch.distributed.all_reduce(table_grads)
        e1.record()
        e1.synchronize()
        step_ms.append(e0.elapsed_time(e1))
    torch.cuda.synchronize()
    wall_region = time.perf_counter() - t_region
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    del graph

    # the dominant kernel's own time: the same graph with its two events recorded inside,
    # replayed as many times again
    dom_ev = stage_timer(ops, torch, [dom])[dom]
    graph = capture()
    ops.set_stage_events(dom)
    dom_ms = []
    for _ in range(args.steps):
        flush.fill_(1.0)
        graph.replay()
        if world > 1:
            torch.distributed.all_reduce(table_grads)
        torch.cuda.synchronize()
        dom_ms.append(dom_ev[0].elapsed_time(dom_ev[1]))
    del graph
    assert ops.read_device_status(ws_f) == 0 and ops.read_device_status(ws_b) == 0

    ms = sum(step_ms) / len(step_ms)
    if world > 1:
        t = torch.tensor([ms], device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    value = flops_all / (ms * 1e-3) / 1e12

    # roofline of the dominant kernel stage, timed inside the measured steps, on its own
    # algorithmic bytes and FLOPs
    avg[dom] = sum(dom_ms) / len(dom_ms)
    roofline = kernel_roofline(b, dom, avg[dom], P, peaks, peak_kind, WORKLOAD_CFG,
                               training=True)
    roofline["stage_ms"] = {s: round(v, 4) for s, v in avg.items()}
    roofline["stage_ms_note"] = ("kernel_ms from replays of the step graph with the kernel's "
                                 "two events inside; the other stages from eager steps with "
                                 "events between all kernels")

    # end to end through the public API with host buffers (pinned), copies inside the region
    e2e = measure_e2e(args, b, ops, torch, kw, flops, world, flops_all)

    blocks = {}
    if world == 1 and not args.quick:
        for cfg in FWD_BLOCKS:
            blocks[FWD_BLOCKS[cfg][0]] = measure_fwd_block(ops, torch, peaks, peak_kind, cfg,
                                                           args, with_cpu=not args.no_cpu)
        blocks["layer_projections"] = measure_layer_block(ops, torch, peaks, peak_kind, args)
    cpu = cpu_baseline_train(b) if (rank == 0 and world == 1 and not args.no_cpu) else None
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC,
        "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "tokens_per_s": round(gb.total_tokens / (ms * 1e-3), 1),
        "pct_bf16_peak": round(100 * value / world / peaks["bf16_tflops"], 3),
        "config": {"workload": synth.WORKLOADS[WORKLOAD_CFG], "global_batch": gb.batch,
                   "tokens_per_gpu": tokens, "tokens_global": gb.total_tokens,
                   "valid_pairs_global": P_all, "flops_per_step_global": flops_all,
                   "max_seqlen": gb.max_seqlen, "parallelism": "dp%d" % world,
                   "sharding": "shard.plan (LPT on valid pairs) over the global batch" if world > 1
                   else "one GPU, whole batch",
                   "l2": "flushed between steps (256 MB write), flush outside per-step events",
                   "launch": "each step replays one CUDA graph of its fwd and bwd library calls",
                   "wall_s_region": round(wall_region, 3)},
        "roofline": roofline, "e2e": e2e, "clocks": clk,
        "gpu_launches": args.steps * LAUNCHES_PER_STEP,
        "cpu_baseline": cpu, "workloads": blocks,
    }
    print(json.dumps(line), flush=True)


# kernels of ours launched per step: fwd attention, fwd LayerNorm+gating, bwd LayerNorm+gating,
# bwd attention, dQ conversion (memsets are not kernels of ours)
LAUNCHES_PER_STEP = 5
LAUNCHES_PER_FWD = 2


def kernel_roofline(b, stage, kms, P, peaks, peak_kind, workload, training, bound=None):
    """Roofline of one kernel stage from its own algorithmic bytes and valid-pair FLOPs:
    HBM-bound unless its arithmetic intensity is above the ridge point (or `bound` says)."""
    byts = {"fwd_attn": accounting.fwd_attn_bytes(b, training=training),
            "fwd_norm": accounting.fwd_norm_bytes(b, training=training),
            "bwd_norm": accounting.bwd_norm_bytes(b),
            "bwd_attn": accounting.bwd_attn_bytes(b)}[stage]
    fl = {"fwd_attn": accounting.fwd_flops(b, P), "bwd_attn": accounting.bwd_flops(b, P)}.get(
        stage, 0)
    gbs = byts / (kms * 1e-3) / 1e9
    tfs = fl / (kms * 1e-3) / 1e12
    hbm, tc = peaks["hbm_gbs"], peaks["bf16_tflops"]
    ridge = tc * 1e12 / (hbm * 1e9)
    if bound is None:
        bound = "tensor" if fl and fl / byts > ridge else "hbm"
    traffic, traffic_note = recorded_traffic(stage, workload)
    r = {"bound": bound}
    if bound == "tensor":
        r.update(achieved=round(tfs, 2), peak=tc, unit="TFLOP/s", frac=round(tfs / tc, 4),
                 peak_note="bf16_tflops (burst: the kernel is timed alone)")
    else:
        r.update(achieved=round(gbs, 1), peak=hbm, unit="GB/s", frac=round(gbs / hbm, 4))
    r.update(traffic=traffic, traffic_note=traffic_note, algorithmic_bytes=byts,
             algorithmic_flops=fl, kernel_stage=stage, kernel_ms=round(kms, 4),
             peak_source=peak_kind, hbm_frac=round(gbs / hbm, 4),
             tensor_frac=round(tfs / tc, 4) if fl else None,
             intensity_flop_per_byte=round(fl / byts, 2), ridge_flop_per_byte=round(ridge, 1))
    return r


def measure_e2e(args, b, ops, torch, kw, flops, world, flops_all):
    """Training steps through the public API with every step's inputs copied in from pinned
    host memory and its results (O, dQ, dK, dV, dU, table gradients) read back.  As a
    training loop would, the copies run on their own streams into and out of double
    buffers, so step i's compute overlaps step i+1's inputs and step i-1's results."""
    host = {}
    dt = torch.bfloat16 if b.dtype == "bf16" else torch.float32
    src = dict(q=(b.q, dt), k=(b.k, dt), v=(b.v, dt), u=(b.u, dt), dout=(b.dout, dt),
               seq_offsets=(b.seq_offsets, None), num_contextuals=(b.num_contextuals, None),
               num_targets=(b.num_targets, None), timestamps=(b.timestamps, None),
               rel_bias=(b.rel_bias, None), time_bias=(b.time_bias, None))
    for name, (a, cast) in src.items():
        t = torch.from_numpy(a)
        if cast is not None:
            t = t.to(cast)
        host[name] = t.pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    T, D = b.u.shape
    nbuf = 2
    dev, outs, saveds, gradss = [], [], [], []
    for _ in range(nbuf):
        dev.append({n: torch.empty_like(t, device="cuda") for n, t in host.items()})
        outs.append(torch.empty((T, D), dtype=dt, device="cuda"))
        saveds.append(ops.Saved(torch.empty((T, D), device="cuda"),
                                torch.empty(T, device="cuda"), torch.empty(T, device="cuda")))
        gradss.append((torch.empty(b.q.shape, dtype=dt, device="cuda"),
                       torch.empty(b.k.shape, dtype=dt, device="cuda"),
                       torch.empty(b.v.shape, dtype=dt, device="cuda"),
                       torch.empty(b.u.shape, dtype=dt, device="cuda"),
                       torch.empty(b.rel_bias.shape, device="cuda"),
                       torch.empty(b.time_bias.shape, device="cuda")))
    results = [[outs[k]] + list(gradss[k]) for k in range(nbuf)]
    host_out = [torch.empty(r.shape, dtype=r.dtype, pin_memory=True) for r in results[0]]
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(nbuf)]
    comp_done = [torch.cuda.Event() for _ in range(nbuf)]
    out_done = [torch.cuda.Event() for _ in range(nbuf)]

    def run(n, start):
        for st in (s_in, s_comp, s_out):
            st.wait_event(start)
        for i in range(n):
            k = i % nbuf
            with torch.cuda.stream(s_in):           # step i's inputs, once step i-2 is done
                if i >= nbuf:
                    s_in.wait_event(comp_done[k])
                for name in host:
                    dev[k][name].copy_(host[name], non_blocking=True)
                in_done[k].record(s_in)
            with torch.cuda.stream(s_comp):         # step i, once its results buffer is read
                s_comp.wait_event(in_done[k])
                if i >= nbuf:
                    s_comp.wait_event(out_done[k])
                d = dev[k]
                ops.fwd(d["q"], d["k"], d["v"], d["u"], d["seq_offsets"], d["num_contextuals"],
                        d["num_targets"], d["timestamps"], d["rel_bias"], d["time_bias"],
                        training=True, out=outs[k], saved=saveds[k], **kw)
                ops.bwd(d["dout"], d["q"], d["k"], d["v"], d["u"], d["seq_offsets"],
                        d["num_contextuals"], d["num_targets"], d["timestamps"], d["rel_bias"],
                        d["time_bias"], saved=saveds[k], grads=gradss[k], **kw)
                if world > 1:
                    torch.distributed.all_reduce(gradss[k][4])
                    torch.distributed.all_reduce(gradss[k][5])
                comp_done[k].record(s_comp)
            with torch.cuda.stream(s_out):          # step i's results back to the host
                s_out.wait_event(comp_done[k])
                for r, h in zip(results[k], host_out):
                    h.copy_(r, non_blocking=True)
                out_done[k].record(s_out)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    run(max(args.warmup, 3), e0)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0.record()
    run(args.steps, e0)
    for st in (s_in, s_comp, s_out):
        torch.cuda.current_stream().wait_stream(st)
    e1.record()
    e1.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    if world > 1:
        t = torch.tensor([ms], device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    return {"value": round(flops_all / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "overlap": "inputs of step i+1 and results of step i-1 copied while step i runs"}


def measure_fwd_block(ops, torch, peaks, peak_kind, cfg, args, with_cpu=True):
    """One inference-forward workload: >= 50 L2-flushed calls through the API (CUDA events
    around each call, the flush outside them), then as many again with the library's stage
    events around the attention kernel; median times; clocks sampled during the first set."""
    name, bound = FWD_BLOCKS[cfg]
    iters = max(50, args.steps)
    b = synth.make_config(cfg)
    P = accounting.valid_pairs(b)
    fl = accounting.fwd_flops(b, P)
    dev = ops.batch_to_device(b)
    out = ops.run_fwd(b, dev)
    ws = ops.fwd.last_workspace
    kw = ops.batch_kwargs(b)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    def call():
        ops.fwd(dev["q"], dev["k"], dev["v"], dev["u"], dev["seq_offsets"],
                dev["num_contextuals"], dev["num_targets"], dev["timestamps"], dev["rel_bias"],
                dev["time_bias"], out=out, workspace=ws, **kw)

    for _ in range(max(args.warmup, 3)):
        flush.fill_(1.0)
        call()
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    times = []
    for _ in range(iters):
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    clk = clocks.stop()
    evs = stage_timer(ops, torch, ["fwd_attn"])
    kt = []
    for _ in range(iters):
        flush.fill_(1.0)
        call()
        torch.cuda.synchronize()
        kt.append(evs["fwd_attn"][0].elapsed_time(evs["fwd_attn"][1]))
    ops.set_stage_events("fwd_attn")
    assert ops.read_device_status(ws) == 0
    ms = statistics.median(times)
    kms = statistics.median(kt)
    blk = {"workload": synth.WORKLOADS[cfg], "metric": "fwd TFLOP/s (valid pairs)",
           "value": round(fl / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
           "ms_per_call": round(ms, 4), "iters": iters, "timing": "median of CUDA-event times",
           "l2": "flushed before every call (256 MB write, outside the events)",
           "tokens_per_s": round(b.total_tokens / (ms * 1e-3), 1), "tokens": b.total_tokens,
           "valid_pairs": P, "flops_per_call": fl, "max_seqlen": b.max_seqlen,
           "roofline": kernel_roofline(b, "fwd_attn", kms, P, peaks, peak_kind, cfg,
                                       training=False, bound=bound),
           "clocks": clk, "gpu_launches": iters * LAUNCHES_PER_FWD}
    if cfg == 3:
        visited = accounting.tiles_with_pairs(b)
        blk["tile_skip_efficiency"] = round(P / (visited * 128 * 128), 4)
        blk["tile_skip_note"] = ("valid pairs / pairs of the 128x128 tiles visited (tiles "
                                 "holding a valid pair: %d of %d)" % (
                                     visited, int(sum(((L + 127) // 128) ** 2 for L in b.lengths))))
    if with_cpu:
        blk["cpu_baseline"] = cpu_baseline_fwd(b)
    return blk


def measure_layer_block(ops, torch, peaks, peak_kind, args, d_model=128):
    """The dense steps of the layer around the attention on the MovieLens-shaped tokens
    (d_model 128, 4 heads of 128): the fused U/V/Q/K projection and the output projection
    with residual, each timed alone (>= 50 L2-flushed calls, median) against HBM (their
    arithmetic intensity is below the ridge point)."""
    b = synth.make_config(1)
    T, H, d = b.total_tokens, b.num_heads, b.d_qk
    N = 4 * H * d
    g = torch.Generator(device="cuda").manual_seed(7)
    x = torch.randn((T, d_model), device="cuda", generator=g).to(torch.bfloat16)
    w = (torch.randn((d_model, N), device="cuda", generator=g) / d_model ** 0.5).to(torch.bfloat16)
    bw = torch.randn(N, device="cuda", generator=g) * 0.1
    z = torch.randn((T, H * d), device="cuda", generator=g).to(torch.bfloat16)
    wo = (torch.randn((H * d, d_model), device="cuda", generator=g) / (H * d) ** 0.5).to(torch.bfloat16)
    bo = torch.randn(d_model, device="cuda", generator=g) * 0.1
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    iters = max(50, args.steps)
    res = {}
    cases = {
        "uvqk_proj": (lambda: ops.uvqk_proj(x, w, bw, H, d, d),
                      2 * T * d_model + 2 * d_model * N + 4 * N + 2 * T * N, 2 * T * d_model * N),
        "out_proj": (lambda: ops.out_proj(z, wo, bo, x),
                     2 * T * H * d + 2 * H * d * d_model + 4 * d_model + 4 * T * d_model,
                     2 * T * H * d * d_model),
    }
    for name, (fn, byts, fl) in cases.items():
        for _ in range(max(args.warmup, 3)):
            fn()
        times = []
        for _ in range(iters):
            flush.fill_(1.0)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
        ms = statistics.median(times)
        gbs = byts / (ms * 1e-3) / 1e9
        res[name] = {"ms": round(ms, 4), "tflops": round(fl / (ms * 1e-3) / 1e12, 2),
                     "roofline": {"bound": "hbm", "achieved": round(gbs, 1),
                                  "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                  "frac": round(gbs / peaks["hbm_gbs"], 4),
                                  "algorithmic_bytes": byts, "peak_source": peak_kind}}
    return {"workload": "layer around the attention on the MovieLens-shaped tokens "
                        "(T=%d, d_model=%d, H=%d, d=%d), bf16" % (T, d_model, H, d),
            "iters": iters, "timing": "median of CUDA-event times, L2 flushed before each call",
            "gpu_launches": 2 * iters, **res}


def _timed_sample(b, run, target_s):
    """Times `run` (the oracle, parallel over sequences) on a sample of b's first sequences:
    one sequence first; if that is quick, as many sequences as the oracle has threads, then
    doubling until a run takes target_s / 4 (or the whole batch).  Returns (sequences,
    sub-batch, seconds, threads busy)."""
    from oracle import oracle

    threads = oracle.num_threads()
    n = 1
    while True:
        sb = synth.sub_batch(b, list(range(n)))
        t0 = time.perf_counter()
        run(sb)
        el = time.perf_counter() - t0
        if el > target_s / 4 or n >= b.batch:
            return n, sb, el, min(n, threads)
        n = min(b.batch, threads if n < threads else n * 2)


def cpu_baseline_train(b, target_s=15.0):
    """The fp64 oracle, as it stands, on a bounded sample of the training workload."""
    from oracle import oracle

    def run(sb):
        oracle.fwd(sb)
        oracle.bwd(sb)

    n, sb, el, cores = _timed_sample(b, run, target_s)
    P = accounting.valid_pairs(sb)
    fl = accounting.fwd_flops(sb, P) + accounting.bwd_flops(sb, P)
    return {"value": round(fl / el / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle", "seconds": round(el, 3),
            "sample": "first %d of %d sequences (%d tokens), fwd+bwd in fp64, one thread "
                      "per sequence" % (n, b.batch, sb.total_tokens)}


def cpu_baseline_fwd(b, target_s=12.0):
    """The fp64 oracle forward, as it stands, on a bounded sample of a forward workload."""
    from oracle import oracle

    n, sb, el, cores = _timed_sample(b, oracle.fwd, target_s)
    P = accounting.valid_pairs(sb)
    fl = accounting.fwd_flops(sb, P)
    return {"value": round(fl / el / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle", "seconds": round(el, 3),
            "sample": "first %d of %d sequences (%d tokens), forward in fp64, one thread "
                      "per sequence" % (n, b.batch, sb.total_tokens)}


def run_reference(args, world, rank):
    """The oracle timed on the host cores as the reference arm (rank 0 only): every step is
    the fp64 forward + backward of all sequences of the training workload."""
    if rank != 0:
        return
    from oracle import oracle

    full = synth.make_config(WORKLOAD_CFG)
    t0 = time.perf_counter()
    oracle.fwd(full)                 # warm-up step on the whole batch, which also sizes it
    oracle.bwd(full)
    el_full = time.perf_counter() - t0
    # keep the run within about two minutes: when K whole-batch steps would take longer,
    # every step takes every k-th sequence (the length mix kept), at least 4 per core
    k = 1
    while (args.steps * el_full / (k * 2) > 120.0 and
           full.batch // (k * 2) >= 4 * oracle.num_threads()):
        k *= 2
    b = full if k == 1 else synth.sub_batch(full, list(range(0, full.batch, k)))
    P = accounting.valid_pairs(b)
    fl = accounting.fwd_flops(b, P) + accounting.bwd_flops(b, P)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.fwd(b)
        oracle.bwd(b)
    el = (time.perf_counter() - t0) / args.steps
    v = fl / el / 1e12
    sample = ("%s %d of %d sequences per step (%d tokens), fwd+bwd in fp64" %
              ("all" if k == 1 else "every %d-th sequence:" % k, b.batch, full.batch,
               b.total_tokens))
    line = {"impl": "reference",
            "metric": METRIC,
            "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(el * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": synth.WORKLOADS[WORKLOAD_CFG], "global_batch": b.batch,
                       "parallelism": "dp%d" % world},
            "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s",
                             "cores": oracle.num_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--quick", action="store_true", help="skip the inference-forward blocks")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baselines")
    ap.add_argument("--fwd-only", type=int, default=None, metavar="WORKLOAD",
                    help="only the inference-forward block of this workload (1, 2 or 3), "
                         "without CPU baseline (for profiling its kernel)")
    ap.add_argument("--layer-only", action="store_true",
                    help="only the layer-projection block (for profiling its GEMMs)")
    args = ap.parse_args()
    if args.layer_only:
        import torch
        from jagged_hstu_attention_02_b200 import ops
        peaks, kind = load_peaks()
        print(json.dumps(measure_layer_block(ops, torch, peaks, kind, args)), flush=True)
        return
    if args.fwd_only is not None:
        import torch
        from jagged_hstu_attention_02_b200 import ops
        peaks, kind = load_peaks()
        print(json.dumps(measure_fwd_block(ops, torch, peaks, kind, args.fwd_only, args,
                                           with_cpu=False)), flush=True)
        return
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
