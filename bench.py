#!/usr/bin/env python3
"""Benchmark of Ulysses sequence-parallel attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 720p]
                    [--impl ours|reference]

One step is one pass of the whole hot path over one batch of synthetic
input: the fused sequence-parallel attention (pack + per-head-group
attention + unpack in one kernel, sp_attention_seqsharded) on the
720p/81-frame-shaped workload (75,600 tokens, 40 heads, d = 128, P = 4
virtual ranks).  The JSON line's value is algorithmic attention TFLOP/s,
4*B*N^2*H*D per step, summed over ranks, divided by the slowest rank's
device time for the K timed steps.  The three unfused rows (pack of Q, K and
V; attention on head-sharded tensors; unpack of O) are timed in the same run
and reported under "rows" (GB/s for the permutations).  Q+K+V are 2.3 GB,
far larger than the 126 MB L2, so no L2 flush is done between steps.

With --gpus N > 1 (launched by torchrun, one rank per GPU) the one 720p
problem is split across the N GPUs the way the method does (--mode ulysses,
the default: P = N ranks, NCCL all-to-all of the sequence shards, each GPU
attends H/N heads over the whole sequence, all-to-all back): strong
scaling.  --mode ulysses-peer moves the exchanges into the kernels: each
rank stores its K/V chunks straight into the head groups' buffers over peer
memory (CUDA IPC) and the attention kernel starts on the chunks that have
arrived while the rest are in flight, reads Q tiles from the ranks that hold
them and stores O rows into the ranks that own them (--kv-exchange nccl
keeps an NCCL all-to-all for K/V).  --mode replicas runs the single-GPU
problem independently on every GPU instead (no data-path collective, weak
scaling).

--impl reference times the fp64 CPU oracle on the host cores instead, each
step a bounded sample (query rows) of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SP attention TFLOP/s & % bf16 tensor peak at 75.6k tokens; pack/unpack GB/s"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = ("video_dit_sequence_b200/csrc/attention.cuh", "video_dit_sequence_b200/csrc/sm100.cuh")
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "attention_kernel_dram_traffic.txt")


def kernel_source_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(cfg):
    """DRAM bytes per launch of the attention kernel for this workload, from
    the ncu record in profiles/, or None when the record is missing, is for
    another workload, or was taken on a different kernel source."""
    try:
        with open(TRAFFIC_RECORD) as f:
            text = f.read()
    except OSError:
        return None
    fields = {}
    for line in text.splitlines():
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("kernel_source_sha256") != kernel_source_sha():
        return None
    try:
        return float(fields[f"traffic_bytes_per_launch_{cfg.name}"])
    except (KeyError, ValueError):
        return None


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The slowest rank's time: an all-reduce MAX over the default process
    group (NCCL on GPUs, gloo in the CPU tests)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, steps: int, flops_per_step: float, t_max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank runs `steps` steps of its own problem;
    the job takes as long as its slowest rank."""
    return world * steps * flops_per_step / (t_max_ms * 1e-3) / 1e12


def workload_desc(cfg):
    s = cfg.shape
    g = "x".join(str(x) for x in cfg.grid) if cfg.grid[0] else "-"
    return {"workload": f"{cfg.name}-shaped Ulysses SP attention, latent grid {g} = {s.N} tokens",
            "B": s.B, "N": s.N, "H": s.H, "D": s.D, "P": s.P,
            "causal": False, "inputs": "bf16 i.i.d. N(0,1), seeded",
            "l2": "inputs larger than L2 (no flush)"}


def oracle_sample(cfg, q, k, v, seconds, max_rows_per_head=64, threads=None):
    """Times the fp64 oracle on sampled query rows (all heads) until about
    `seconds` of CPU work; returns (TFLOP/s, rows, seconds, threads)."""
    import numpy as np

    import oracle
    import synth
    s = cfg.shape
    threads = threads or synth.host_threads()
    rows = synth.sampled_rows(cfg, max_rows_per_head)
    per_row_flops = 4.0 * s.N * s.D
    done, spent, i = 0, 0.0, 0
    while spent < seconds and i < len(rows):
        batch = rows[i:i + max(1, threads // s.H + 1)]
        rr = np.array([(0, h, t) for t in batch for h in range(s.H)], dtype=np.int64)
        t0 = time.perf_counter()
        oracle.attention_rows(q, k, v, rr, threads=threads)
        spent += time.perf_counter() - t0
        done += len(rr)
        i += len(batch)
    return done * per_row_flops / spent / 1e12, done, spent, threads


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while running."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(", ") for r in self.file.read().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except (ValueError, IndexError):
                continue
            for n, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def run_reference(args):
    """Reference arm: the fp64 CPU oracle on the host cores."""
    import synth
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = synth.CONFIGS[args.config]
    q, k, v = synth.qkv_logical(cfg)
    per_step = max(1.0, args.ref_step_seconds)
    for _ in range(args.warmup):
        oracle_sample(cfg, q, k, v, per_step / 4, max_rows_per_head=2)
    vals, rows_done, secs, thr = [], 0, 0.0, 1
    for _ in range(args.steps):
        val, r, sp_, thr = oracle_sample(cfg, q, k, v, per_step, max_rows_per_head=8)
        vals.append(val)
        rows_done += r
        secs += sp_
    value = rows_done * 4.0 * cfg.shape.N * cfg.shape.D / secs / 1e12
    sample = (f"{rows_done} query rows over {args.steps} steps (all {cfg.shape.H} heads, "
              f"full {cfg.shape.N}-key softmax each), fp64")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_desc(cfg),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ulysses(args):
    """--mode ulysses / ulysses-peer: the multi-GPU form, one rank per GPU.
    ulysses: Q, K and V exchanged by NCCL all-to-alls around the fused
    attention of the head group, O exchanged back the same way.
    ulysses-peer: K and V pushed into the head groups over peer memory and
    attended as they arrive (or, with --kv-exchange nccl, exchanged by an
    NCCL all-to-all); Q read and O written by the attention kernel itself
    over peer memory (UlyssesPeerRank)."""
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    import synth
    import video_dit_sequence_b200 as sp

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    # one rank without torchrun: a single-member group, the exchange a self-copy
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29533")
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev,
                            rank=rank, world_size=world)
    sp.load()
    cfg = synth.CONFIGS[args.config]
    s = cfg.shape
    if s.H % world:
        raise SystemExit(f"the degree {world} must divide the head count {s.H}")
    shape = sp.Shape(s.B, s.N, s.H, s.D, world)
    flops = s.flops()
    q, k, v = synth.qkv_logical(cfg)

    def pinned_shard(a):
        shard = np.ascontiguousarray(synth.to_seq_shards(a, world)[rank])
        return torch.from_numpy(shard.view(np.int16)).view(torch.bfloat16).pin_memory()

    hq, hk, hv = (pinned_shard(a) for a in (q, k, v))
    ho = torch.empty(shape.rank_shard, dtype=torch.bfloat16).pin_memory()
    dq, dk, dv = (h.to(dev) for h in (hq, hk, hv))
    stream = torch.cuda.current_stream(dev)
    a2a = sp.nccl_all_to_all()
    out = [None]
    peer = args.mode == "ulysses-peer"
    if peer:
        pr = sp.UlyssesPeerRank(shape, device=dev, kv_exchange=args.kv_exchange)
        pr.q_shard.copy_(dq)                 # Q lives in the exported shard buffer

        def step():
            out[0] = pr.step(dk, dv)
    else:
        ur = sp.UlyssesRank(shape)           # exchange buffers reused across steps

        def step():
            out[0] = sp.ulysses_attention_distributed(dq, dk, dv, shape, a2a, rank=ur)

    def timed(fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist.barrier()
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        dist.barrier()
        return a.elapsed_time(b)

    for _ in range(max(3, args.warmup)):
        step()
    if sp.device_status(stream) != sp.SP_OK:
        raise SystemExit("device status not ok after warm-up")
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = str(local)
    sampler = ClockSampler(uuid)
    time.sleep(0.3)
    n0 = sp.launch_count()
    t_ms = timed(step)
    launches = sp.launch_count() - n0
    clocks = sampler.stop()
    t_max = max_over_ranks(t_ms, world, dev)

    # end to end: the same steps on host-resident shards through the public
    # StepPipeline (H2D, the step and D2H on three streams); two rank objects
    # take turns, since a rank's buffers are reused by its next step (for the
    # peer form, other ranks write its output shard, so each step's closing
    # all-reduce also waits for the previous output's copy back)
    if peer:
        e2e_ranks = [sp.UlyssesPeerRank(shape, device=dev, kv_exchange=args.kv_exchange)
                     for _ in range(2)]
        e2e_bufs = [(r.q_shard, torch.empty_like(dk), torch.empty_like(dv)) for r in e2e_ranks]

        def e2e_fn(i, t, left):
            return e2e_ranks[i].step(t[1], t[2], release_after=left)
        groups = 1
    else:
        # the all-to-all form in head groups: each group of H/G heads is a
        # Ulysses step of its own, with a rank object per buffer set and group
        groups = sp.pipeline_head_groups(
            shape, torch.cuda.get_device_properties(dev).multi_processor_count, gpus=world)
        gshape = sp.Shape(shape.B, shape.N, shape.H // groups, shape.D, shape.P, shape.scale)
        e2e_ranks = [sp.UlyssesRank(gshape) for _ in range(2 * groups)]
        part = ((groups,) if groups > 1 else ()) + gshape.rank_shard
        e2e_bufs = [tuple(torch.empty(part, dtype=torch.bfloat16, device=dev) for _ in range(3))
                    for _ in range(2)]

        def e2e_fn(k, t, left):
            return sp.ulysses_attention_distributed(t[0], t[1], t[2], gshape, a2a,
                                                    rank=e2e_ranks[k])
    pipe = sp.StepPipeline(e2e_bufs, e2e_fn, dev, head_groups=groups)
    for _ in range(2):
        pipe.submit((hq, hk, hv), ho)
    pipe.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize(dev)
    a.record(pipe.h2d)
    last = None
    for _ in range(args.steps):
        last = pipe.submit((hq, hk, hv), ho)
    pipe.d2h.wait_event(last)
    b.record(pipe.d2h)
    torch.cuda.synchronize(dev)
    dist.barrier()
    te = max_over_ranks(a.elapsed_time(b), world, dev)
    pipe.synchronize()
    if sp.device_status(stream) != sp.SP_OK:
        raise SystemExit("device status not ok after the timed steps")
    pk, pkq = peaks()
    per_gpu = flops / world / (t_max / args.steps * 1e-3) / 1e12
    shard_bytes = 2 * math.prod(shape.rank_shard)
    if rank == 0:
        line = {"metric": METRIC, "value": args.steps * flops / (t_max * 1e-3) / 1e12,
                "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
                "ms_per_step": t_max / args.steps, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": dict(workload_desc(cfg), P=world, parallelism=f"ulysses{world}",
                               exchange=(("K/V: pushed into the head groups over peer memory, "
                                          "attention overlapped with their arrival"
                                          if args.kv_exchange == "push" else
                                          "K/V: NCCL all_to_all_single")
                                         + "; Q/O: inside the attention kernel over peer memory "
                                           "(CUDA IPC)") if peer else "NCCL all_to_all_single"),
                "e2e": {"value": args.steps * flops / (te * 1e-3) / 1e12, "unit": UNIT,
                        "h2d_bytes_per_step": int(3 * shard_bytes),
                        "d2h_bytes_per_step": int(shard_bytes),
                        "ms_per_step": te / args.steps,
                        "how": "StepPipeline: H2D, the rank's step and D2H on three streams, "
                               "two rank objects taking turns"
                               + (f", each step as {groups} groups of {shape.H // groups} heads"
                                  if groups > 1 else "")
                               + "; every step moves its own bytes"},
                "gpu_launches": int(launches), "clocks": clocks,
                "roofline": {"bound": "tensor", "kernel": "whole step per GPU",
                             "achieved": per_gpu, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": per_gpu / pk["bf16_tflops"],
                             "peak_kind": f"{pkq} bf16 dense (burst)", "traffic": None},
                "cpu_baseline": None}
        print(json.dumps(line), flush=True)
    if peer:
        pr.close()
        for r in e2e_ranks:
            r.close()
    dist.barrier()
    dist.destroy_process_group()
    return 0


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import synth
    import video_dit_sequence_b200 as sp

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    sp.load()
    cfg = synth.CONFIGS[args.config]
    if args.tokens:
        # a smaller token count of the same layout (profiling captures)
        import dataclasses
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}-N{args.tokens}",
                                  shape=dataclasses.replace(cfg.shape, N=args.tokens))
    s = cfg.shape
    shape = sp.Shape(s.B, s.N, s.H, s.D, s.P)
    flops = s.flops()
    q, k, v = synth.qkv_logical(cfg)

    def pinned(a):
        return torch.from_numpy(np.ascontiguousarray(synth.to_seq_shards(a, s.P)).view(np.int16)
                                ).view(torch.bfloat16).pin_memory()

    hq, hk, hv = pinned(q), pinned(k), pinned(v)
    ho = torch.empty(shape.seq_sharded, dtype=torch.bfloat16).pin_memory()
    qs, ks, vs = (h.to(dev) for h in (hq, hk, hv))
    os_ = torch.empty(shape.seq_sharded, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        sp.attention_seqsharded(qs, ks, vs, os_, shape, stream=stream)

    # the first call at this shape (the first warm-up step): module load,
    # tensor maps encoded, launch attributes set, one launch; no autotuning.
    # Host clock around it, synchronised on both sides.
    torch.cuda.synchronize(dev)
    t_cold = time.perf_counter()
    step()
    torch.cuda.synchronize(dev)
    cold_ms = (time.perf_counter() - t_cold) * 1e3
    for _ in range(max(3, args.warmup) - 1):
        step()
    if sp.device_status(stream) != sp.SP_OK:
        raise SystemExit("device status not ok after warm-up")

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = str(local)
    sampler = ClockSampler(uuid)
    time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = sp.launch_count()
    barrier()
    torch.cuda.synchronize(dev)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    launches = sp.launch_count() - n0
    clocks = sampler.stop()
    if sp.device_status(stream) != sp.SP_OK:
        raise SystemExit("device status not ok after the timed steps")
    t_ms = ev0.elapsed_time(ev1)
    t_max = max_over_ranks(t_ms, world, dev)
    value = weak_scaling_value(world, args.steps, flops, t_max)
    per_launch_ms = t_ms / args.steps

    # ---- unfused rows: pack (Q, K, V), attention on head-sharded, unpack (O)
    hs = shape.head_sharded
    qh, kh, vh, oh = (torch.empty(hs, dtype=torch.bfloat16, device=dev) for _ in range(4))
    os2 = torch.empty_like(os_)
    reps = max(3, args.steps)

    def timed(fn):
        for _ in range(2):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps

    tensor_bytes = 2.0 * math.prod(shape.seq_sharded)
    pk, pkq = peaks()
    t_pack = timed(lambda: sp.pack(qs, qh, shape, stream=stream))
    # the head-sharded attention row runs on the packed Q, K and V (operand
    # values change the power draw, and with it the clock, so they must be real)
    sp.pack(ks, kh, shape, stream=stream)
    sp.pack(vs, vh, shape, stream=stream)
    t_attn = timed(lambda: sp.attention(qh, kh, vh, oh, shape, stream=stream))
    t_unpack = timed(lambda: sp.unpack(oh, os2, shape, stream=stream))
    # FP8 variant of the fused step: the same problem with E4M3 Q/K/V
    t_fp8 = None
    if not args.no_fp8:
        q8, k8, v8, dq8, dk8, dv8 = synth.fp8_qkv(cfg)
        dev8 = [torch.from_numpy(np.ascontiguousarray(synth.to_seq_shards(x, s.P))).to(dev)
                for x in (q8, k8, v8)]
        fac8 = [torch.from_numpy(x).to(dev) for x in (dq8, dk8, dv8)]
        o8 = torch.empty_like(os_)
        t_fp8 = timed(lambda: sp.attention_fp8_seqsharded(*dev8, *fac8, o8, shape, stream=stream))
        del dev8, fac8, o8
    # block-sparse variant on the same problem: a synthetic cube mask of
    # density 0.2 (the pages' sparsity 0.8), one selection per 256 query tokens
    t_sparse = None
    if not args.no_sparse and s.D == 128:
        mask = synth.cube_mask(cfg, density=0.2, group=4)
        words = torch.from_numpy(sp.sparse_mask_words(mask).view(np.int32)).to(dev)
        o_sp = torch.empty_like(os_)
        t_sparse = timed(lambda: sp.attention_sparse_seqsharded(qs, ks, vs, words, o_sp, shape,
                                                                stream=stream))
        sparse_flops = 4.0 * synth.attended_pairs(mask, s.N) * s.D
        # the same density with an independent selection per query cube
        mask_ind = synth.cube_mask(cfg, density=0.2, group=1)
        words_ind = torch.from_numpy(sp.sparse_mask_words(mask_ind).view(np.int32)).to(dev)
        t_sparse_ind = timed(lambda: sp.attention_sparse_seqsharded(qs, ks, vs, words_ind, o_sp,
                                                                    shape, stream=stream))
        sparse_ind_flops = 4.0 * synth.attended_pairs(mask_ind, s.N) * s.D
        del words, words_ind, o_sp
    # the projection in front of attention (hidden -> q, k, v) with its
    # epilogue writing the sequence-sharded layout; cuBLAS on the same GEMM
    # (x @ w^T, one contiguous output) timed beside it
    t_proj = t_cublas = t_oproj = t_oproj_cublas = None
    if not args.no_proj and s.D == 128:
        hidden = s.H * s.D
        M = s.P * s.B * shape.Nl
        gen = torch.Generator(device=dev).manual_seed(5)
        xw = torch.randn(M, hidden, device=dev, generator=gen).to(torch.bfloat16)
        ww = (torch.randn(3 * hidden, hidden, device=dev, generator=gen)
              / math.sqrt(hidden)).to(torch.bfloat16)
        pq, pkk, pv = (torch.empty_like(qs) for _ in range(3))
        t_proj = timed(lambda: sp.qkv_projection(xw, ww, None, pq, pkk, pv, shape, stream=stream))
        yc = torch.empty(M, 3 * hidden, dtype=torch.bfloat16, device=dev)
        t_cublas = timed(lambda: torch.matmul(xw, ww.t(), out=yc))
        proj_flops = 2.0 * M * hidden * 3 * hidden
        del xw, ww, pq, pkk, pv, yc
        # the output projection after attention (O as sequence shards -> hidden),
        # on the fused call's output; cuBLAS on the same GEMM beside it
        wo = (torch.randn(hidden, s.H * s.D, device=dev, generator=gen)
              / math.sqrt(s.H * s.D)).to(torch.bfloat16)
        yo = torch.empty(M, hidden, dtype=torch.bfloat16, device=dev)
        t_oproj = timed(lambda: sp.out_projection(os_, wo, None, yo, shape, stream=stream))
        o2d = os_.view(M, s.H * s.D)
        t_oproj_cublas = timed(lambda: torch.matmul(o2d, wo.t(), out=yo))
        oproj_flops = 2.0 * M * s.H * s.D * hidden
        del wo, yo
    if sp.device_status(stream) != sp.SP_OK:
        raise SystemExit("device status not ok after the unfused rows")
    pack_gbs = 2 * tensor_bytes / (t_pack * 1e-3) / 1e9
    unpack_gbs = 2 * tensor_bytes / (t_unpack * 1e-3) / 1e9
    rows = {
        "pack": {"ms": t_pack, "GB/s": pack_gbs, "frac_hbm": pack_gbs / pk["hbm_gbs"],
                 "bytes": 2 * tensor_bytes, "per": "one tensor (Q, K or V), read + write"},
        "unpack": {"ms": t_unpack, "GB/s": unpack_gbs, "frac_hbm": unpack_gbs / pk["hbm_gbs"],
                   "bytes": 2 * tensor_bytes, "per": "O, read + write"},
        "attention_head_sharded": {"ms": t_attn, "TFLOP/s": flops / (t_attn * 1e-3) / 1e12},
        "fused_fp8": None if t_fp8 is None else {
            "ms": t_fp8, "TFLOP/s": flops / (t_fp8 * 1e-3) / 1e12,
            # no fp8 peak is measured: the bf16 burst figure times the nominal
            # 8-bit / 16-bit dense ratio (4.5 / 2.25 PFLOP/s)
            "peak_TFLOP/s": 2.0 * pk["bf16_tflops"],
            "frac": flops / (t_fp8 * 1e-3) / 1e12 / (2.0 * pk["bf16_tflops"]),
            "peak_source": f"{pkq} bf16 burst x 2 (nominal fp8/bf16 ratio)",
            "inputs": "E4M3 Q/K/V; factors per 128-token block (Q, K) and per "
                      "channel (V); bf16 output"},
        "sparse": None if t_sparse is None else {
            "ms": t_sparse, "speedup_vs_dense": per_launch_ms / t_sparse,
            "attended_TFLOP/s": sparse_flops / (t_sparse * 1e-3) / 1e12,
            "mask": "64-token cubes, density 0.2, one selection per 4 query cubes (synthetic)",
            "independent": {
                "ms": t_sparse_ind, "speedup_vs_dense": per_launch_ms / t_sparse_ind,
                "attended_TFLOP/s": sparse_ind_flops / (t_sparse_ind * 1e-3) / 1e12,
                "mask": "64-token cubes, density 0.2, an independent selection per query cube"}},
        "qkv_projection": None if t_proj is None else {
            "ms": t_proj, "TFLOP/s": proj_flops / (t_proj * 1e-3) / 1e12,
            "frac": proj_flops / (t_proj * 1e-3) / 1e12 / pk["bf16_tflops"],
            "cublas_ms": t_cublas, "cublas_TFLOP/s": proj_flops / (t_cublas * 1e-3) / 1e12,
            "what": f"hidden {s.H * s.D} -> q, k, v (bf16) written as sequence shards; cuBLAS: "
                    "the same GEMM into one [M][3HD] matrix"},
        "out_projection": None if t_oproj is None else {
            "ms": t_oproj, "TFLOP/s": oproj_flops / (t_oproj * 1e-3) / 1e12,
            "frac": oproj_flops / (t_oproj * 1e-3) / 1e12 / pk["bf16_tflops"],
            "cublas_ms": t_oproj_cublas,
            "cublas_TFLOP/s": oproj_flops / (t_oproj_cublas * 1e-3) / 1e12,
            "what": f"attention output {s.H * s.D} -> hidden {s.H * s.D} (bf16), O read as "
                    "sequence shards; cuBLAS: the same GEMM"},
        "unfused_step_ms": 3 * t_pack + t_attn + t_unpack,
        "fused_step_ms": per_launch_ms,
        "cold_first_call": {"ms": cold_ms, "steady_ms": per_launch_ms,
                            "what": "first fused call at this shape by the host clock: module "
                                    "load, tensor maps, launch attributes and one launch; "
                                    "no autotuning"},
    }

    # ---- end to end through the public API with host buffers: every step
    # copies its inputs in from pinned host memory and its output back out;
    # HostPipeline overlaps those transfers with the neighbouring steps'
    # compute (three streams, two device buffer sets).
    e2e = None
    if not args.no_e2e:
        del qh, kh, vh, oh, os2
        pipe = sp.HostPipeline(shape, device=dev, depth=2)
        pipe.submit(hq, hk, hv, ho)
        pipe.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        a.record(pipe.h2d)
        last = None
        for _ in range(args.steps):
            last = pipe.submit(hq, hk, hv, ho)
        pipe.d2h.wait_event(last)
        b.record(pipe.d2h)
        torch.cuda.synchronize(dev)
        barrier()
        te = max_over_ranks(a.elapsed_time(b), world, dev)
        e2e = {"value": weak_scaling_value(world, args.steps, flops, te), "unit": UNIT,
               "h2d_bytes_per_step": int(3 * tensor_bytes), "d2h_bytes_per_step": int(tensor_bytes),
               "ms_per_step": te / args.steps,
               "how": f"HostPipeline: H2D, fused attention and D2H on three streams, "
                      f"two device buffer sets, each step as {pipe.head_groups} groups of "
                      f"{pipe.group_shape.H} heads (copied in, attended and copied out one "
                      f"group at a time); every step moves its own bytes"}
        if sp.device_status(stream) != sp.SP_OK:
            raise SystemExit("device status not ok after e2e")

    achieved = flops / (per_launch_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": "attention_kernel<128> (sp_attention_seqsharded)",
                "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16_tflops"],
                "peak_kind": f"{pkq} bf16 dense (burst)",
                "frac_of_sustained": achieved / pk["bf16_tflops_sustained"],
                "traffic": args.traffic_bytes if args.traffic_bytes else recorded_traffic(cfg),
                "kernel_source_sha256": kernel_source_sha(),
                "flops_per_launch": flops}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, r, secs, thr = oracle_sample(cfg, q, k, v, args.cpu_seconds)
        cpu = {"value": val, "unit": UNIT, "cores": thr, "kind": "oracle",
               "sample": f"{r} query rows ({r // s.H} per head x {s.H} heads), each a full "
                         f"{s.N}-key fp64 softmax row, {secs:.1f} s"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": max(3, args.warmup),
                "ms_per_step": t_max / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": workload_desc(cfg), "e2e": e2e, "gpu_launches": int(launches),
                "clocks": clocks, "roofline": roofline, "cpu_baseline": cpu, "rows": rows}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--mode", choices=["replicas", "ulysses", "ulysses-peer"], default=None,
                    help="N > 1 only: one problem split across the GPUs with the Ulysses "
                         "all-to-all (ulysses, the default), the same with the exchanges in the "
                         "kernels (ulysses-peer), or independent problems per GPU (replicas)")
    ap.add_argument("--kv-exchange", choices=["push", "nccl"], default="push",
                    help="ulysses-peer: K/V pushed over peer memory and overlapped with "
                         "attention (default) or exchanged by an NCCL all-to-all")
    ap.add_argument("--config", default="720p")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-step-seconds", type=float, default=8.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 row")
    ap.add_argument("--no-sparse", action="store_true", help="skip the block-sparse row")
    ap.add_argument("--no-proj", action="store_true", help="skip the projection row")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override N (same heads, head dim and degree); for profiling captures")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="DRAM bytes per launch of the attention kernel from an ncu capture")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.mode is None:
        args.mode = "ulysses" if args.gpus > 1 else "replicas"
    if args.mode in ("ulysses", "ulysses-peer"):
        return run_ulysses(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
