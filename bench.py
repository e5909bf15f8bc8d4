"""Benchmark of the MRA-2 forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 4] [--impl reference]

One step = one whole forward pass (pool, low-resolution logits and keys,
top-k selection, CSR build, [low-resolution PV], block-sparse attention and
combine) over one batch of the seeded synthetic workload, inputs resident in
HBM.  L2 is flushed before every timed step (a 256 MiB write, then a 256 MiB
read, so that the step starts with its inputs out of L2 and no dirty lines
left to write back); each step is
timed with CUDA events on the launching stream.  Under torchrun every rank
runs its own copy of the workload (independent (batch, head) shards: weak
scaling, no data-path collective); the reported time is the max over ranks.

Rank 0 prints one JSON line.  ``--impl reference`` times the CPU oracle (the
reference arm of this build) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from resolution_block_sparse_b200.sharding import max_over_ranks, weak_scaling_seed  # noqa: E402
from resolution_block_sparse_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "MRA-2 attention fwd tokens/s and TFLOP/s (selected blocks) at N=4096; % of roofline"
L2_FLUSH_BYTES = 256 << 20
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


class L2Flush:
    """Evicts everything from L2: writes a 256 MiB buffer, then reads another
    one, so that L2 ends up holding clean lines of the second buffer (the
    write-back of the first happens here, not in the next timed kernel)."""

    def __init__(self, dev):
        self.w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.acc = torch.zeros((), dtype=torch.float32, device=dev)

    def zero_(self):
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.acc)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class ClockSampler:
    """nvidia-smi clock / throttle samples taken while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxs.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sms) if sms else None,
                "sm_max_mhz": max(maxs) if maxs else None,
                "reasons": sorted(reasons), "samples": len(sms)}


def traffic_for(kernel_phase: str, src_file: str, workload: int):
    """DRAM bytes per launch from the committed ncu record of this workload,
    or None when there is none or the kernel source changed since the
    counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(str(workload), {}).get(kernel_phase)
    except (OSError, ValueError, AttributeError):
        return None
    if not rec:
        return None
    with open(os.path.join(ROOT, "resolution_block_sparse_b200", "csrc", src_file), "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()[:16]
    if rec.get("source") != src_file or rec.get("source_sha256_16") != h:
        return None
    return rec.get("dram_bytes_per_launch")


def attention_source(w, impl: str = "") -> str:
    """Source file of the attention kernel the library runs on workload w (the
    library's dispatch rule): the tcgen05 kernel for bf16 with head size 64
    when at least 45 % of the block map is selected, the warp-level kernel
    otherwise; MRA_ATTN_IMPL=tc / =mma (impl) forces either."""
    tc_attn = w.dtype == "bf16" and w.D == 64 and (
        impl.startswith("t") or (not impl.startswith("m") and
                                 20 * min(w.block_per_row, w.nbr) * w.nbr >= 9 * w.nbr * w.nbr))
    return "mra_attn_tc.cu" if tc_attn else "mra_attn.cu"


def algorithmic(w):
    """Selected-block FLOPs and compulsory bytes of one step (per workload)."""
    esz = 2 if w.dtype == "bf16" else 4
    BH = w.B * w.H
    flops_hi = BH * w.num_block * 4 * 32 * 32 * w.D
    qkvo = 4 * BH * w.N * w.D * esz             # Q, K, V read + O write
    return flops_hi, qkvo


def run_cuda(args, w, world, rank, local):
    import resolution_block_sparse_b200 as mra

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    mra.load_library()
    # weak scaling: every rank owns a full-size batch of independent
    # (batch, head) slices of its own (rank 0 holds the seeded workload itself)
    inputs = make_inputs(w, seed=None if rank == 0 else weak_scaling_seed(1000 + w.index, rank))
    q, k, v = (inputs[x].to(dev) for x in ("q", "k", "v"))
    mask = None if inputs["mask"] is None else inputs["mask"].to(dev)
    out = torch.empty_like(q)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)
    fwd = mra.mra_attention_fwd if w.dtype == "bf16" else mra.mra_attention_fwd_f32

    def step(st=None):
        fwd(q, k, v, mask, out, w.block_per_row, w.approx_mode, w.first_n, w.diag_n,
            st if st is not None else torch.cuda.current_stream(dev))

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    status = mra.mra_get_device_status()
    launches_per_step = mra.mra_last_launch_count()

    # the forward call captured once in a CUDA graph (workspace already sized)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()

    if world > 1:
        torch.distributed.barrier()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    # per-phase kernel times: a GPU-side delay in front of each step lets the
    # host queue all launches first, so the phase events see kernels only
    mra.mra_profile_enable(True)
    mra.mra_profile_read()
    for i in range(args.steps):
        flush.zero_()
        torch.cuda._sleep(2_000_000)
        step(stream)
    torch.cuda.synchronize()
    phases = mra.mra_profile_read()
    mra.mra_profile_enable(False)
    # eager calls (same delay trick), then the timed graph replays
    for i in range(args.steps):
        flush.zero_()
        torch.cuda._sleep(2_000_000)
        starts[i].record(stream)
        step(stream)
        stops[i].record(stream)
    torch.cuda.synchronize()
    eager_ms = [s_.elapsed_time(e_) for s_, e_ in zip(starts, stops)]
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        graph.replay()
        stops[i].record(stream)
    torch.cuda.synchronize()
    step_ms = [s_.elapsed_time(e_) for s_, e_ in zip(starts, stops)]
    if world > 1:
        torch.distributed.barrier()

    # end to end through the host-buffer entry point (pinned memory)
    qh, kh, vh = (inputs[x].pin_memory() for x in ("q", "k", "v"))
    mh = None if inputs["mask"] is None else inputs["mask"].pin_memory()
    oh = torch.empty_like(qh).pin_memory()
    e2e_ms = []
    for i in range(max(args.warmup, 3) + args.steps):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        mra.mra_attention_fwd_host(qh, kh, vh, mh, oh, w.block_per_row, w.approx_mode, w.first_n,
                                   w.diag_n, stream)
        b.record(stream)
        b.synchronize()
        if i >= max(args.warmup, 3):
            e2e_ms.append(a.elapsed_time(b))
    clocks = sampler.stop()

    ms = statistics.mean(step_ms)
    e2e = statistics.mean(e2e_ms)
    eager = statistics.mean(eager_ms)
    ms, e2e, eager = max_over_ranks([ms, e2e, eager], device=dev)
    del graph
    return {"ms": ms, "e2e_ms": e2e, "eager_ms": eager, "phases": phases, "status": status,
            "launches_per_step": launches_per_step, "clocks": clocks,
            "h2d": sum(x.numel() * x.element_size() for x in (qh, kh, vh)) +
                   (0 if mh is None else mh.numel() * 4),
            "d2h": oh.numel() * oh.element_size()}


def run_cuda_backward(args, w, world, rank, local):
    """The backward pass (mra_attention_bwd) on the same workload: seeded
    incoming gradient, CUDA-graph replays timed with events, per-phase
    events (forward re-run, clearing, per-item kernel, low-resolution part)."""
    import resolution_block_sparse_b200 as mra

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    mra.load_library()
    inputs = make_inputs(w, seed=None if rank == 0 else weak_scaling_seed(1000 + w.index, rank))
    q, k, v = (inputs[x].to(dev) for x in ("q", "k", "v"))
    mask = None if inputs["mask"] is None else inputs["mask"].to(dev)
    gen = torch.Generator("cpu").manual_seed(2000 + w.index + 7919 * rank)
    dout = torch.randn(q.shape, generator=gen).to(q.dtype).to(dev)
    dq, dk, dv = (torch.empty(q.shape, dtype=torch.float32, device=dev) for _ in range(3))
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def step(st=None):
        mra.mra_attention_bwd(q, k, v, mask, dout, dq, dk, dv, w.block_per_row, w.approx_mode, w.first_n,
                              w.diag_n, st if st is not None else torch.cuda.current_stream(dev))

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    status = mra.mra_get_device_status()
    launches_per_step = mra.mra_last_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    mra.mra_profile_enable(True)
    mra.mra_profile_read()
    for _ in range(args.steps):
        flush.zero_()
        torch.cuda._sleep(2_000_000)
        step(stream)
    torch.cuda.synchronize()
    phases = mra.mra_profile_read()
    mra.mra_profile_enable(False)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        graph.replay()
        stops[i].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = statistics.mean(s_.elapsed_time(e_) for s_, e_ in zip(starts, stops))
    ms = max_over_ranks([ms], device=dev)[0]
    del graph
    return {"ms": ms, "phases": phases, "status": status, "launches_per_step": launches_per_step,
            "clocks": clocks}


def bigbird_lists(bw, rank=0):
    """Per-(batch, head) BigBird block lists of the workload from the
    library's host generator, -1 padded to the longest: int32 [BH, cap]."""
    import numpy as np

    import resolution_block_sparse_b200 as mra
    from resolution_block_sparse_b200.workloads import bigbird_random_blocks

    BH = bw.B * bw.H
    rb = bigbird_random_blocks(BH, bw.N // bw.block_size, bw.num_random, bw.seed + 7919 * rank)
    lists = [mra.mra_bigbird_block_list(bw.N, bw.block_size, rb[h]) for h in range(BH)]
    cap = max(len(x) for x in lists)
    arr = np.full((BH, cap), -1, dtype=np.int32)
    for h, x in enumerate(lists):
        arr[h, :len(x)] = x
    return arr, rb


def run_cuda_bigbird(args, bw, world, rank, local):
    """Block-sparse attention on the BigBird pattern (mra_blocksparse_attention_fwd):
    the lists are built once on the host (the layer's fixed pattern, like a
    weight) and stay on the device; CUDA-graph replays timed with events;
    end to end: pinned-host Q, K, V in, output back, through the same call."""
    import resolution_block_sparse_b200 as mra
    from resolution_block_sparse_b200.workloads import random_inputs

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    mra.load_library()
    inputs = random_inputs(bw.B, bw.H, bw.N, bw.D, dtype=torch.bfloat16, seed=bw.seed + 7919 * rank)
    q, k, v = (inputs[x].to(dev) for x in ("q", "k", "v"))
    lists, _ = bigbird_lists(bw, rank)
    idx = torch.from_numpy(lists).to(dev)
    out = torch.empty_like(q)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def step(st=None):
        # the current stream at call time: the capture stream inside torch.cuda.graph
        mra.mra_blocksparse_attention_fwd(q, k, v, None, out, idx,
                                          st if st is not None else torch.cuda.current_stream(dev))

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    status = mra.mra_get_device_status()
    launches_per_step = mra.mra_last_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    mra.mra_profile_enable(True)
    mra.mra_profile_read()
    for _ in range(args.steps):
        flush.zero_()
        torch.cuda._sleep(2_000_000)
        step(stream)
    torch.cuda.synchronize()
    phases = mra.mra_profile_read()
    mra.mra_profile_enable(False)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        graph.replay()
        stops[i].record(stream)
    torch.cuda.synchronize()
    ms = statistics.mean(s_.elapsed_time(e_) for s_, e_ in zip(starts, stops))
    # end to end: host Q, K, V (pinned) to the device, the call, the output back
    qh, kh, vh = (inputs[x].pin_memory() for x in ("q", "k", "v"))
    oh = torch.empty_like(qh).pin_memory()
    e2e_ms = []
    for i in range(max(args.warmup, 3) + args.steps):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        q.copy_(qh, non_blocking=True)
        k.copy_(kh, non_blocking=True)
        v.copy_(vh, non_blocking=True)
        step(stream)
        oh.copy_(out, non_blocking=True)
        b.record(stream)
        b.synchronize()
        if i >= max(args.warmup, 3):
            e2e_ms.append(a.elapsed_time(b))
    clocks = sampler.stop()
    e2e = statistics.mean(e2e_ms)
    ms, e2e = max_over_ranks([ms, e2e], device=dev)
    del graph
    return {"ms": ms, "e2e_ms": e2e, "phases": phases, "status": status, "launches_per_step": launches_per_step,
            "clocks": clocks, "sel_blocks": int((lists >= 0).sum()),
            "h2d": 3 * q.numel() * q.element_size(), "d2h": out.numel() * out.element_size()}


def oracle_bigbird_sampler(bw, target_s: float = 15.0):
    """The oracle's sparse-mode attention on the BigBird lists (the oracle's
    own pattern generator), the first S (batch, head) slices, scaled."""
    import numpy as np

    import oracle
    from resolution_block_sparse_b200.workloads import bigbird_random_blocks, random_inputs

    inputs = random_inputs(bw.B, bw.H, bw.N, bw.D, dtype=torch.bfloat16, seed=bw.seed)
    BH = bw.B * bw.H
    rb = bigbird_random_blocks(BH, bw.N // bw.block_size, bw.num_random, bw.seed)
    cores = os.cpu_count() or 1

    def timed(S):
        xs = [inputs[x].reshape(BH, 1, bw.N, bw.D)[:S].double().numpy() for x in ("q", "k", "v")]
        lists = [oracle.bigbird_blocks(bw.N, bw.block_size, rb[h]) for h in range(S)]
        cap = max(len(x) for x in lists)
        sel = np.stack([np.concatenate([x, np.full(cap - len(x), x[0], np.int32)]) for x in lists])
        t0 = time.perf_counter()
        oracle.attend_with_selection(xs[0], xs[1], xs[2], None, sel, approx_mode=1, nthreads=cores)
        return time.perf_counter() - t0

    S = 1
    while True:
        dt = timed(S)
        if dt >= target_s / 4 or S >= BH:
            break
        S = min(BH, S * 2)
    return bw.B * bw.N / (dt * BH / S), f"{S} of {BH} (batch, head) slices, fp64, scaled to the full step", cores


def run_cuda_layer(args, lw, world, rank, local):
    """The MraSelfAttention layer (mra_self_attention_fwd): CUDA-graph replays
    timed with events, per-phase events, and end to end with pinned-host x in
    and the output back."""
    import resolution_block_sparse_b200 as mra
    from resolution_block_sparse_b200.workloads import layer_inputs

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    mra.load_library()
    xh, wq, bq = layer_inputs(lw, seed=None if rank == 0 else lw.seed + 7919 * rank)
    x, w, b = xh.to(dev), wq.to(dev), bq.to(dev)
    out = torch.empty_like(x)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def step(st=None):
        mra.mra_self_attention_fwd(x, w, b, None, out, lw.H, lw.block_per_row, lw.approx_mode, lw.first_n,
                                   lw.diag_n, st if st is not None else torch.cuda.current_stream(dev))

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    status = mra.mra_get_device_status()
    launches_per_step = mra.mra_last_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    mra.mra_profile_enable(True)
    mra.mra_profile_read()
    for _ in range(args.steps):
        flush.zero_()
        torch.cuda._sleep(2_000_000)
        step(stream)
    torch.cuda.synchronize()
    phases = mra.mra_profile_read()
    mra.mra_profile_enable(False)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        graph.replay()
        stops[i].record(stream)
    torch.cuda.synchronize()
    ms = statistics.mean(s_.elapsed_time(e_) for s_, e_ in zip(starts, stops))
    # the projection alone against the library GEMM on the same shape
    # (cuBLAS through torch: x W^T + b with a row-major output), back to back
    qkv = torch.empty((3, lw.B, lw.H, lw.N, 32 if lw.hidden // lw.H <= 32 else 64), dtype=torch.bfloat16,
                      device=dev)
    x2 = x.reshape(-1, lw.hidden)
    b16 = b.to(torch.bfloat16)
    lib_out = torch.empty(x2.shape[0], 3 * lw.hidden, dtype=torch.bfloat16, device=dev)
    cmp_us = {}
    for name, fn in (("mra_qkv_projection", lambda: mra.mra_qkv_projection(x, w, b, qkv, lw.H)),
                     ("torch_addmm_cublas", lambda: torch.addmm(b16, x2, w.t(), out=lib_out))):
        for _ in range(10):
            fn()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(200):
            fn()
        ev1.record(stream)
        torch.cuda.synchronize()
        cmp_us[name] = ev0.elapsed_time(ev1) / 200 * 1e3
    xp = xh.pin_memory()
    oh = torch.empty_like(xp).pin_memory()
    e2e_ms = []
    for i in range(max(args.warmup, 3) + args.steps):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        x.copy_(xp, non_blocking=True)
        step(stream)
        oh.copy_(out, non_blocking=True)
        e.record(stream)
        e.synchronize()
        if i >= max(args.warmup, 3):
            e2e_ms.append(a.elapsed_time(e))
    clocks = sampler.stop()
    e2e = statistics.mean(e2e_ms)
    ms, e2e = max_over_ranks([ms, e2e], device=dev)
    del graph
    return {"ms": ms, "e2e_ms": e2e, "phases": phases, "status": status, "launches_per_step": launches_per_step,
            "clocks": clocks, "h2d": x.numel() * x.element_size(), "d2h": out.numel() * out.element_size(),
            "projection_vs_library_us": cmp_us}


def oracle_layer_sampler(lw, target_s: float = 15.0):
    """The oracle's layer on a sample of the work: the first S heads of the
    first batch entry (their slice of the projection and their attention),
    scaled to the full step by the number of (batch, head) slices."""
    import oracle
    from resolution_block_sparse_b200.workloads import layer_inputs

    x, w, b = layer_inputs(lw)
    cores = os.cpu_count() or 1
    d = lw.hidden // lw.H
    xd = x[:1].double().numpy()

    def timed(S):
        rows = [j * lw.hidden + i for j in range(3) for i in range(S * d)]
        ws = w.double().numpy()[rows][:, :]
        bs = b.double().numpy()[rows]
        t0 = time.perf_counter()
        # S heads of one batch entry: hidden_out = S * d, input width unchanged
        proj = xd @ ws.T + bs
        q, k, v = (proj[:, :, j * S * d:(j + 1) * S * d].reshape(1, lw.N, S, d).transpose(0, 2, 1, 3)
                   for j in range(3))
        oracle.forward(q, k, v, None, block_per_row=lw.block_per_row, approx_mode=lw.approx_mode,
                       first_n=lw.first_n, diag_n=lw.diag_n, nthreads=cores, want_intermediates=False)
        return time.perf_counter() - t0

    S = 1
    while True:
        dt = timed(S)
        if dt >= target_s / 4 or S >= lw.H:
            break
        S = min(lw.H, S * 2)
    heads_total = lw.B * lw.H
    return (lw.B * lw.N / (dt * heads_total / S),
            f"{S} of {heads_total} (batch, head) slices (their projection and attention), fp64, scaled", cores)


def oracle_backward_sampler(w, target_s: float = 15.0):
    """The oracle's backward on a bounded sample of the workload, like
    oracle_sampler."""
    import oracle

    inputs = make_inputs(w)
    gen = torch.Generator("cpu").manual_seed(2000 + w.index)
    dout = torch.randn(inputs["q"].shape, generator=gen).to(inputs["q"].dtype)
    cores = os.cpu_count() or 1
    BH = w.B * w.H

    def slices(S):
        xs = [inputs[x].reshape(BH, 1, w.N, w.D)[:S].double().numpy() for x in ("q", "k", "v")]
        g = dout.reshape(BH, 1, w.N, w.D)[:S].double().numpy()
        m = None
        if inputs["mask"] is not None:
            m = inputs["mask"].repeat_interleave(w.H, dim=0)[:S].double().numpy()
        return xs[0], xs[1], xs[2], m, g

    def timed(a):
        t0 = time.perf_counter()
        oracle.backward(*a, block_per_row=w.block_per_row, approx_mode=w.approx_mode, first_n=w.first_n,
                        diag_n=w.diag_n, nthreads=cores)
        return time.perf_counter() - t0

    S = 1
    while True:
        dt = timed(slices(S))
        if dt >= target_s / 4 or S >= BH:
            break
        S = min(BH, S * 2)
    return w.B * w.N / (dt * BH / S), f"{S} of {BH} (batch, head) slices, fp64, scaled to the full step", cores


def oracle_sampler(w, target_s: float = 15.0):
    """A bounded sample of the workload for the CPU oracle: the first S
    (batch, head) slices, S grown (once) until one run takes about target_s
    / 4 to target_s seconds.  Returns (run, sample text, cores); run() times
    one oracle pass over the sample and returns tokens/s of the whole
    workload at that rate."""
    import oracle

    inputs = make_inputs(w)
    cores = os.cpu_count() or 1
    BH = w.B * w.H

    def slices(S):
        q = inputs["q"].reshape(BH, 1, w.N, w.D)[:S].double().numpy()
        k = inputs["k"].reshape(BH, 1, w.N, w.D)[:S].double().numpy()
        v = inputs["v"].reshape(BH, 1, w.N, w.D)[:S].double().numpy()
        m = None
        if inputs["mask"] is not None:
            m = inputs["mask"].repeat_interleave(w.H, dim=0)[:S].double().numpy()
        return q, k, v, m

    def timed(args):
        t0 = time.perf_counter()
        oracle.forward(*args, block_per_row=w.block_per_row, approx_mode=w.approx_mode,
                       first_n=w.first_n, diag_n=w.diag_n, nthreads=cores, want_intermediates=False)
        return time.perf_counter() - t0

    S = 1
    while True:
        dt = timed(slices(S))
        if dt >= target_s / 4 or S >= BH:
            break
        S = min(BH, S * 2)
    sample = slices(S)
    tokens = w.B * w.N

    def run():
        return tokens / (timed(sample) * BH / S)

    return run, f"{S} of {BH} (batch, head) slices, fp64, scaled to the full step", cores


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=4)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="which", default="forward", choices=["forward", "backward", "bigbird", "layer"],
                    help="backward: time mra_attention_bwd on the workload instead; bigbird: block-sparse "
                         "attention on the BigBird pattern; layer: the MraSelfAttention layer (own JSON lines)")
    args = ap.parse_args()
    world, rank, local = dist_env()
    w = WORKLOADS[args.workload]
    flops_hi, qkvo = algorithmic(w)
    tokens = w.B * w.N
    config = {"workload": w.describe(), "B": w.B, "H": w.H, "N": w.N, "D": w.D,
              "block_per_row": w.block_per_row, "num_block": w.num_block,
              "approx_mode": "full" if w.approx_mode == 0 else "sparse",
              "first_n": w.first_n, "diag_n": w.diag_n,
              "l2": "flushed before every timed step (256 MiB write, then 256 MiB read)",
              "timing": "CUDA-graph replay of one mra_attention_fwd call per step, CUDA events",
              "parallelism": f"replicas x{world} (independent (batch, head) shards)"}

    if args.impl == "reference":
        if rank != 0:
            return
        # W warm-up and K timed steps, each a bounded sample (about 2 s of
        # oracle work) of the workload, scaled to the full step
        run, sample, cores = oracle_sampler(w, target_s=2.0)
        for _ in range(args.warmup):
            run()
        steps_s = [run() for _ in range(max(1, args.steps))]
        value = statistics.mean(steps_s)
        config = dict(config, timing="oracle on the host cores, wall clock per bounded sample, "
                                     "scaled to the full step")
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
                "n_gpus": 1, "steps": len(steps_s), "warmup": args.warmup,
                "ms_per_step": 1000.0 * tokens / value, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": config,
                "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                                 "kind": "oracle", "sample": sample},
                "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    if args.which == "layer":
        from resolution_block_sparse_b200.workloads import LAYER as lw

        res = run_cuda_layer(args, lw, world, rank, local)
        ms = res["ms"]
        lt = lw.B * lw.N
        phases = {k_: {"launches": v_[0], "avg_us": 1e3 * v_[1] / max(1, v_[0])} for k_, v_ in res["phases"].items()}
        proj_flops = 2 * lw.B * lw.N * 3 * lw.hidden * lw.hidden
        prj = phases.get("qkv_proj", {"avg_us": 0.0})
        peaks, src = load_peaks()
        achieved = proj_flops / (prj["avg_us"] * 1e-6) / 1e12 if prj["avg_us"] > 0 else None
        lconfig = {"workload": lw.name, "B": lw.B, "N": lw.N, "hidden": lw.hidden, "H": lw.H,
                   "block_per_row": lw.block_per_row, "approx_mode": "full" if lw.approx_mode == 0 else "sparse",
                   "first_n": lw.first_n, "diag_n": lw.diag_n,
                   "l2": "flushed before every timed step (256 MiB write, then 256 MiB read)",
                   "timing": "CUDA-graph replay of one mra_self_attention_fwd call per step, CUDA events",
                   "parallelism": f"replicas x{world} (independent batch shards)"}
        line = {"metric": f"MraSelfAttention layer fwd tokens/s at N={lw.N}", "pass": "layer",
                "value": world * lt / (ms / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": lconfig,
                "phases_us": phases,
                "roofline": {"kernel": "qkv_proj", "bound": "tensor", "achieved": achieved,
                             "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": (achieved / peaks["bf16_tflops"]) if achieved else None, "traffic": None,
                             "peak_source": f"{src} (burst)", "algorithmic_flops_per_launch": proj_flops},
                "e2e": {"value": world * lt / (res["e2e_ms"] / 1e3), "unit": "tokens/s",
                        "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"]},
                "projection_vs_library_us": res["projection_vs_library_us"],
                "gpu_launches": res["launches_per_step"] * args.steps, "device_status": res["status"],
                "clocks": res["clocks"]}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            val, sample, cores = oracle_layer_sampler(lw)
            line["cpu_baseline"] = {"value": val, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                    "sample": sample}
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        if rank == 0:
            print(json.dumps(line))
        return
    if args.which == "bigbird":
        from resolution_block_sparse_b200.workloads import BIGBIRD as bw

        res = run_cuda_bigbird(args, bw, world, rank, local)
        ms = res["ms"]
        bb_tokens = bw.B * bw.N
        flops = 4 * 32 * 32 * bw.D * res["sel_blocks"]
        bytes_ = 4 * bw.B * bw.H * bw.N * bw.D * 2          # Q, K, V read + O write (bf16)
        att = res["phases"].get("attention", (1, 0.0))
        att_s = att[1] / max(1, att[0]) / 1e3
        peaks, src = load_peaks()
        t_hbm = bytes_ / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops / (peaks["bf16_tflops"] * 1e12)
        if t_tc >= t_hbm:
            bound, unit, achieved, peak = "tensor", "TFLOP/s", flops / att_s / 1e12, peaks["bf16_tflops"]
        else:
            bound, unit, achieved, peak = "hbm", "GB/s", bytes_ / att_s / 1e9, peaks["hbm_gbs"]
        bconfig = {"workload": bw.name, "B": bw.B, "H": bw.H, "N": bw.N, "D": bw.D,
                   "block_size": bw.block_size, "num_random_blocks": bw.num_random,
                   "selected_32x32_blocks": res["sel_blocks"],
                   "l2": "flushed before every timed step (256 MiB write, then 256 MiB read)",
                   "timing": "CUDA-graph replay of one mra_blocksparse_attention_fwd call per step, CUDA events",
                   "parallelism": f"replicas x{world} (independent (batch, head) shards)"}
        line = {"metric": f"BigBird block-sparse attention fwd tokens/s at N={bw.N}", "pass": "bigbird",
                "value": world * bb_tokens / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic", "config": bconfig,
                "tflops_selected_blocks": world * flops / (ms / 1e3) / 1e12,
                "phases_us": {k_: {"launches": v_[0], "avg_us": 1e3 * v_[1] / max(1, v_[0])}
                              for k_, v_ in res["phases"].items()},
                "roofline": {"kernel": "attention", "bound": bound, "achieved": achieved, "peak": peak,
                             "unit": unit, "frac": achieved / peak, "traffic": None,
                             "peak_source": f"{src} (burst)", "algorithmic_bytes_per_launch": bytes_,
                             "algorithmic_flops_per_launch": flops},
                "e2e": {"value": world * bb_tokens / (res["e2e_ms"] / 1e3), "unit": "tokens/s",
                        "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"]},
                "gpu_launches": res["launches_per_step"] * args.steps, "device_status": res["status"],
                "clocks": res["clocks"]}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            val, sample, cores = oracle_bigbird_sampler(bw)
            line["cpu_baseline"] = {"value": val, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                    "sample": sample}
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        if rank == 0:
            print(json.dumps(line))
        return
    if args.which == "backward":
        res = run_cuda_backward(args, w, world, rank, local)
        ms = res["ms"]
        sel_blocks = w.B * w.H * w.num_block
        flops = 10 * 32 * 32 * w.D * sel_blocks   # S, dP, dQ, dK, dV per selected block
        item_us = res["phases"].get("bwd_items", (1, 0.0))
        item_s = item_us[1] / max(1, item_us[0]) / 1e3
        clk = res["clocks"].get("sm_max_mhz") or 1965.0
        achieved = flops / item_s / 1e12 if item_s > 0 else None
        if w.dtype == "bf16":   # the per-item kernel runs its products on the tensor cores
            peaks, src = load_peaks()
            bound, peak = "tensor", peaks["bf16_tflops"]
            peak_source = f"{src} (burst) bf16 tensor"
        else:                   # fp32 inputs: FFMA
            bound, peak = "alu", 148 * 128 * 2 * clk * 1e6 / 1e12
            peak_source = "derived: 148 SMs x 128 fp32 lanes x 2 flop x max SM clock"
        line = {"metric": f"MRA-2 attention bwd tokens/s (selected blocks) at N={w.N}", "pass": "backward",
                "value": world * tokens / (ms / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32 (" + w.dtype + " inputs)", "data": "synthetic",
                "config": dict(config, timing="CUDA-graph replay of one mra_attention_bwd call per step "
                                              "(forward re-run included), CUDA events"),
                "phases_us": {k_: {"launches": v_[0], "avg_us": 1e3 * v_[1] / max(1, v_[0])}
                              for k_, v_ in res["phases"].items()},
                "roofline": {"kernel": "bwd_items", "bound": bound, "achieved": achieved, "peak": peak,
                             "unit": "TFLOP/s", "frac": (achieved / peak) if achieved else None, "traffic": None,
                             "peak_source": peak_source, "algorithmic_flops_per_launch": flops},
                "gpu_launches": res["launches_per_step"] * args.steps, "device_status": res["status"],
                "clocks": res["clocks"]}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            val, sample, cores = oracle_backward_sampler(w)
            line["cpu_baseline"] = {"value": val, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                    "sample": sample}
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        if rank == 0:
            print(json.dumps(line))
        return
    res = run_cuda(args, w, world, rank, local)
    peaks, peak_src = load_peaks()

    ms = res["ms"]
    value = world * tokens / (ms / 1e3)
    tflops = world * flops_hi / (ms / 1e3) / 1e12
    phases = {k: {"launches": n, "avg_us": 1000.0 * t / max(n, 1)} for k, (n, t) in res["phases"].items()}
    # dominant kernel phase and its roofline
    dom = max((k for k in phases if k != "memset"), key=lambda k: phases[k]["avg_us"])
    dom_s = phases[dom]["avg_us"] * 1e-6
    esz = 2 if w.dtype == "bf16" else 4
    BH = w.B * w.H
    kernel_src = {"attention": attention_source(w, os.environ.get("MRA_ATTN_IMPL", "")), "pool": "mra_pool.cu",
                  "lowres_keys": "mra_lowres.cu", "lowres_pv": "mra_lowres.cu", "select": "mra_select.cu",
                  "lowres_select": "mra_lowres_select.cu", "group_plan": "mra_group_plan.cu"}
    if dom == "attention":
        # compulsory Q, K, V read + O write of the attended heads; intensity
        # 16*block_per_row flop/B is below the bf16 ridge -> HBM bound
        bytes_ = qkvo
        bound, unit, achieved, peak = "hbm", "GB/s", bytes_ / dom_s / 1e9, peaks["hbm_gbs"]
    elif dom == "pool":
        ntens = 3 if w.approx_mode == 0 else 2
        bytes_ = ntens * BH * w.N * w.D * esz + ntens * BH * w.nbr * w.D * 4
        bound, unit, achieved, peak = "hbm", "GB/s", bytes_ / dom_s / 1e9, peaks["hbm_gbs"]
    else:
        bytes_ = 8 * BH * w.nbr * w.nbr * 2
        bound, unit, achieved, peak = "hbm", "GB/s", bytes_ / dom_s / 1e9, peaks["hbm_gbs"]
    roofline = {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak, "peak_source": f"{peak_src} (burst)",
                "algorithmic_bytes_per_launch": bytes_,
                "traffic": traffic_for(dom, kernel_src.get(dom, "mra_attn.cu"), w.index)}
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic", "config": config,
            "tflops_selected_blocks": tflops,
            "tensor_frac_selected_blocks": tflops / peaks["bf16_tflops"],
            "roofline": roofline, "phases_us": phases,
            "ms_per_step_eager": res["eager_ms"],
            "e2e": {"value": world * tokens / (res["e2e_ms"] / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"]},
            "gpu_launches": res["launches_per_step"] * args.steps,
            "device_status": res["status"], "clocks": res["clocks"]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        run, sample, cores = oracle_sampler(w)
        val = run()
        line["cpu_baseline"] = {"value": val, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": sample}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))


if __name__ == "__main__":
    main()
