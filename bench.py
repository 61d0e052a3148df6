#!/usr/bin/env python3
"""Benchmark of the VQ decode linear on B200: microseconds per layer and the
achieved HBM bandwidth of the algorithmic weight stream.

A step is one call of the layer (one pass of the whole path, x[B,K] -> y[B,N])
on one batch of synthetic input.  To keep the weights out of L2 the steps walk
a ring of distinct layer instances whose index bytes total more than twice the
L2 size; the calls are captured in CUDA graphs and replayed.  Exactly --steps
steps are timed with CUDA events that the graphs record themselves, between
two barriers.

Default workload: the Llama-2-7B-shaped 4096x4096 2-bit layer at batch 1, as a
chain of dependent calls (each call waits for the one before it and reads its
output), the latency a decode step pays per layer.  The same line carries the
ring as independent overlapping calls, as grouped calls of three layers, and
the end-to-end host-buffer call.
Multi-GPU (torchrun): every rank runs its own ring (replicas, weak scaling);
the elapsed time is the maximum over ranks and the value is the total
work of all ranks divided by it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                  [--config llama7b_layer] [--layer 0] [--batch 1]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0
METRIC = "µs/layer and achieved HBM GB/s (% of B200 peak), 2-bit VQ linear"
# About 1 ms at 1.965 GHz: queued ahead of a timed region, long enough for the
# host to enqueue every replay before the GPU reaches the start event.
SPIN_CYCLES = 2_000_000
# Untimed calls ahead of the start event (inside the same graph), and the
# calls per replay of the middle graph of a long timed region.
LEAD_IN = 8
MID_GRAPH_CALLS = 512
KERNEL_SOURCES = ("vector_quantized_weight_b200/csrc/eva_vq.cu",
                  "vector_quantized_weight_b200/csrc/eva_vq_kernels.cuh",
                  "vector_quantized_weight_b200/csrc/eva_vq_layout.cuh",
                  "vector_quantized_weight_b200/csrc/eva_vq_plan.h")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", default="eva", choices=["eva", "reference"])
    ap.add_argument("--config", default="llama7b_layer")
    ap.add_argument("--layer", type=int, default=0)
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--ring", type=int, default=0, help="ring length (0: > 2x L2)")
    ap.add_argument("--path", type=int, default=0)
    ap.add_argument("--chain", default="dependent", choices=["independent", "dependent"],
                    help="dependent (the headline): every call waits for the kernel before it "
                         "and, for a square layer, reads its output, as when each layer feeds "
                         "the next in a decode step; independent: the ring's layers are declared "
                         "independent (EVA_RUN_INDEPENDENT) and overlap")
    ap.add_argument("--no-dependent", action="store_true",
                    help="with --chain independent: skip the extra dependent-chain measurement")
    ap.add_argument("--no-independent", action="store_true",
                    help="with --chain dependent: skip the extra independent-ring measurement")
    ap.add_argument("--x-pool", type=int, default=4,
                    help="distinct activation buffers cycled by the ring (activations stay in L2, "
                         "as the output of the preceding op does in a decode step)")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--no-block", action="store_true",
                    help="skip the Llama-2-7B decoder-block leg (seven linears with their dependencies)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--group", type=int, default=3,
                    help="also time the ring as eva_vq_linear_run_group calls of this many independent "
                         "layers (e.g. a block's q, k, v); 0 skips that leg")
    return ap.parse_args()


def source_sha() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def load_traffic(workload: str):
    """dram bytes per launch of the lookup kernel from a committed ncu summary,
    or None when the kernel sources changed since it was captured."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("source_sha") == source_sha():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.15)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], [], set()
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(ms: float, pg, device) -> float:
    """Elapsed time of a replicated measurement: the maximum over ranks."""
    if pg is None:
        return ms
    import torch
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput_gbs(world: int, steps: int, bytes_per_step: int, ms: float) -> float:
    """Whole-job GB/s: every rank streams `steps` layers of `bytes_per_step`."""
    return world * steps * bytes_per_step / (ms * 1e-3) / 1e9


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def cpu_baseline(shape, B, seed, seconds):
    """The oracle, as written, on the host cores: whole layers, repeated for
    about `seconds` of CPU time."""
    import numpy as np
    import oracle
    from vector_quantized_weight_b200 import synth
    layer = synth.make_layer(shape, seed)
    x = synth.make_x(shape.K, B, seed)
    nthreads = os.cpu_count() or 1
    oracle.layer_linear(layer, x, nthreads=nthreads)     # load + page in
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.layer_linear(layer, x, nthreads=nthreads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds or (reps >= 1 and el * (reps + 1) / reps > 3 * seconds):
            break
    us = el / reps * 1e6
    return us, reps, nthreads


def stream_bytes(shape, B):
    wi = shape.N * shape.J * shape.index_bits // 8
    sg = shape.N * shape.K // 8 if shape.residual_group else 0
    al = shape.N * (shape.K // shape.residual_group) * 2 if shape.residual_group else 0
    return wi + sg + al + 2 * B * shape.K


def base_config(args, shape, B):
    """The workload keys both arms report."""
    return {"workload": f"{args.config}:{shape.name}:B{B}", "N": shape.N, "K": shape.K, "d": shape.d,
            "index_bits": shape.index_bits, "batch": B, "codebook_rows": shape.codebook_rows,
            "residual_group": shape.residual_group, "hadamard_block": shape.hadamard_block}


def oracle_rows(layer, x, rows, nthreads):
    """The oracle on output rows [0, rows) of the layer (whole codebook groups)."""
    import oracle
    s = layer.shape
    ncb = rows // s.codebook_rows if s.codebook_rows else 1
    return oracle.linear(layer.wc[:ncb], layer.wi[:rows], x,
                         signs=None if layer.signs is None else layer.signs[:rows],
                         alpha=None if layer.alpha is None else layer.alpha[:rows], hsign=layer.hsign,
                         codebook_rows=s.codebook_rows, residual_group=s.residual_group,
                         hadamard_block=s.hadamard_block, nthreads=nthreads, index_bits=s.index_bits)


def run_reference(args, shape, B, seed, world, rank):
    """The reference arm: the oracle as written on the host cores, timed for
    exactly --steps steps after --warmup untimed ones.  A step is the oracle
    on a bounded sample of the layer's output rows (the whole layer when K
    steps of it fit in about --cpu-seconds), scaled to the whole layer."""
    if rank != 0:
        return
    from vector_quantized_weight_b200 import synth
    layer = synth.make_layer(shape, seed)
    x = synth.make_x(shape.K, B, seed)
    threads = os.cpu_count() or 1
    steps = args.steps if args.steps else 20
    warmup = max(1, args.warmup if args.warmup is not None else 1)
    unit = max(16, shape.codebook_rows)
    t0 = time.perf_counter()
    oracle_rows(layer, x, shape.N, threads)                     # one whole layer sizes the sample
    t_full = time.perf_counter() - t0
    rows = shape.N
    if steps * t_full > args.cpu_seconds:
        rows = max(unit, int(shape.N * args.cpu_seconds / (steps * t_full)) // unit * unit)
    for _ in range(warmup):
        oracle_rows(layer, x, rows, threads)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle_rows(layer, x, rows, threads)
    el = time.perf_counter() - t0
    us = el / steps * 1e6 * shape.N / rows
    gbs = stream_bytes(shape, B) / (us * 1e-6) / 1e9
    sample = (f"each step: the fp64 oracle (dequantise + GEMV) on output rows [0, {rows}) of {shape.N}, "
              f"{threads} OpenMP threads over rows; time scaled to the whole layer")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "us_per_layer": round(us, 3), "n_gpus": args.gpus, "steps": steps, "warmup": warmup,
        "ms_per_step": round(us / 1e3, 6), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": base_config(args, shape, B),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world, rank, local = dist_setup()
    from vector_quantized_weight_b200 import synth
    cfg = synth.CONFIGS[args.config]
    shape = cfg.layers[args.layer]
    B = args.batch or cfg.batches[0]
    seed = synth.layer_seed(cfg.index, args.layer)

    if args.impl == "reference":
        run_reference(args, shape, B, seed, world, rank)
        return

    import numpy as np
    import torch
    from vector_quantized_weight_b200 import eva_vq

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2**20) or 126 * 2**20)
    wi_bytes = shape.N * shape.J
    ring = args.ring or max(2, math.ceil(2 * l2 / wi_bytes) + 1)
    steps = args.steps if args.steps is not None else ring * max(1, 400_000 // ring)
    warmup = max(3, args.warmup if args.warmup is not None else 2 * ring)

    # Ring of distinct layers: each replica draws its own weights (seeded).
    stream = torch.cuda.Stream(device=dev)
    layers, xs, ys = [], [], []
    with torch.cuda.stream(stream):
        for r in range(ring):
            lay = synth.make_layer(shape, seed + 1000 * (r + 1) + 7919 * rank)
            layers.append(eva_vq.from_layer(lay, max_batch=B, path=args.path, device=dev))
            if r < max(1, args.x_pool):
                xs.append(torch.from_numpy(synth.make_x(shape.K, B, seed + r)).to(dev))
            ys.append(torch.empty((B, shape.N), dtype=torch.float16, device=dev))
    torch.cuda.synchronize(dev)
    info = layers[0].info()

    group = [1]   # layers per call in the sweep

    # Dependent calls of a square layer form a true chain: call r reads the
    # output of call r - 1 (the ring wraps around).  Otherwise every call
    # reads one of the x-pool buffers, written before the timed region.
    true_chain = shape.N == shape.K

    def x_of(r, independent):
        if not independent and true_chain:
            return ys[(r - 1) % ring]
        return xs[r % len(xs)]

    def sweep(n, independent, start=0):
        i = 0
        while i < n:
            k = min(group[0], n - i)
            if k == 1:
                r = (start + i) % ring
                layers[r](x_of(r, independent), out=ys[r], stream=stream, independent=independent)
            else:
                rs = [(start + i + j) % ring for j in range(k)]
                eva_vq.run_group([layers[r] for r in rs], [x_of(r, independent) for r in rs], [ys[r] for r in rs],
                                 stream=stream, independent=independent)
            i += k

    uuid = getattr(props, "uuid", None)
    gpu_id = f"GPU-{uuid}" if uuid is not None else str(local)

    # Written before every timed region: evicts the ring from L2, so the
    # timed layers stream their weights from HBM even when the region covers
    # fewer calls than one sweep of the ring.
    flush = torch.empty(2 * l2 + (1 << 20), dtype=torch.uint8, device=dev)
    side = torch.cuda.Stream(device=dev)

    def timed_units(emit, n_units, period, lead, sample_clocks=False):
        """Time exactly n_units units on the device; emit(n, start) enqueues n
        units starting at unit `start` (mod period) on `stream`.

        The units are captured in CUDA graphs: a first graph holds a lead-in
        of units (the period's last ones, untimed), the start event and the
        first timed units; a middle graph of several periods is replayed as
        often as needed; a last graph holds the remaining units and the stop
        event.  The two events are recorded by the graphs themselves (external
        event nodes; the start event on a side branch that completes with the
        last lead-in unit), so the region holds the timed units alone, in
        steady state: no graph launch or host submission gap, and the first
        timed unit overlaps the lead-in as any unit overlaps its predecessor.  Every graph is
        replayed once untimed first; L2 is flushed and a spin kernel queued
        before the timed replays, so the timed layers stream their weights
        from HBM and the host has enqueued every replay before the GPU gets to
        them."""
        e0 = torch.cuda.Event(enable_timing=True, external=True)
        e1 = torch.cuda.Event(enable_timing=True, external=True)
        lead = min(lead, period)
        first = min(n_units, period)
        per_mid = period * max(1, MID_GRAPH_CALLS // period)
        mids, last = divmod(n_units - first, per_mid)
        graphs = []
        g_first = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_first, stream=stream):
            if lead:
                emit(lead, period - lead)
            # The start event on a branch of its own: it completes with the
            # last lead-in call, and the first timed call still depends on
            # that call alone (its programmatic launch overlap is kept).
            side.wait_stream(stream)
            e0.record(side)
            emit(first, 0)
            if n_units == first:
                e1.record(stream)
            stream.wait_stream(side)
        graphs.append((g_first, 1))
        start = first % period
        if mids:
            g_mid = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_mid, stream=stream):
                emit(per_mid, start)
            graphs.append((g_mid, mids))
        if n_units > first:
            g_last = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_last, stream=stream):
                emit(last, start)
                e1.record(stream)
            graphs.append((g_last, 1))
        with torch.cuda.stream(stream):
            for g, _ in graphs:
                g.replay()
        torch.cuda.synchronize(dev)
        if pg:
            pg.barrier()
        torch.cuda.synchronize(dev)
        clk = ClockSampler(gpu_id) if sample_clocks else None
        if clk:
            clk.__enter__()
        with torch.cuda.stream(stream):
            flush.zero_()
            torch.cuda._sleep(SPIN_CYCLES)
            for g, n in graphs:
                for _ in range(n):
                    g.replay()
        torch.cuda.synchronize(dev)
        if clk:
            clk.__exit__(None, None, None)
        if pg:
            pg.barrier()
        torch.cuda.synchronize(dev)
        ms = max_over_ranks(e0.elapsed_time(e1), pg, dev)
        del graphs
        return ms, clk

    def timed(independent, n_steps, sample_clocks):
        """Eager warm-up, then exactly n_steps calls of the ring, timed."""
        with torch.cuda.stream(stream):
            sweep(warmup, independent)
        torch.cuda.synchronize(dev)
        return timed_units(lambda n, st: sweep(n, independent, st), n_steps, ring, LEAD_IN, sample_clocks)

    head_indep = args.chain == "independent"
    ms, clk = timed(head_indep, steps, True)
    info = layers[0].info()   # the grid and path of the timed calls
    # The extra legs run whole ring sweeps (at least ten: an overlapped leg
    # fills and drains its pipeline once per timed region).
    extra_steps = ring * max(10, min(steps, 200_000) // ring)
    dep = None
    if head_indep and not args.no_dependent:
        ms_dep, _ = timed(False, extra_steps, False)
        dep = (extra_steps, ms_dep, layers[0].info().grid)
    indep = None
    if not head_indep and not args.no_independent:
        ms_ind, _ = timed(True, extra_steps, False)
        indep = (extra_steps, ms_ind, layers[0].info().grid)

    # The same independent layers, `--group` of them per eva_vq_linear_run_group call.
    grouped = None
    if args.group > 1:
        group[0] = args.group
        ms_g, _ = timed(True, extra_steps, False)
        grouped = (extra_steps, ms_g)
        group[0] = 1

    # A whole Llama-2-7B decoder block per unit (the workload's seven linears
    # with their real dependencies): q, k and v in one grouped launch reading
    # the block input; o reading q's output (standing in for the attention
    # output); gate and up in one grouped launch reading o's output; down
    # reading gate's output (standing in for act(gate) * up); the next block
    # reads down's output.  Every launch waits for the one before it.
    block = None
    if not args.no_block:
        bcfg = synth.CONFIGS["llama7b_block"]
        bsh = bcfg.layers
        block_wi = sum(sh.N * sh.J for sh in bsh)
        nblk = max(2, math.ceil(2 * l2 / block_wi) + 1)
        blayers, bys = [], []
        with torch.cuda.stream(stream):
            for b in range(nblk):
                blayers.append([eva_vq.from_layer(synth.make_layer(sh, synth.layer_seed(bcfg.index, li) + 1000 * (b + 1)
                                                                   + 7919 * rank), max_batch=B, device=dev)
                                for li, sh in enumerate(bsh)])
                bys.append([torch.zeros((B, sh.N), dtype=torch.float16, device=dev) for sh in bsh])
            bys[-1][6].copy_(torch.from_numpy(synth.make_x(bsh[6].N, B, seed)).to(dev))
        torch.cuda.synchronize(dev)

        def emit_blocks(n, start):
            for i in range(n):
                b = (start + i) % nblk
                L, Y, xin = blayers[b], bys[b], bys[(b - 1) % nblk][6]
                eva_vq.run_group(L[0:3], [xin] * 3, Y[0:3], stream=stream)
                L[3](Y[0], out=Y[3], stream=stream)
                eva_vq.run_group(L[4:6], [Y[3]] * 2, Y[4:6], stream=stream)
                L[6](Y[4], out=Y[6], stream=stream)

        with torch.cuda.stream(stream):
            emit_blocks(2 * nblk, 0)
        torch.cuda.synchronize(dev)
        n_blocks = nblk * max(10, min(steps, 200_000) // (7 * nblk))
        ms_blk, _ = timed_units(emit_blocks, n_blocks, nblk, 1)
        bbytes = sum(stream_bytes(sh, B) for sh in bsh)
        us_blk = ms_blk * 1e3 / n_blocks
        block = {"us_per_block": round(us_blk, 3), "us_per_layer": round(us_blk / len(bsh), 4),
                 "blocks": n_blocks, "ring_blocks": nblk, "launches_per_block": 4,
                 "value": round(job_throughput_gbs(world, n_blocks, bbytes, ms_blk), 4), "unit": "GB/s",
                 "algorithmic_bytes_per_block": bbytes,
                 "grids": [lay.info().grid for lay in blayers[0]],
                 "note": ("Llama-2-7B decoder block, B=%d: q,k,v (one run_group) -> o -> gate,up (one run_group) "
                          "-> down, each launch waiting for the one before it and reading its output" % B)}
        for row in blayers:
            for lay in row:
                lay.close()
        del blayers, bys

    # End to end through the public host-buffer call: x copied in from
    # pinned memory and y read back every step.
    e2e = None
    if not args.no_e2e:
        n_e2e = min(steps, 2000)
        xh = [torch.from_numpy(synth.make_x(shape.K, B, seed + r)).pin_memory() for r in range(ring)]
        yh = torch.empty((B, shape.N), dtype=torch.float16).pin_memory()
        for i in range(ring):        # every handle's first host call (captures its graph)
            layers[i].run_host(xh[i], yh, stream=stream)
        if pg:
            pg.barrier()
        torch.cuda.synchronize(dev)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for i in range(n_e2e):
            r = i % ring
            layers[r].run_host(xh[r], yh, stream=stream)
        a1.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = max_over_ranks(a0.elapsed_time(a1), pg, dev)
        sb = stream_bytes(shape, B)
        e2e = {"value": round(job_throughput_gbs(world, n_e2e, sb, ms_e2e), 4), "unit": "GB/s",
               "us_per_layer": round(ms_e2e * 1e3 / n_e2e, 3),
               "h2d_bytes_per_step": 2 * B * shape.K, "d2h_bytes_per_step": 2 * B * shape.N,
               "steps": n_e2e}

    for lay in layers:
        lay.close()
    if pg:
        pg.destroy_process_group()
    if rank != 0:
        return

    sb = stream_bytes(shape, B)
    us_layer = ms * 1e3 / steps
    gbs = job_throughput_gbs(world, steps, sb, ms)
    peak, peak_kind = load_peaks()
    workload = f"{args.config}:{shape.name}:B{B}"
    # Dominant kernel: the fused lookup kernel, one launch per step; its
    # average launch duration is the timed region over the launches.
    lookup_us = us_layer
    achieved = sb / (lookup_us * 1e-6) / 1e9
    line = {
        "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "us_per_layer": round(us_layer, 4),
        "pct_of_8tbs": round(100 * gbs / world / 8000.0, 2),
        "pct_of_measured_hbm": round(100 * gbs / world / peak, 2),
        "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": round(ms / steps, 7),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": {**base_config(args, shape, B),
                   "ring_layers": ring, "ring_index_bytes": ring * wi_bytes,
                   "l2_bytes": l2, "l2_policy": "inputs larger than L2: ring of distinct layers > 2x L2",
                   "x_pool": len(xs),
                   "graph": "calls captured in CUDA graphs, the start and stop events recorded inside them",
                   "parallelism": f"replicas x{world}",
                   "call": ("eva_vq_linear_run_ex(EVA_RUN_INDEPENDENT): the ring's layers read "
                            "activations produced before the timed region and write distinct outputs"
                            if head_indep else
                            ("eva_vq_linear_run: every call waits for the kernel before it and reads "
                             "its output y as x (a chain of layers)" if true_chain else
                             "eva_vq_linear_run: every call waits for the kernel before it (stream "
                             "order) and reads an x-pool activation")),
                   "timing": ("exactly `steps` calls between two CUDA events recorded by the graphs, after "
                              f"{LEAD_IN} untimed lead-in calls; every graph replayed once before, L2 flushed "
                              "and a spin kernel queued ahead of the replays"),
                   "grid": info.grid, "kernels_per_step": info.kernels_per_run},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 3), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": load_traffic(workload),
                     "peak_kind": peak_kind,
                     "kernel": {eva_vq.EVA_PATH_DEQUANT_MMA: "eva_dequant_kernel",
                                eva_vq.EVA_PATH_TCGEN05: "eva_tc_kernel"}.get(info.path, "eva_lookup_kernel"),
                     "algorithmic_bytes_per_launch": sb},
        "gpu_launches": steps * info.kernels_per_run,
        "clocks": clk.summary(),
    }
    if grouped:
        gs_, gms = grouped
        line["grouped_calls"] = {
            "layers_per_call": args.group, "us_per_layer": round(gms * 1e3 / gs_, 4), "steps": gs_,
            "value": round(job_throughput_gbs(world, gs_, sb, gms), 4), "unit": "GB/s",
            "note": ("eva_vq_linear_run_group(EVA_RUN_INDEPENDENT) of consecutive ring layers, one launch "
                     "each (as for a decoder block's q, k and v)")}
    if indep:
        i_steps, ms_ind, i_grid = indep
        line["independent_ring"] = {
            "us_per_layer": round(ms_ind * 1e3 / i_steps, 4), "steps": i_steps, "grid": i_grid,
            "value": round(job_throughput_gbs(world, i_steps, sb, ms_ind), 4), "unit": "GB/s",
            "note": "eva_vq_linear_run_ex(EVA_RUN_INDEPENDENT) over the ring: layers that read activations "
                    "produced earlier overlap (a throughput figure, not one layer's latency)"}
    if dep:
        dep_steps, ms_dep, dep_grid = dep
        us_dep = ms_dep * 1e3 / dep_steps
        line["dependent_chain"] = {
            "us_per_layer": round(us_dep, 4), "steps": dep_steps, "grid": dep_grid,
            "value": round(job_throughput_gbs(world, dep_steps, sb, ms_dep), 4), "unit": "GB/s",
            "note": "every call waits for the kernel before it (plain eva_vq_linear_run), as when each "
                    "layer's output feeds the next"}
    if block:
        line["decoder_block"] = block
    if e2e:
        line["e2e"] = e2e
    if not args.no_cpu:
        us_cpu, reps, threads = cpu_baseline(shape, B, seed, args.cpu_seconds)
        line["cpu_baseline"] = {"value": round(sb / (us_cpu * 1e-6) / 1e9, 4), "unit": "GB/s",
                                "us_per_layer": round(us_cpu, 2), "cores": threads, "kind": "oracle",
                                "sample": f"{reps} whole-layer oracle calls of {shape.name} B={B} "
                                          f"(dequantise + fp64 GEMV), OpenMP over output rows"}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
