#!/usr/bin/env python
"""DF11 decode benchmark: decoded BF16 GB/s and fraction of the HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
                    [--impl {b200,reference}]

A step is one pass of the whole decode path over one workload: every tensor
of it decoded from its resident compressed form into BF16 in HBM (one
batched launch per 16 tensors).  The default workload is the 36-layer
Qwen3-8B-shaped stack (embedding, 36 blocks of 7 weights, LM head:
8,190,427,136 elements, one codebook per tensor), decoded layer by layer
into one reused scratch buffer on one stream.  Other workloads: single
(1024x1024), block (one Qwen3-8B-shaped block), adversarial (64M mix),
fibonacci (32-bit codewords), embedding (151936x4096).

Inputs are seeded synthetic tensors; every step's output is checked
bit-exact against the original tensor before any number is printed.

Multi-GPU (torchrun): every rank decodes its own copy of the workload (its
own seed) -- the decode has no exchange step, so there is no collective on
the data path; the timed region is bracketed by barriers and the time is the
maximum over ranks.

--impl reference times the CPU oracle (single-threaded C, bit-serial decode)
on the host on the same workload and metric, as the comparison arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = ("decoded BF16 GB/s and % of HBM roofline (1×B200), "
          "bit-exact vs CPU oracle")
UNIT = "GB/s"
GEMM_METRIC = ("BF16-equivalent weight GB/s through the fused decode and tensor-core "
               "matrix product (1×B200), within the fp32 sum bound of the exact product")
GEMV_METRIC = ("BF16-equivalent weight GB/s through the fused decode and matrix-vector "
               "product (1×B200), within the fp32 sum bound of the exact product")
BUILD_METRIC = ("compressed BF16 GB/s (device-side format builder, 1×B200), "
                "byte-identical to the host builder")
# launches of the library's own kernels per batched device build besides
# the histograms: tile bits, scan, pack and finish for the batch
BUILD_LAUNCHES_PER_BATCH = 4
BUILD_TILE = 16384        # elements per histogram tile
BUILD_HIST_JOBS = 32      # tensors per histogram launch
KERNEL_SRC = os.path.join(ROOT, "huffman_decode_df11_b200", "csrc", "df11_decode.cu")
BUILD_SRC = os.path.join(ROOT, "huffman_decode_df11_b200", "csrc", "df11_gpu_build.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.txt")
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, the data-sheet figure


# ---------------------------------------------------------------------------
# workloads as lists of (name, thunk(device) -> int16 bits)

def workload_units(config: str, seed: int):
    if config == "single":
        return [("w_1024x1024", lambda d: workloads.single_matrix(seed, d))]
    if config == "block":
        return [(name, (lambda d, i=i: workloads.block_tensor(seed, i, d)))
                for i, (name, _, _) in enumerate(workloads.BLOCK_SHAPES)]
    if config == "adversarial":
        return [("adversarial_64M", lambda d: workloads.adversarial_mix(64 << 20, seed, d))]
    if config == "fibonacci":
        return [("fibonacci34", lambda d: workloads.fibonacci_exponents(seed, d))]
    if config == "embedding":
        return [("embed_151936x4096", lambda d: workloads.embedding(seed, d))]
    if config == "stack":
        return [(name, thunk) for name, _, thunk in workloads.stack_units(seed)]
    if config in ("build", "gemv", "gemm"):  # the block's tensors
        return workload_units("block", seed)
    if config == "offload":  # the stack's first layers, without embedding and LM head
        return [(name, thunk) for name, _, thunk
                in workloads.stack_units(seed, OFFLOAD_LAYERS)[1:-1]]
    raise ValueError(config)


def block_groups(config: str, names):
    """Groups of tensors decoded by one batched call (a layer at a time)."""
    if config not in ("stack", "offload"):
        return [list(range(len(names)))]
    groups, cur, layer = [], [], None
    for i, n in enumerate(names):
        key = n.split(".")[1] if n.startswith("layers.") else n
        if key != layer and cur:
            groups.append(cur)
            cur = []
        layer = key
        cur.append(i)
    groups.append(cur)
    return groups


def workload_elements(config: str) -> int:
    """Elements of a workload, from its shapes (no tensor is generated)."""
    block = sum(r * c for _, r, c in workloads.BLOCK_SHAPES)
    emb = workloads.VOCAB * workloads.HIDDEN
    return {"single": 1 << 20, "block": block, "build": block, "gemv": block, "gemm": block,
            "adversarial": 64 << 20, "fibonacci": 14_930_351, "embedding": emb,
            "stack": 2 * emb + workloads.LAYERS * block,
            "offload": OFFLOAD_LAYERS * block}[config]


def algorithmic_bytes(h, counts: bool = True) -> int:
    """Bytes one decode of this tensor must move: compressed input (stream,
    sign/mantissa, gaps, chunk counts when used, block positions, tables,
    code lengths) + 2 B/elem of BF16 output."""
    p = h.params
    chunks = p.num_blocks * p.threads_per_block
    return ((p.total_bits + 7) // 8 + p.n + (5 * chunks + 7) // 8 + 4 * (p.num_blocks + 1)
            + (chunks if counts else 0) + 1024 * p.num_luts + 256 + 2 * p.n)


def kernel_hash(src: str = KERNEL_SRC) -> str:
    return hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]


def recorded_traffic(workload: str, src: str = KERNEL_SRC):
    """Per-launch (per-step for the builder) DRAM bytes from an ncu capture
    of the current kernel source (profiles/dram_traffic.txt: '<source sha16>
    <workload>/c<C>/t<T> <bytes>')."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    kh = kernel_hash(src)
    for line in open(TRAFFIC_FILE):
        parts = line.split()
        if len(parts) >= 3 and not line.startswith("#") and parts[0] == kh and parts[1] == workload:
            return float(parts[2])
    return None


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        try:
            return float(json.load(open(path))["hbm_gbs"]), "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------

def setup_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


L2_BYTES = 126 * 2 ** 20  # B200 L2 cache
FLUSH_BYTES = 2 * L2_BYTES


def flush_wanted(mode: str, step_bytes: int) -> bool:
    """Whether L2 is rewritten before every timed step: always ('on'), never
    ('off'), or when one step's inputs and outputs fit in L2 ('auto')."""
    if mode == "on":
        return True
    if mode == "off":
        return False
    return step_bytes < L2_BYTES


def gpu_sleep(cycles: int = 200_000):
    """A kernel that spins for about `cycles` SM clocks (~0.1 ms): queued
    before a per-launch event pair so that the GPU is still busy while the
    host queues the pair and the launch between them."""
    torch.cuda._sleep(cycles)


def time_steps(step, steps: int, stream, new_event, flush=None) -> float:
    """Mean device milliseconds of one step over `steps` steps, from events
    recorded on `stream`.  Without `flush`, one event pair brackets all the
    steps, so that launches run back to back.  With `flush` (a tensor larger
    than L2), the tensor is rewritten before each step, which evicts the
    previous step's data, and each step is timed by its own event pair."""
    if steps < 1:
        raise ValueError("time at least one step")
    if flush is None:
        a, b = new_event(), new_event()
        a.record(stream)
        for _ in range(steps):
            step()
        b.record(stream)
        b.synchronize()
        return a.elapsed_time(b) / steps
    pairs = []
    for s in range(steps):
        flush.fill_(s + 1)
        a, b = new_event(), new_event()
        a.record(stream)
        step()
        b.record(stream)
        pairs.append((a, b))
    pairs[-1][1].synchronize()
    return sum(a.elapsed_time(b) for a, b in pairs) / steps


def prepare(config: str, seed: int, device: str, chunk_bytes: int = 24,
            threads_per_block: int = 256, host_build: bool = False):
    """Compress every unit and keep the compressed tensors resident in HBM.
    By default one decode group (a layer) at a time on the device
    (compress_on_device_batched, byte-identical to the host builder);
    host_build=True runs the host builder instead.  Originals are
    regenerated from the seed when checked."""
    import huffman_decode_df11_b200 as df11
    units = workload_units(config, seed)
    groups = block_groups(config, [u[0] for u in units])
    devs = [None] * len(units)
    for g in groups:
        if host_build:
            for i in g:
                h = df11.compress(units[i][1](device), chunk_bytes=chunk_bytes,
                                  threads_per_block=threads_per_block)
                devs[i] = df11.to_device(h, device)
            continue
        ws = [units[i][1](device) for i in g]
        for i, d in zip(g, df11.compress_on_device_batched(ws, chunk_bytes, threads_per_block)):
            devs[i] = d
        del ws
    torch.cuda.synchronize()
    return units, groups, devs


class LazyHosts:
    """Host copies of device-resident compressed tensors, made on first use
    (the CPU baseline and the end-to-end leg touch only a few of them)."""

    def __init__(self, devs):
        self._devs, self._cache = devs, {}

    def __len__(self):
        return len(self._devs)

    def __getitem__(self, i):
        if i not in self._cache:
            import huffman_decode_df11_b200 as df11
            self._cache[i] = df11.to_host(self._devs[i])
        return self._cache[i]

    def __iter__(self):
        return (self[i] for i in range(len(self)))


def run_b200(args, world, rank, local):
    import huffman_decode_df11_b200 as df11
    device = f"cuda:{local}"
    seed = args.seed + rank
    units, groups, devs = prepare(args.config, seed, device, args.chunk_bytes,
                                  args.threads_per_block, args.host_build)
    names = [u[0] for u in units]
    n_total = sum(d.n for d in devs)
    # one reused scratch buffer sized for the largest group
    group_elems = [sum(devs[i].n for i in g) for g in groups]
    scratch = torch.empty(max(group_elems), dtype=torch.bfloat16, device=device)
    outs_for = []
    for g in groups:
        off, outs = 0, []
        for i in g:
            outs.append(scratch[off:off + devs[i].n])
            off += devs[i].n
        outs_for.append(outs)
    err = df11.new_error_word(device)
    stream = torch.cuda.current_stream()

    counts = not args.no_counts

    plans = [df11.DecodePlan([devs[i] for i in g], outs_for[gi], counts=counts)
             for gi, g in enumerate(groups)]

    def step(events=None):
        for gi, plan in enumerate(plans):
            if events is not None:
                # keep the GPU busy while the host queues the event and the
                # launch, so that the pair times the launch, not host latency
                gpu_sleep()
                events[gi][0].record(stream)
            plan.run(err=err, stream=stream)
            if events is not None:
                events[gi][1].record(stream)

    # the decode-before-use pattern: after each layer's decode a small
    # kernel that is not a decode reads the decoded weights (a sum over a
    # slice of every tensor), so that no decode launch follows another
    probe = torch.zeros(len(groups), dtype=torch.int16, device=device)
    # every 1021st word of the layer's output: one reduction kernel per
    # layer, which reads every tensor of it
    heads = [scratch[: group_elems[gi]: 1021].view(torch.int16) for gi in range(len(groups))]

    def consume(gi):
        torch.amax(heads[gi], dim=0, out=probe[gi])

    def step_consumed():
        for gi, plan in enumerate(plans):
            plan.run(err=err, stream=stream)
            consume(gi)

    def consumers_only():
        for gi in range(len(plans)):
            consume(gi)

    # parity: every group's output equals the original, bit for bit
    for gi, g in enumerate(groups):
        df11.decode_batched([devs[i] for i in g], outs_for[gi], err=err, stream=stream,
                            counts=not args.no_counts)
        torch.cuda.synchronize()
        for i, o in zip(g, outs_for[gi]):
            ref = units[i][1](device)
            if not torch.equal(o.view(torch.int16), ref):
                raise SystemExit(f"parity failure on {names[i]}")
            del ref
    df11.check_device_error(err)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    launches_per_step = sum((len(g) + 15) // 16 for g in groups)
    alg = [sum(algorithmic_bytes(devs[i], counts) for i in g) for g in groups]
    flush_used = flush_wanted(args.flush_l2, sum(alg))
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=device) if flush_used else None
    # per-launch events only in a separate pass after the timed region: an
    # event between two launches keeps the second from starting while the
    # first finishes (programmatic dependent launch)
    pg_steps = min(args.steps, 50)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in groups] for _ in range(pg_steps)]
    cons_steps = max(3, min(args.steps, 50))
    new_ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    with ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                      else local) as clocks:
        # keep the GPU busy (untimed) while the sampler starts, so that the
        # samples taken around a short timed region show clocks under load
        t_busy = time.perf_counter()
        while not args.no_clock_window and time.perf_counter() - t_busy < 0.4:
            step()
            torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        ms_local = time_steps(step, args.steps, stream, new_ev, flush)
        torch.cuda.synchronize()
        barrier(world)
        for s in range(pg_steps):
            step(ev[s])
        torch.cuda.synchronize()
        if not flush_used:
            step_consumed()
            consumers_only()
            torch.cuda.synchronize()
            cons_ms = time_steps(step_consumed, cons_steps, stream, new_ev)
            only_ms = time_steps(consumers_only, cons_steps, stream, new_ev)
            torch.cuda.synchronize()
    df11.check_device_error(err)
    del flush
    ms = max_over_ranks(ms_local, world)
    out_bytes_all = sum_over_ranks(2.0 * n_total, world)
    value = out_bytes_all / (ms * 1e-3) / 1e9

    # per-launch (per-layer) durations, each launch timed alone by events on
    # the launch stream; the roofline divides the algorithmic bytes of a
    # step by the step's time in the timed region, where only the decode
    # kernel runs, launch after launch
    per_group_ms = [statistics.mean(ev[s][gi][0].elapsed_time(ev[s][gi][1])
                                    for s in range(pg_steps)) for gi in range(len(groups))]
    achieved = sum(alg) / (ms_local * 1e-3) / 1e9
    # each launch alone: no overlap with the launch before it
    achieved_call = sum(alg) / (sum(per_group_ms) * 1e-3) / 1e9
    peak, peak_kind = measured_peak()
    # the capture covers the chunk-count kernel; the page-layout kernel has none
    traffic = (recorded_traffic(f"{args.config}/c{args.chunk_bytes}/t{args.threads_per_block}")
               if counts else None)
    consumer = None
    if not flush_used:
        dec_ms = cons_ms - only_ms
        consumer = {
            "ms_per_step": round(cons_ms, 4), "consumers_only_ms": round(only_ms, 4),
            "decode_ms": round(dec_ms, 4),
            "frac": round(sum(alg) / (dec_ms * 1e-3) / 1e9 / peak, 4),
            "what": "each layer's decode followed by a non-decode kernel reading its output "
                    "(one reduction over every 1021st word of the layer); decode_ms = "
                    "ms_per_step - consumers_only_ms"}

    hosts = LazyHosts(devs)
    # end to end through the public API: host (pinned) compressed tensors in,
    # host BF16 out, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(args, units, hosts, groups, device, world,
                          ns=[d.n for d in devs])

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(hosts, args.cpu_budget_s)

    if rank == 0:
        compressed = sum(d.compressed_bytes() for d in devs)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT,
            "elements_per_s": round(out_bytes_all / 2.0 / (ms * 1e-3), 1),
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u32",
            "data": "synthetic (seeded; fp32 samples rounded to BF16 RNE)",
            "config": {
                "workload": WORKLOAD_NAMES[args.config], "tensors": len(units),
                "elements": n_total, "chunk_bytes": args.chunk_bytes,
                "threads_per_block": args.threads_per_block,
                "compressed_bytes": compressed,
                "bits_per_weight": round(8.0 * compressed / n_total, 3),
                "builder": "host" if args.host_build else "device (byte-identical to host)",
                "l2": (f"L2 flushed before every step ({FLUSH_BYTES >> 20} MiB written); "
                       "each step timed alone by its own events") if flush_used else
                      "inputs larger than L2 (no flush)" if sum(alg) >= L2_BYTES else
                      "inputs smaller than L2, not flushed: numbers include L2 reuse",
                "us_per_call": round(1e3 * ms / launches_per_step, 2),
                "parallelism": f"replicas x{world} (no collective)",
                "parity": "bit-exact vs original on every tensor before timing",
                "chunk_counts": not args.no_counts,
            },
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1),
                         "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4),
                         "frac_what": "decode launches back to back; consecutive launches "
                                      "overlap by programmatic dependent launch",
                         "achieved_per_call": round(achieved_call, 1),
                         "frac_per_call": round(achieved_call / peak, 4),
                         "frac_per_call_what": "each launch timed alone by events on its "
                                               "stream (no overlap with a neighbour; a "
                                               "spin kernel ahead of each event pair keeps "
                                               "host latency out)",
                         "traffic": traffic, "peak_kind": peak_kind,
                         "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                         "nominal_peak": NOMINAL_HBM_GBS,
                         "algorithmic_bytes_per_step": sum(alg)},
            "decode_then_consumer": consumer,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks.summary(),
            "e2e": e2e,
            "cpu_baseline": cpu,
            "per_group_ms": [round(x, 4) for x in per_group_ms]
            if len(groups) <= 8 else {"min": round(min(per_group_ms), 4),
                                      "max": round(max(per_group_ms), 4),
                                      "mean": round(statistics.mean(per_group_ms), 4),
                                      "sum": round(sum(per_group_ms), 4),
                                      "groups": len(groups),
                                      "names": [names[g[0]].split(".")[0] if len(g) == 1
                                                else ".".join(names[g[0]].split(".")[:2])
                                                for g in (groups[0], groups[-1])]},
        }
        print(json.dumps(line), flush=True)


def run_offload(args, world, rank, local):
    """Layers kept in pinned host memory, each copied to the GPU (one copy of
    its packed compressed buffers) and decoded there, the next layer's copy
    overlapping the current decode (OffloadPipeline).  Timed per pass over
    all layers.  Beside it: the same two-slot copy pipeline moving the raw
    BF16 layers (what offloading uncompressed weights costs), and a plain
    pinned host-to-device copy as the PCIe bandwidth the pass is held to."""
    import huffman_decode_df11_b200 as df11
    from huffman_decode_df11_b200 import offload
    device = f"cuda:{local}" if world > 1 else "cuda"
    seed = args.seed + rank
    units = workload_units(args.config, seed)
    names = [u[0] for u in units]
    groups = block_groups(args.config, names)
    hosts, raw = [], []
    for _, thunk in units:
        bits = thunk(device)
        hosts.append(df11.compress(bits, chunk_bytes=args.chunk_bytes,
                                   threads_per_block=args.threads_per_block))
        raw.append(bits.cpu())
        del bits
    packed = [offload.pack_layer([hosts[i] for i in g], device) for g in groups]
    layer_n = [sum(hosts[i].n for i in g) for g in groups]
    n_total = sum(layer_n)
    scratch = torch.empty(max(layer_n), dtype=torch.int16, device=device)
    outs = []
    for g in groups:
        off, o = 0, []
        for i in g:
            o.append(scratch[off:off + hosts[i].n])
            off += hosts[i].n
        outs.append(o)
    pipe = offload.OffloadPipeline(packed, outs, device=device)
    err = df11.new_error_word(device)
    stream = torch.cuda.current_stream()

    # parity: every layer's output against the original, right after its decode
    bad = []

    def check(li):
        for i, o in zip(groups[li], outs[li]):
            if not torch.equal(o, units[i][1](device)):
                bad.append(names[i])
    pipe.run(err=err, after_layer=check)
    torch.cuda.synchronize()
    if bad:
        raise SystemExit(f"parity failure on {bad[0]}")
    df11.check_device_error(err)

    err_host = torch.empty(1, dtype=torch.int32).pin_memory()

    def step():
        pipe.run(err=err, stream=stream)
        err_host.copy_(err, non_blocking=True)  # the step's result read back

    def timed(fn, steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps

    for _ in range(args.warmup):
        step()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        barrier(world)
        ms_local = timed(step, args.steps)
        barrier(world)
    df11.check_device_error(err)
    ms = max_over_ranks(ms_local, world)
    value = sum_over_ranks(2.0 * n_total, world) / (ms * 1e-3) / 1e9

    # uncompressed offload: the same two slots and streams, raw BF16 layers
    layer_raw = [torch.cat([raw[i].view(-1) for i in g]).pin_memory() for g in groups]
    slots = [torch.empty(max(t.numel() for t in layer_raw), dtype=torch.int16, device=device)
             for _ in range(2)]
    cs = torch.cuda.Stream()
    ev = [torch.cuda.Event() for _ in range(len(layer_raw))]
    free = [torch.cuda.Event() for _ in range(2)]

    def raw_step():
        for e in free:
            e.record(stream)
        for li, t in enumerate(layer_raw):
            s = li % 2
            with torch.cuda.stream(cs):
                cs.wait_event(free[s])
                slots[s][: t.numel()].copy_(t, non_blocking=True)
                ev[li].record(cs)
            stream.wait_event(ev[li])
            free[s].record(stream)
    raw_step()
    raw_ms = timed(raw_step, max(3, args.steps // 4))
    # PCIe: one pinned copy of the largest packed layer, back to back
    big = packed[0].host
    dst = torch.empty(big.numel(), dtype=torch.uint8, device=device)
    h2d_ms = timed(lambda: dst.copy_(big, non_blocking=True), 10)
    h2d_gbs = big.numel() / (h2d_ms * 1e-3) / 1e9
    achieved = pipe.h2d_bytes / (ms_local * 1e-3) / 1e9
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u32",
            "data": "synthetic (seeded; fp32 samples rounded to BF16 RNE)",
            "config": {
                "workload": WORKLOAD_NAMES[args.config], "tensors": len(units),
                "layers": len(groups), "elements": n_total,
                "chunk_bytes": args.chunk_bytes,
                "threads_per_block": args.threads_per_block,
                "h2d_bytes_per_pass": pipe.h2d_bytes,
                "parallelism": f"replicas x{world} (no collective)",
                "parity": "bit-exact vs original on every tensor before timing",
            },
            "roofline": {"bound": "pcie", "achieved": round(achieved, 1),
                         "peak": round(h2d_gbs, 1), "unit": "GB/s",
                         "frac": round(achieved / h2d_gbs, 4), "traffic": None,
                         "peak_kind": "measured here (pinned host-to-device copy)",
                         "algorithmic_bytes_per_step": pipe.h2d_bytes},
            "bf16_offload": {"ms_per_step": round(raw_ms, 4),
                             "value": round(2.0 * n_total / (raw_ms * 1e-3) / 1e9, 2),
                             "unit": UNIT, "h2d_bytes_per_pass": 2 * n_total},
            "gpu_launches": len(groups) * args.steps,
            "clocks": clocks.summary(),
            "e2e": {"value": round(value, 2), "unit": UNIT,
                    "h2d_bytes_per_step": pipe.h2d_bytes, "d2h_bytes_per_step": 4},
            "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)


def build_algorithmic_bytes(h) -> int:
    """Bytes a build of this tensor must move: the BF16 input read twice (the
    code depends on the whole histogram, so the codewords can only be
    written in a second pass; the input is larger than L2) and the
    compressed tensor written once."""
    return 4 * h.n + h.compressed_bytes()


def _same_bytes(d, h) -> bool:
    for f in ("bitstream", "gaps", "chunk_counts", "block_out_pos", "luts", "code_lengths",
              "sign_mantissa"):
        got = getattr(d, f).cpu().numpy().view(np.uint8)
        want = np.ascontiguousarray(getattr(h, f)).view(np.uint8)
        if got.shape != want.shape or not np.array_equal(got, want):
            return False
    return all(getattr(d.params, f) == getattr(h.params, f) for f, _ in d.params._fields_)


def build_hist_launches(sizes) -> int:
    """Histogram launches of one batched device build of tensors of these
    sizes: the tensors in order, at most BUILD_HIST_JOBS per launch, and the
    shortest run of last tensors that holds a quarter of the tiles in a
    launch of its own; a launch whose tensors are all empty runs no kernel."""
    tiles = [-(-n // BUILD_TILE) for n in sizes]
    if not tiles:
        return 0
    count, total = len(tiles), sum(tiles)
    tail, tail_tiles = count - 1, tiles[-1]
    while tail > 0 and count - tail < BUILD_HIST_JOBS and 4 * tail_tiles < total:
        tail -= 1
        tail_tiles += tiles[tail]
    cuts = list(range(0, tail, BUILD_HIST_JOBS)) + [tail, count]
    return sum(1 for a, b in zip(cuts, cuts[1:]) if sum(tiles[a:b]))


def run_build(args, world, rank, local):
    """The format builder on the device: every tensor of the workload
    compressed from BF16 already in HBM (df11_gpu_build_begin_batched /
    _finish_batched via compress_on_device_batched, one call per step).
    Parity: byte-identical buffers and parameters to the host builder, and a
    decode back to the original words, before any timing.  A step builds
    every tensor once: the counts come back to the host for the codebooks,
    and the largest block, chunk and warp counts at the end (two round trips
    per step, in the timed region)."""
    import huffman_decode_df11_b200 as df11
    device = f"cuda:{local}"
    seed = args.seed + rank
    units = workload_units(args.config, seed)
    C, T = args.chunk_bytes, args.threads_per_block
    ws = [thunk(device) for _, thunk in units]
    hosts = []
    for (name, _), w in zip(units, ws):
        h = df11.compress(w, chunk_bytes=C, threads_per_block=T)
        d = df11.compress_on_device(w, C, T)
        if not _same_bytes(d, h):
            raise SystemExit(f"device build differs from the host build on {name}")
        out = df11.decode(d)
        torch.cuda.synchronize()
        if not torch.equal(out.view(torch.int16).view(w.shape), w):
            raise SystemExit(f"device build does not decode to the original on {name}")
        hosts.append(h)
        del d, out
    n_total = sum(h.n for h in hosts)
    stream = torch.cuda.current_stream()

    def step():
        df11.compress_on_device_batched(ws, C, T, decode_table=False)

    for _ in range(args.warmup):
        step()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        # keep the GPU busy (untimed) while the sampler starts, so that the
        # samples taken around a short timed region show clocks under load
        t_busy = time.perf_counter()
        while not args.no_clock_window and time.perf_counter() - t_busy < 0.4:
            step()
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms_local = t0.elapsed_time(t1) / args.steps
    ms = max_over_ranks(ms_local, world)
    value = sum_over_ranks(2.0 * n_total, world) / (ms * 1e-3) / 1e9
    alg = sum(build_algorithmic_bytes(h) for h in hosts)
    achieved = alg / (ms_local * 1e-3) / 1e9
    peak, peak_kind = measured_peak()
    traffic = recorded_traffic(f"build/c{C}/t{T}", BUILD_SRC)

    # end to end: BF16 in pinned host memory, copied in, built, and the
    # compressed buffers copied back to pinned host memory, every step
    e2e = None
    if not args.no_e2e:
        pins = [w.cpu().pin_memory() for w in ws]
        devs = [torch.empty_like(w) for w in ws]
        backs = [{f: torch.empty(getattr(h, f).nbytes, dtype=torch.uint8).pin_memory()
                  for f in ("bitstream", "gaps", "chunk_counts", "block_out_pos", "luts",
                            "code_lengths", "sign_mantissa")} for h in hosts]

        def e2e_step():
            for pin, dev in zip(pins, devs):
                dev.copy_(pin, non_blocking=True)
            built = df11.compress_on_device_batched(devs, C, T, decode_table=False)
            for d, back in zip(built, backs):
                for f, b in back.items():
                    b.copy_(getattr(d, f).view(torch.uint8).view(-1), non_blocking=True)
            torch.cuda.synchronize()

        for _ in range(2):
            e2e_step()
        e_steps = max(3, min(args.steps, 20))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        a.record(stream)
        for _ in range(e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e_ms = max_over_ranks(a.elapsed_time(b) / e_steps, world)
        e2e = {"value": round(sum_over_ranks(2.0 * n_total, world) / (e_ms * 1e-3) / 1e9, 2),
               "unit": UNIT, "h2d_bytes_per_step": 2 * n_total,
               "d2h_bytes_per_step": sum(h.compressed_bytes() for h in hosts),
               "ms_per_step": round(e_ms, 4)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_build_baseline(ws, args.cpu_budget_s)
    if rank == 0:
        line = {
            "metric": BUILD_METRIC, "value": round(value, 2), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u32",
            "data": "synthetic (seeded; fp32 samples rounded to BF16 RNE)",
            "config": {
                "workload": WORKLOAD_NAMES[args.config], "tensors": len(units),
                "elements": n_total, "chunk_bytes": C, "threads_per_block": T,
                "compressed_bytes": sum(h.compressed_bytes() for h in hosts),
                "l2": "inputs larger than L2 (no flush)",
                "parallelism": f"replicas x{world} (no collective)",
                "parity": "byte-identical to the host builder and bit-exact decode, "
                          "every tensor, before timing",
            },
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": traffic, "peak_kind": peak_kind,
                         "algorithmic_bytes_per_step": alg,
                         "kernel": "the whole build (histogram launches of up to 32 "
                                   "tensors, 4 batch launches, 2 host round trips per "
                                   "step), timed as one"},
            "gpu_launches": (build_hist_launches([h.n for h in hosts]) +
                             BUILD_LAUNCHES_PER_BATCH) * args.steps,
            "clocks": clocks.summary(),
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def run_gemv(args, world, rank, local):
    """y = W x for each weight of the block, W decoded inside the product
    (decode_gemv: one launch for the seven weights, the BF16 weights never
    written), against the same product done in two steps (batched decode
    into a BF16 scratch buffer, then a cuBLAS matrix-vector product per
    weight) and against BF16 weights kept uncompressed (cuBLAS alone).
    Parity: every output within the fp32 summation bound of the float64
    product of the original weights, before timing."""
    import huffman_decode_df11_b200 as df11
    device = f"cuda:{local}"
    seed = args.seed + rank
    B = args.batch
    tc = args.config == "gemm"  # the tensor-core product (decode_gemm)
    if not 1 <= B <= (128 if tc else 8):
        raise SystemExit(f"--batch must be 1..{128 if tc else 8}")
    # the fused path's format: decode_gemm takes 128 rows interleaved and
    # 8-byte chunks; decode_gemv the --chunk-bytes and --interleave given
    fc = args.chunk_bytes if not tc else (args.chunk_bytes if args.chunk_bytes in (8, 16) else 8)
    fil = 128 if tc else args.interleave
    units = workload_units(args.config, seed)
    shapes = [(r, c) for _, r, c in workloads.BLOCK_SHAPES]
    ds, ws_bf16, fused_ds = [], [], []
    for (name, thunk), shape in zip(units, shapes):
        bits = thunk(device)
        # the two-step path's weights: row-major, the decode's own format
        d = df11.compress_on_device(bits, chunk_bytes=24 if tc else args.chunk_bytes,
                                    threads_per_block=args.threads_per_block)
        d.shape = shape
        ds.append(d)
        if fil != 1 or fc != args.chunk_bytes:  # the fused path's weights
            fused_ds.append(df11.compress_on_device(bits.view(shape), chunk_bytes=fc,
                                                    threads_per_block=args.threads_per_block,
                                                    interleave=fil))
        ws_bf16.append(bits.view(shape).view(torch.bfloat16))
    hosts = LazyHosts(ds)
    n_total = sum(d.n for d in ds)
    g = torch.Generator(device=device)
    g.manual_seed(seed + 77)
    xs = [torch.randn(B, c, generator=g, device=device).to(torch.bfloat16) for _, c in shapes]
    ys = [torch.empty(B, r, dtype=torch.float32, device=device) for r, _ in shapes]
    err = df11.new_error_word(device)
    stream = torch.cuda.current_stream()

    fds = fused_ds if fused_ds else ds
    product = df11.decode_gemm if tc else df11.decode_gemv
    # parity: within gamma_cols * |x||W|^T of the float64 product
    product(fds, xs, ys, err=err)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    for (name, _), (r, c), x, y, w in zip(units, shapes, xs, ys, ws_bf16):
        W = w.double()
        ref = x.double() @ W.T
        k = c * 2.0 ** -24
        bound = (k / (1 - k)) * (x.double().abs() @ W.abs().T)
        if not torch.all((y.double() - ref).abs() <= bound):
            raise SystemExit(f"gemv outside the fp32 bound on {name}")
        del W, ref, bound

    scratch = torch.empty(max(d.n for d in ds), dtype=torch.bfloat16, device=device)
    plans = [df11.DecodePlan([d], [scratch[: d.n]]) for d in ds]

    def fused():
        product(fds, xs, ys, err=err, stream=stream)

    ybs = [torch.empty(B, r, dtype=torch.bfloat16, device=device) for r, _ in shapes]

    def two_step():  # decode each weight into the scratch buffer, then cuBLAS (BF16 out)
        for plan, d, x, yb, (r, c) in zip(plans, ds, xs, ybs, shapes):
            plan.run(err=err, stream=stream)
            torch.matmul(x, scratch[: d.n].view(r, c).T, out=yb)

    def bf16():  # uncompressed weights resident in HBM, cuBLAS (BF16 out)
        for w, x, yb in zip(ws_bf16, xs, ybs):
            torch.matmul(x, w.T, out=yb)

    def timed(fn, steps):
        for _ in range(args.warmup):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return a.elapsed_time(b) / steps

    with ClockSampler(torch.cuda.current_device()) as clocks:
        t_busy = time.perf_counter()
        while not args.no_clock_window and time.perf_counter() - t_busy < 0.4:
            fused()
            torch.cuda.synchronize()
        ms_local = timed(fused, args.steps)
    df11.check_device_error(err)
    ms_two = timed(two_step, max(3, args.steps // 4))
    ms_bf16 = timed(bf16, max(3, args.steps // 4))
    ms = max_over_ranks(ms_local, world)
    value = sum_over_ranks(2.0 * n_total, world) / (ms * 1e-3) / 1e9
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        x_host = [workloads.as_numpy_u16(x.view(torch.int16)) for x in xs]
        done, secs, what = _oracle_gemv_sample(hosts, shapes, x_host, args.cpu_budget_s)
        cpu = {"value": round(2.0 * done / secs / 1e9, 4), "unit": UNIT, "cores": 1,
               "kind": "oracle", "sample": what + " (bit-serial C decode, float64 product)"}
    alg = sum(algorithmic_bytes(d) - 2 * d.n for d in fds) + \
        sum(x.numel() * 2 for x in xs) + sum(y.numel() * 4 for y in ys)
    achieved = alg / (ms_local * 1e-3) / 1e9
    peak, peak_kind = measured_peak()
    if rank == 0:
        line = {
            "metric": GEMM_METRIC if tc else GEMV_METRIC, "value": round(value, 2), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u32+f32",
            "data": "synthetic (seeded; fp32 samples rounded to BF16 RNE)",
            "config": {
                "workload": WORKLOAD_NAMES[args.config], "tensors": len(units),
                "elements": n_total, "batch": B, "interleave": fil,
                "chunk_bytes": fc, "two_step_chunk_bytes": 24 if tc else args.chunk_bytes,
                "threads_per_block": args.threads_per_block,
                "l2": "inputs larger than L2 (no flush)",
                "parallelism": f"replicas x{world} (no collective)",
                "parity": "every output within gamma_cols*|x||W|^T of the float64 product "
                          "of the original weights, before timing",
                "y": "y = W x (the call clears y first)",
            },
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": None,
                         "peak_kind": peak_kind, "algorithmic_bytes_per_step": alg,
                         "kernel": ("df11_decode_gemm_kernel (decode into shared memory, "
                                    "tcgen05.mma into tensor memory)" if tc else
                                    "df11_decode_ws_kernel (fused product epilogue)") +
                                   ", one launch per step for the seven weights"},
            "decode_then_cublas": {"ms_per_step": round(ms_two, 4),
                                   "value": round(2.0 * n_total / (ms_two * 1e-3) / 1e9, 2)},
            "bf16_cublas": {"ms_per_step": round(ms_bf16, 4),
                            "value": round(2.0 * n_total / (ms_bf16 * 1e-3) / 1e9, 2)},
            "gpu_launches": args.steps,
            "clocks": clocks.summary(),
            "e2e": None,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def _oracle_encode_sample(ws, budget_s: float):
    """Encode leading slices of the workload's tensors with the oracle until
    the budget is spent; returns (elements, seconds, description)."""
    import oracle
    done, t_used, names = 0, 0.0, 0
    for w in ws:
        if t_used >= budget_s:
            break
        # bound one call to what fits the remaining budget (~40 ns/element)
        count = int(min(w.numel(), max(2048, (budget_s - t_used) / 40e-9)))
        a = workloads.as_numpy_u16(w.reshape(-1)[:count])
        t = time.perf_counter()
        oracle.encode(a, 24, 256)
        t_used += time.perf_counter() - t
        done += count
        names += 1
    return done, t_used, f"{done} elements from the first {names} tensor(s), encoded in order"


def cpu_build_baseline(ws, budget_s: float):
    done, secs, what = _oracle_encode_sample(ws, budget_s)
    return {"value": round(2.0 * done / secs / 1e9, 4), "unit": UNIT, "cores": 1,
            "kind": "oracle", "sample": what + " (single-threaded C encoder)"}


def measure_e2e(args, units, hosts, groups, device, world, ns=None):
    import huffman_decode_df11_b200 as df11
    # bounded host memory: the first groups up to ~2G elements
    keep, elems = [], 0
    for g in groups:
        g_n = sum(ns[i] if ns is not None else hosts[i].n for i in g)
        if keep and elems + g_n > 2_000_000_000:
            break
        keep.append(g)
        elems += g_n
    sampled = len(keep) < len(groups)
    groups = keep
    idx = [i for g in groups for i in g]
    hosts = {i: hosts[i] for i in idx}
    # pinned host copies of the compressed tensors; device staging; pinned out
    pinned, staged, out_dev, out_host = {}, {}, {}, {}
    for i, h in hosts.items():
        pinned[i] = {k: torch.from_numpy(getattr(h, k).view(np.uint8)).pin_memory()
                     for k in ("bitstream", "gaps", "block_out_pos", "luts",
                               "code_lengths", "sign_mantissa", "chunk_counts")}
        staged[i] = df11.to_device(h, device)
        out_dev[i] = df11.empty_output(staged[i])
        out_host[i] = torch.empty(h.n, dtype=torch.bfloat16).pin_memory()
    err = df11.new_error_word(device)
    stream = torch.cuda.current_stream()
    h2d = sum(sum(t.numel() for t in p.values()) for p in pinned.values())
    d2h = sum(2 * h.n for h in hosts.values())

    # per tensor: host-to-device copy on one stream, decode on the compute
    # stream, device-to-host copy on a third, so that the copy in of a
    # tensor, the decode of the one before and the copy out of the one before
    # that overlap (PCIe moves both directions at once)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = {i: torch.cuda.Event() for i in idx}
    ev_dec = {i: torch.cuda.Event() for i in idx}
    # smallest tensor first: the copy out, the slowest stage, starts as early as possible
    order = sorted(idx, key=lambda i: hosts[i].n)

    def step():
        s_in.wait_stream(stream)   # the previous step's decodes are done with the inputs
        stream.wait_stream(s_out)  # and its copies out are done with the outputs
        for i in order:
            with torch.cuda.stream(s_in):
                for k, t in pinned[i].items():
                    getattr(staged[i], k).view(torch.uint8).copy_(t, non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            df11.decode_batched([staged[i]], [out_dev[i]], err=err, stream=stream,
                                counts=not args.no_counts)
            ev_dec[i].record(stream)
            s_out.wait_event(ev_dec[i])
            with torch.cuda.stream(s_out):
                out_host[i].copy_(out_dev[i], non_blocking=True)
        stream.wait_stream(s_out)  # the step ends with its last result on the host

    step()
    torch.cuda.synchronize()
    for i in idx:  # the host result is the original tensor, bit for bit
        if not torch.equal(out_host[i].view(torch.int16), units[i][1](device).cpu()):
            raise SystemExit(f"e2e parity failure on {units[i][0]}")
    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 10))
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    df11.check_device_error(err)
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world)
    out_bytes_all = sum_over_ranks(2.0 * sum(h.n for h in hosts.values()), world)
    res = {"value": round(out_bytes_all / (ms * 1e-3) / 1e9, 2), "unit": UNIT,
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
           "ms_per_step": round(ms, 3), "steps": steps,
           "path": "per tensor: pinned host compressed -> H2D (copy stream) -> "
                   "df11_decode_batched -> D2H pinned (second copy stream), overlapped"}
    if sampled:
        res["sample"] = f"first {len(groups)} decode groups ({len(idx)} tensors)"
    return res


def _oracle_sample(hosts, budget_s: float):
    """Decode the workload's tensors with the oracle until the budget is
    spent; returns (decoded elements, seconds, description)."""
    import oracle
    done, t_used, names = 0, 0.0, 0
    for h in hosts:
        if t_used >= budget_s:
            break
        count = h.n
        # bound one call to what fits the remaining budget (~15 ns/element)
        cap = int(max(1, (budget_s - t_used) / 15e-9))
        count = min(count, cap)
        t = time.perf_counter()
        out, _, _ = oracle.decode(h.bitstream, h.code_lengths, h.sign_mantissa, count)
        t_used += time.perf_counter() - t
        done += count
        names += 1
    return done, t_used, f"{done} elements from the first {names} tensor(s), decoded in order"


def cpu_baseline(hosts, budget_s: float):
    done, secs, what = _oracle_sample(hosts, budget_s)
    return {"value": round(2.0 * done / secs / 1e9, 4), "unit": UNIT, "cores": 1,
            "kind": "oracle", "sample": what + " (single-threaded bit-serial C decode)"}


def _oracle_prefix_formats(units, elements: int, chunk_bytes: int, threads_per_block: int):
    """The workload's tensors generated on the host and their leading
    elements (up to `elements` in all, in order) encoded by the oracle's own
    encoder: the bounded sample the reference arm decodes.  No library of
    the GPU path is loaded.  Returns (formats, description).  `units` may
    also give a row length per tensor, (name, thunk, cols), to encode whole
    rows only."""
    import oracle
    fmts, left, names = [], elements, []
    for unit in units:
        name, thunk = unit[0], unit[1]
        if left <= 0:
            break
        w = thunk("cpu")
        take = int(min(w.numel(), left))
        if len(unit) > 2:  # whole rows
            take = min(w.numel(), -(-take // unit[2]) * unit[2])
        fmts.append(oracle.encode(workloads.as_numpy_u16(w.reshape(-1)[:take]),
                                  chunk_bytes, threads_per_block))
        names.append(f"{name}[:{take}]")
        left -= take
        del w
    return fmts, f"oracle-encoded leading elements of {', '.join(names)}"


def run_reference(args, world, rank):
    """The comparison arm: the CPU oracle, as it stands, on the host cores.
    Its input is encoded by the oracle itself, so this process loads no
    library of the GPU path."""
    if rank != 0:
        return
    units = workload_units(args.config, args.seed)
    if args.config == "build":
        return run_reference_build(args, world, units)
    if args.config in ("gemv", "gemm"):
        return run_reference_gemv(args, world, units)
    n_total = workload_elements(args.config)
    budget = args.cpu_budget_s / max(1, args.steps + args.warmup)
    # a step decodes as many leading elements as fit its share of the budget
    # (the bit-serial decoder runs at roughly 10 ns per element)
    # the stack's sample is taken from its first layers (94% of its elements
    # are in the 36 blocks), not from the 622M-element embedding, whose
    # generation on the host would take longer than the sample itself
    sample_units = units[1:-1] + [units[0], units[-1]] if args.config == "stack" else units
    hosts, encoded = _oracle_prefix_formats(sample_units, int(budget / 8e-9) + 1,
                                            args.chunk_bytes, args.threads_per_block)
    for _ in range(args.warmup):
        _oracle_sample(hosts, budget)
    tot_done, tot_s, what = 0, 0.0, ""
    for _ in range(args.steps):
        d, s, what = _oracle_sample(hosts, budget)
        tot_done += d
        tot_s += s
    value = 2.0 * tot_done / tot_s / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * tot_s / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u32",
        "data": "synthetic (seeded; fp32 samples rounded to BF16 RNE)",
        "config": {"workload": WORKLOAD_NAMES[args.config], "tensors": len(units),
                   "elements": n_total, "chunk_bytes": args.chunk_bytes, "threads_per_block": args.threads_per_block,
                   "step": f"bounded sample of the workload, ~{budget:.3f} s of CPU work"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": what + " per step (single-threaded bit-serial C decode); "
                                   "input: " + encoded},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def _oracle_gemv_sample(hosts, shapes, x_rows, budget_s: float):
    """The oracle's product (bit-serial decode, float64 matmul) on leading
    rows of the workload's weights until the budget is spent; returns
    (weights applied, seconds, description)."""
    import oracle
    done, t_used, names = 0, 0.0, 0
    for h, (r, c), x in zip(hosts, shapes, x_rows):
        if t_used >= budget_s:
            break
        rows = int(min(r, h.n // c, max(1, (budget_s - t_used) / 20e-9 / c)))
        t = time.perf_counter()
        w, _, _ = oracle.decode(h.bitstream, h.code_lengths, h.sign_mantissa, rows * c)
        W = oracle.bf16_to_f64(w).reshape(rows, c)
        _ = oracle.bf16_to_f64(x).reshape(-1, c) @ W.T
        t_used += time.perf_counter() - t
        done += rows * c
        names += 1
    return done, t_used, f"{done} weights from the leading rows of {names} weight(s)"


def run_reference_gemv(args, world, units):
    """The comparison arm for the fused product: the oracle's decode and
    float64 product, as they stand, on bounded samples of the workload."""
    shapes = [(r, c) for _, r, c in workloads.BLOCK_SHAPES]
    budget = args.cpu_budget_s / max(1, args.steps + args.warmup)
    # leading rows of the weights, encoded by the oracle itself (this process
    # loads no library of the GPU path); the product runs at roughly 20 ns per
    # weight
    hosts, encoded = _oracle_prefix_formats(
        [(n, t, c) for (n, t), (_, c) in zip(units, shapes)], int(budget / 15e-9) + 1,
        args.chunk_bytes, args.threads_per_block)
    shapes = shapes[: len(hosts)]
    xs = [workloads.as_numpy_u16(workloads.gaussian_bf16(args.batch * c, 1.0, 77 + i))
          for i, (_, c) in enumerate(shapes)]
    n_total = workload_elements(args.config)
    for _ in range(args.warmup):
        _oracle_gemv_sample(hosts, shapes, xs, budget)
    tot_done, tot_s, what = 0, 0.0, ""
    for _ in range(args.steps):
        d, s_, what = _oracle_gemv_sample(hosts, shapes, xs, budget)
        tot_done += d
        tot_s += s_
    value = 2.0 * tot_done / tot_s / 1e9
    line = {
        "impl": "reference", "metric": GEMM_METRIC if args.config == "gemm" else GEMV_METRIC,
        "value": round(value, 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * tot_s / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u32+f64",
        "data": "synthetic (seeded; fp32 samples rounded to BF16 RNE)",
        "config": {"workload": WORKLOAD_NAMES[args.config], "tensors": len(units),
                   "elements": n_total, "batch": args.batch, "chunk_bytes": args.chunk_bytes,
                   "threads_per_block": args.threads_per_block,
                   "step": f"bounded sample of the workload, ~{budget:.1f} s of CPU work"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": what + " per step (bit-serial C decode, float64 product); "
                                   "input: " + encoded},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def run_reference_build(args, world, units):
    """The comparison arm for the builder: the oracle's encoder, as it
    stands, on bounded samples of the workload."""
    ws = [thunk("cpu") for _, thunk in units]
    n_total = sum(w.numel() for w in ws)
    budget = args.cpu_budget_s / max(1, args.steps + args.warmup)
    for _ in range(args.warmup):
        _oracle_encode_sample(ws, budget)
    tot_done, tot_s, what = 0, 0.0, ""
    for _ in range(args.steps):
        d, s_, what = _oracle_encode_sample(ws, budget)
        tot_done += d
        tot_s += s_
    value = 2.0 * tot_done / tot_s / 1e9
    line = {
        "impl": "reference", "metric": BUILD_METRIC, "value": round(value, 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * tot_s / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u32",
        "data": "synthetic (seeded; fp32 samples rounded to BF16 RNE)",
        "config": {"workload": WORKLOAD_NAMES[args.config], "tensors": len(units),
                   "elements": n_total, "chunk_bytes": 24, "threads_per_block": 256,
                   "step": f"bounded sample of the workload, ~{budget:.1f} s of CPU work"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": what + " per step (single-threaded C encoder)"},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


OFFLOAD_LAYERS = 8

WORKLOAD_NAMES = {
    "single": "single 1024x1024 N(0,0.02)",
    "block": "Qwen3-8B-shaped block (q,k,v,o,gate,up,down), 192,937,984 elems",
    "adversarial": "adversarial exponent mix, 64M elems",
    "fibonacci": "Fibonacci exponent counts (32-bit codewords), 14,930,351 elems",
    "embedding": "embedding 151936x4096 N(0,0.02), 622,329,856 elems",
    "stack": "36-layer Qwen3-8B-shaped stack + embedding + LM head, 8,190,427,136 elems",
    "gemv": "fused decode and matrix-vector product: Qwen3-8B-shaped block "
            "(q,k,v,o,gate,up,down), 192,937,984 weights, BF16 activations",
    "gemm": "fused decode and tensor-core matrix product: Qwen3-8B-shaped block "
            "(q,k,v,o,gate,up,down), 192,937,984 weights, BF16 activations",
    "build": "format builder on the GPU: Qwen3-8B-shaped block (q,k,v,o,gate,up,down) "
             "compressed from BF16 in HBM, 192,937,984 elems",
    "offload": f"{OFFLOAD_LAYERS} Qwen3-8B-shaped layers streamed from pinned host memory "
               f"(compressed, one host-to-device copy per layer), "
               f"{OFFLOAD_LAYERS * 192_937_984:,} elems",
}


DEFAULT_STEPS = {"stack": 200, "build": 20, "gemv": 200, "gemm": 200, "offload": 40}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 200 for the stack, 2000 for one tensor "
                         "or block, 20 for build, 200 for gemv, 40 for offload)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="stack", choices=sorted(WORKLOAD_NAMES))
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--chunk-bytes", type=int, default=24, choices=[4, 8, 16, 24],
                    help="bitstream bytes per chunk (C) of the compressed format")
    ap.add_argument("--threads-per-block", type=int, default=256, choices=[128, 256, 512],
                    help="chunks per format block (T) of the compressed format")
    ap.add_argument("--batch", type=int, default=1,
                    help="activation rows of the gemv workload (1-8)")
    ap.add_argument("--interleave", type=int, default=1,
                    help="gemv workload: rows interleaved per 16 columns in the fused "
                         "path's compressed weights (1: row-major)")
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--flush-l2", default="auto", choices=["auto", "on", "off"],
                    help="rewrite a buffer twice the size of L2 before every timed decode "
                         "step (auto: when one step's bytes fit in L2) and time each step "
                         "alone")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-counts", action="store_true",
                    help="decode without the format's chunk counts (count by decoding)")
    ap.add_argument("--no-clock-window", action="store_true",
                    help="skip the busy untimed loop before the timed region "
                         "(for profiler runs)")
    ap.add_argument("--host-build", action="store_true",
                    help="compress the workload with the host builder instead of the "
                         "device builder (same bytes)")
    args = ap.parse_args(argv)
    if args.steps is None:
        args.steps = DEFAULT_STEPS.get(args.config, 2000)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = setup_dist()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            if not torch.cuda.is_available():
                raise SystemExit("the b200 arm needs a CUDA device")
            if args.config == "offload":
                run_offload(args, world, rank, local)
            elif args.config == "build":
                run_build(args, world, rank, local)
            elif args.config in ("gemv", "gemm"):
                run_gemv(args, world, rank, local)
            else:
                run_b200(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
