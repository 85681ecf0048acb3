"""Benchmark of the paged-decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama8b]
    python bench.py --impl reference ...      # the fp64 CPU oracle, timed

One step = one decode iteration of a serving loop over the whole batch:
host slot assignment for one new token per request (C++ allocator),
copy-on-write copies if any, pa_reshape_and_cache of the new K/V, and
pa_decode (main kernel + split-K merge) over every request's cache.

Prints one JSON line.  ``value`` is KV-read GB/s of pa_decode's algorithmic
bytes (sum of L*2*Hkv*D*2 plus q/out/table bytes) over the device time of
the K timed steps with every input resident in HBM; ``e2e`` is the same
metric with each step's host allocator call, host->device copies of its
inputs from pinned memory and the device->host read of its output inside the
timed region.  Weak scaling over GPUs: every rank runs its own batch (its
own pool and allocator), no data-path collective.
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "paged-decode KV-read GB/s & % of HBM peak; decode seqs/s at Llama-3-8B shape"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "source": "fallback"}
INPUT_SETS = 4  # distinct q/k/v sets cycled through the steps
SPEC_HBM_GBS = 8000.0  # B200 data-sheet HBM3e bandwidth


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "paged_decode_traffic.json")
DECODE_SOURCES = ("paged_kv_cache_354_b200/csrc/pa_decode.cu", "paged_kv_cache_354_b200/csrc/pa_device.cuh",
                  "paged_kv_cache_354_b200/csrc/pa_decode_common.cuh", "paged_kv_cache_354_b200/csrc/pa_decode_tc.cu",
                  "paged_kv_cache_354_b200/csrc/pa_tcgen05.cuh")


def decode_source_digest():
    h = hashlib.sha256()
    for rel in DECODE_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def captured_traffic(workload, variant, partition_tokens):
    """DRAM bytes per decode launch from the committed ncu capture, or None
    when there is none for this configuration or the kernel changed since."""
    try:
        with open(TRAFFIC_FILE) as f:
            entry = json.load(f).get(f"{workload}/{variant}/{partition_tokens}")
    except Exception:
        return None
    if not entry or entry.get("source_sha256") != decode_source_digest():
        return None
    return entry["dram_bytes_per_launch"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "source": "measured"}
    except Exception:
        return dict(PEAKS_FALLBACK)


# --------------------------------------------------------------------------
# clocks during the timed region (NVML, polled from a thread)
# --------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index, period_s=0.002):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self._stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _poll(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(self.period)

    def sample(self):
        if self.nv is None:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for mask, name in self.REASONS.items():
                if bits & mask and name != "gpu_idle":
                    self.reasons.add(name)
        except Exception:
            pass

    def __enter__(self):
        self.sample()
        self.t = threading.Thread(target=self._poll, daemon=True)
        self.t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------
# workload state
# --------------------------------------------------------------------------
def decode_bytes(lens, hq, hkv, d, bs):
    lens = np.asarray(lens, dtype=np.int64)
    kv = int(lens.sum()) * 2 * hkv * d * 2
    qo = 2 * len(lens) * hq * d * 2
    tables = int((-(-lens // bs)).sum()) * 4 + len(lens) * 4
    return kv + qo + tables, kv


L2_BYTES = 126e6  # B200 L2


def l2_note(plan_step, kv_logical, cache):
    """How the timed steps stand to the L2 (no flush between steps): the K/V
    a step reads, logically and as distinct physical blocks."""
    _, _, tables, lens = plan_step
    nblk = -(-np.asarray(lens, dtype=np.int64) // cache.bs)
    used = np.unique(np.concatenate([t[:n] for t, n in zip(tables, nblk)]))
    distinct = len(used) * 2 * cache.hkv * cache.bs * cache.d * 2
    if distinct > L2_BYTES:
        return (f"inputs larger than L2, no flush: K/V per step {kv_logical / 1e6:.0f} MB "
                f"({distinct / 1e6:.0f} MB distinct) > 126 MB")
    if kv_logical > L2_BYTES:
        return (f"K/V per step {kv_logical / 1e6:.0f} MB logical but {distinct / 1e6:.0f} MB distinct "
                f"(shared blocks): blocks read again within a step or the next may come from L2; no flush")
    return (f"inputs fit in L2 ({kv_logical / 1e6:.1f} MB), no flush: a launch-bound workload, "
            f"not a bandwidth measurement")


def workload_l2(p):
    """Whether the workload's K/V of one step exceeds the L2 (no flush is
    used between steps): from its tables as the decode steps start (the
    beams' divergent tokens appended), so both arms print the same
    statement."""
    from paged_kv_cache_354_b200 import PaAlloc

    s = p.shape
    alloc = PaAlloc(p.num_blocks, s.block_size, p.initial_order)
    ids = workloads.populate(alloc, p)
    if p.name == "beam":
        alloc.append_batch(ids, p.append_tokens)
    tables, lens = workloads.block_tables(alloc, ids)
    nblk = -(-np.asarray(lens, dtype=np.int64) // s.block_size)
    per_block = 2 * s.num_kv_heads * s.block_size * s.head_dim * 2
    logical = int(nblk.sum()) * per_block
    distinct = len(np.unique(np.concatenate([t[:n] for t, n in zip(tables, nblk)]))) * per_block
    if distinct > L2_BYTES:
        return f"inputs larger than L2 ({distinct / 1e6:.0f} MB of K/V blocks > 126 MB), no flush"
    if logical > L2_BYTES:
        return (f"{logical / 1e6:.0f} MB of K/V read per step from {distinct / 1e6:.0f} MB of shared blocks "
                f"(L2 126 MB), no flush: shared blocks may come from L2")
    return f"inputs fit in L2 ({logical / 1e6:.1f} MB), no flush: launch-bound, not a bandwidth measurement"


def workload_config(name, steps_total, world):
    """The workload fields of the JSON line's ``config``, shared by both arms."""
    p = workloads.plan(name, extra_tokens=steps_total + 1)
    s = p.shape
    batch = len(p.seq_lens) * (p.beams or 1)
    return {
        "workload": f"{name}: B{batch} Hq{s.num_q_heads}/Hkv{s.num_kv_heads} D{s.head_dim} bs{s.block_size}",
        "batch": batch, "num_q_heads": s.num_q_heads, "num_kv_heads": s.num_kv_heads, "head_dim": s.head_dim,
        "block_size": s.block_size, "num_blocks": p.num_blocks,
        "parallelism": f"dp{world} (independent batches, no collective)",
        "l2": workload_l2(p),
    }


def build_cache(name, steps_total, rank, device, prefill=True, variant=0, partition_tokens=0):
    """Pool (seeded bf16 N(0,1)), allocator state and request ids of a workload.

    With ``prefill`` the beam workload's 256 divergent tokens per beam are
    appended (copy-on-write + cache write) before the decode loop starts.
    """
    import torch

    from paged_kv_cache_354_b200.engine import PagedDecodeCache

    p = workloads.plan(name, extra_tokens=steps_total + 1)
    s = p.shape
    lens0 = np.asarray(p.seq_lens, dtype=np.int64)
    max_len = int(lens0.max()) + (p.prefix_len and 256) + steps_total + 2
    batch = len(lens0) * (p.beams or 1)
    cache = PagedDecodeCache(p.num_blocks, s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size,
                             batch, max_len, initial_order=p.initial_order, device=device,
                             partition_tokens=partition_tokens, variant=variant, staging_sets=INPUT_SETS)
    gen = torch.Generator(device=device)
    gen.manual_seed(workloads.seed_of(name) * 1000 + rank)
    cache.pool.copy_(torch.randn(cache.pool.shape, generator=gen, device=device,
                                 dtype=torch.float32).to(torch.bfloat16))
    ids = workloads.populate(cache.alloc, p)
    if prefill and p.name == "beam":
        beam_prefill(p, cache, ids, gen, device)
    return p, cache, ids, gen


def beam_prefill(p, cache, ids, gen, device):
    """Append each beam's divergent tokens: allocator, copy_blocks, cache write.

    Returns (slots, pairs, k, v) as used, for an independent replay."""
    import torch

    from paged_kv_cache_354_b200 import pa_copy_blocks, pa_reshape_and_cache

    s = p.shape
    slots, pairs = cache.alloc.append_batch(ids, p.append_tokens, as_numpy=True)
    k = torch.randn((len(slots), s.num_kv_heads, s.head_dim), generator=gen, device=device).bfloat16()
    v = torch.randn((len(slots), s.num_kv_heads, s.head_dim), generator=gen, device=device).bfloat16()
    pa_copy_blocks(cache.pool, torch.as_tensor(pairs, device=device))
    pa_reshape_and_cache(k, v, cache.pool, torch.as_tensor(slots, device=device))
    return slots, pairs, k, v


def make_inputs(cache, batch, gen, device):
    import torch

    qs = [torch.randn((batch, cache.hq, cache.d), generator=gen, device=device).bfloat16()
          for _ in range(INPUT_SETS)]
    ks = [torch.randn((batch, cache.hkv, cache.d), generator=gen, device=device).bfloat16()
          for _ in range(INPUT_SETS)]
    vs = [torch.randn((batch, cache.hkv, cache.d), generator=gen, device=device).bfloat16()
          for _ in range(INPUT_SETS)]
    return qs, ks, vs


# --------------------------------------------------------------------------
# the GPU arm
# --------------------------------------------------------------------------
def combine_ranks(times_ms, totals, device, world):
    """Whole-job figures: the max of every rank's times, the sum of their work.

    Works on any process group backend (NCCL on the GPUs, gloo in the CPU
    tests); with one rank it returns the inputs."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(list(times_ms), device=device, dtype=torch.float64)
    w = torch.tensor(list(totals), device=device, dtype=torch.float64)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return tuple(t.tolist()) + tuple(w.tolist())


MIN_TIMED_S = 0.5  # device time each timed loop reaches (the clock record needs it)
OTHER_WORKLOADS = ("long", "beam", "mixed", "tiny")


def repeats_for(est_ms, units, min_s):
    """Repetitions of a loop of ``units`` items of ``est_ms`` each that reach
    ``min_s`` of device time."""
    if est_ms <= 0:
        return 1
    return max(1, int(math.ceil(min_s * 1e3 / (est_ms * units))))


def timed_ms(stream, fn):
    """Device time of ``fn``'s launches: CUDA events on the launching stream,
    synchronised on both sides."""
    import torch

    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def agree_max(x, device, world):
    """The largest of every rank's x (so all ranks repeat a loop equally often)."""
    import torch
    import torch.distributed as dist

    if world == 1:
        return x
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return int(t.item())


def device_arm(name, K, W, rank, device, world, variant=0, partition_tokens=0, min_s=MIN_TIMED_S):
    """Device-timed figures of one workload, every input resident in HBM.

    Steps: W warm-up steps, then the same K steps (copy-on-write copies, the
    fused cache write + decode + merge of one new token per request),
    recorded once as a CUDA graph and replayed R times so the timed region
    holds at least ``min_s`` of device time.  Decode alone: K back-to-back
    pa_decode calls (main kernel + merge) on the last step's inputs, as a
    graph replayed likewise.  Clocks are sampled over both timed loops."""
    import torch
    import torch.distributed as dist

    p, cache, ids, gen = build_cache(name, steps_total(W, K), rank, device, variant=variant,
                                     partition_tokens=partition_tokens)
    batch = len(ids)
    qs, ks, vs = make_inputs(cache, batch, gen, device)
    out = torch.empty_like(qs[0])
    stream = torch.cuda.current_stream()
    plans = [cache.plan_append(ids) for _ in range(W + K)]
    d_slots = [torch.as_tensor(pl[0], device=device) for pl in plans]
    d_pairs = [torch.as_tensor(pl[1].reshape(-1, 2), device=device) for pl in plans]
    d_tables = [torch.as_tensor(pl[2], device=device) for pl in plans]
    d_lens = [torch.as_tensor(pl[3], device=device) for pl in plans]
    step_bytes = [decode_bytes(pl[3], cache.hq, cache.hkv, cache.d, cache.bs) for pl in plans]

    def dev_step(i):
        j = i % INPUT_SETS
        cache.run(qs[j], ks[j], vs[j], out, d_slots[i], d_tables[i], d_lens[i], d_pairs[i])

    last = W + K - 1

    def decode_once(i):
        cache.decode(qs[i % INPUT_SETS], out, d_tables[last], d_lens[last])

    # W warm-up steps launched one by one, then the K timed steps (and K
    # decode-only calls) recorded once as CUDA graphs: a replay runs every
    # kernel of the K steps with no host launch work between them
    for i in range(W):
        dev_step(i)
    for i in range(3):
        decode_once(i)
    torch.cuda.synchronize()

    def record(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g

    g_steps = record(lambda: [dev_step(i) for i in range(W, W + K)])
    g_dec = record(lambda: [decode_once(i) for i in range(K)])
    est_step = timed_ms(stream, g_steps.replay) / K
    est_dec = timed_ms(stream, g_dec.replay) / K
    R = agree_max(repeats_for(est_step, K, min_s), device, world)
    Rd = agree_max(repeats_for(est_dec, K, min_s), device, world)
    if world > 1:
        dist.barrier()
    with ClockSampler(device.index) as clocks:
        step_ms = timed_ms(stream, lambda: [g_steps.replay() for _ in range(R)])
        dec_ms = timed_ms(stream, lambda: [g_dec.replay() for _ in range(Rd)])
    if world > 1:
        dist.barrier()
    merge = 1 if (cache.schedule == "balanced" or cache.num_partitions > 1) else 0
    return {
        "p": p, "cache": cache, "ids": ids, "gen": gen, "qs": qs, "ks": ks, "vs": vs, "out": out,
        "plans": plans, "step_bytes": step_bytes, "R": R, "Rd": Rd,
        "step_ms": step_ms, "steps_timed": R * K,
        "bytes_timed": R * sum(b for b, _ in step_bytes[W:]),
        "kv_timed": R * sum(kv for _, kv in step_bytes[W:]),
        "decode_ms": dec_ms / (Rd * K), "decode_bytes": step_bytes[last][0],
        "launches": R * sum(cache.launches_per_step(len(pl[1])) for pl in plans[W:]),
        "decode_launches": Rd * K * (1 + merge),
        "clocks": clocks.summary(),
    }


E2E_BLOCK = 10  # steps per block; blocks of the two output paths alternate


def e2e_arm(arm, K, W, device, world):
    """End to end through the engine, for both ways the output can reach
    the host.  Per step the host allocator writes the step's metadata into a
    pinned staging buffer that already holds the step's q/k/v; one CUDA
    graph copies it to the device and runs the fused cache write + decode +
    merge, whose kernels either store the output straight into pinned host
    memory ("zero_copy") or write it on the device for a D2H copy at the end
    of the graph ("copy"); the allocator work for step i+1 runs on the host
    while the GPU works on step i; the host waits for step i's output before
    going on.  One timed loop of 2K steps runs blocks of E2E_BLOCK steps of
    each path in turn (so both see the same lengths), a CUDA event at every
    block boundary; returns {path: (ms, bytes)} over its K steps and the H2D
    and D2H bytes per step."""
    import torch
    import torch.distributed as dist

    cache, ids, out = arm["cache"], arm["ids"], arm["out"]
    stream = torch.cuda.current_stream()
    for j in range(INPUT_SETS):
        cache.staged("q", j).copy_(arm["qs"][j].cpu())
        cache.staged("k", j).copy_(arm["ks"][j].cpu())
        cache.staged("v", j).copy_(arm["vs"][j].cpu())
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_lens = []
    pending = {}

    def e2e_step(i, zero_copy):
        # step i's metadata was staged in buffer j during step i-1
        j = i % INPUT_SETS
        cache.replay_step(j, pending.pop(i), zero_copy)  # upload, decode, output to the host: one graph
        e2e_lens.append(cache.staged("lens", j).numpy().copy())  # bookkeeping while the GPU works
        pending[i + 1] = cache.host_step(ids, (i + 1) % INPUT_SETS)
        stream.synchronize()  # the step's result is on the host

    cache.host_step(ids, 0)  # one eager step, then record the graphs on its staged data
    cache.upload(0)
    cache.capture(out)
    cache.capture_steps(out, h_out, zero_copy=False)
    cache.capture_steps(out, h_out, zero_copy=True)
    pending[0] = cache.host_step(ids, 0)
    for i in range(2 * W):
        e2e_step(i, i % 2 == 0)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    blocks = []  # (path, first step, steps)
    done = {"zero_copy": 0, "copy": 0}
    while done["zero_copy"] < K or done["copy"] < K:
        for path in ("zero_copy", "copy"):
            n = min(E2E_BLOCK, K - done[path])
            if n > 0:
                blocks.append((path, 2 * W + done["zero_copy"] + done["copy"], n))
                done[path] += n
    events = [torch.cuda.Event(enable_timing=True) for _ in range(len(blocks) + 1)]
    e2e_lens.clear()
    torch.cuda.synchronize()
    for b, (path, first, n) in enumerate(blocks):
        events[b].record(stream)
        for i in range(first, first + n):
            e2e_step(i, path == "zero_copy")
    events[-1].record(stream)
    torch.cuda.synchronize()
    results = {"zero_copy": [0.0, 0], "copy": [0.0, 0]}
    for b, (path, first, n) in enumerate(blocks):
        results[path][0] += events[b].elapsed_time(events[b + 1])
        lens_b = e2e_lens[first - 2 * W:first - 2 * W + n]
        results[path][1] += sum(decode_bytes(ln, cache.hq, cache.hkv, cache.d, cache.bs)[0] for ln in lens_b)
    return {k: tuple(v) for k, v in results.items()}, cache.stage_bytes, int(h_out.nbytes)


def steps_total(W, K):
    """Tokens each request may gain over a run (device arm, the e2e loop
    over both output paths, slack): sizes the workload's pool, so both arms'
    configs use it."""
    return 3 * (W + K) + 8


def workload_entry(name, arm, peaks, world):
    """One workload's device-timed figures for the JSON line."""
    step_gbs = arm["bytes_timed"] / (arm["step_ms"] * 1e-3) / 1e9
    dec_gbs = arm["decode_bytes"] / (arm["decode_ms"] * 1e-3) / 1e9
    cache = arm["cache"]
    return {
        "workload": workload_config(name, 0, world)["workload"],
        "step_gbs": round(step_gbs, 2),
        "step_ms": round(arm["step_ms"] / arm["steps_timed"], 5),
        "step_frac_of_hbm_peak": round(step_gbs / peaks["hbm_gbs"], 4),
        "decode_gbs": round(dec_gbs, 2),
        "decode_ms": round(arm["decode_ms"], 5),
        "decode_frac_of_hbm_peak": round(dec_gbs / peaks["hbm_gbs"], 4),
        "decode_seqs_per_s": round(len(arm["ids"]) / (arm["step_ms"] / arm["steps_timed"] * 1e-3), 1),
        "steps_timed": arm["steps_timed"],
        "decode_launches_timed": arm["Rd"],
        "decode_schedule": (f"balanced persistent: {cache.num_partitions} CTAs"
                            if cache.schedule == "balanced" else
                            f"per-partition grid: {cache.num_partitions} partitions"),
        "l2": l2_note(arm["plans"][-1], arm["step_bytes"][-1][1], cache),
        "clocks": arm["clocks"],
    }


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(device)
    from paged_kv_cache_354_b200 import pa_device_error

    K, W = args.steps, args.warmup
    variant = {"auto": 0, "cuda_core": 1, "mma": 2}[args.variant]
    arm = device_arm(args.workload, K, W, rank, device, world, variant, args.partition_tokens, args.min_seconds)
    e2e, stage_bytes, d2h_bytes = e2e_arm(arm, K, W, device, world)
    dev_err = pa_device_error()

    # ---- max over ranks (times), sum over ranks (work)
    (step_ms, e2e_ms, e2e_copy_ms, decode_ms, bytes_all, e2e_bytes_all, e2e_copy_bytes_all,
     kv_all) = combine_ranks([arm["step_ms"], e2e["zero_copy"][0], e2e["copy"][0], arm["decode_ms"]],
                             [arm["bytes_timed"], e2e["zero_copy"][1], e2e["copy"][1], arm["kv_timed"]],
                             device, world)
    cache, steps_timed = arm["cache"], arm["steps_timed"]
    batch = len(arm["ids"])
    summary = {
        "mean_seq_len": round(float(np.mean(arm["plans"][W][3])), 1),
        "decode_schedule": (f"balanced persistent: {cache.num_partitions} CTAs"
                            if cache.schedule == "balanced" else
                            f"per-partition grid: {cache.num_partitions} partitions"),
        "l2": l2_note(arm["plans"][W], arm["step_bytes"][W][1], cache),
        "variant": args.variant,
    }
    launches, dec_launches, decode_bytes_last = arm["launches"], arm["decode_launches"], arm["decode_bytes"]
    clocks = arm["clocks"]
    del arm, cache
    torch.cuda.empty_cache()

    # ---- wide GQA groups (the tcgen05 consumer) against mma.sync on the same
    # lengths, and multi-token decode with T = 1, 2, 4 query tokens: decode +
    # merge back to back (one GPU, default workload only)
    wide, multi = [], []
    if world == 1 and args.workload == "llama8b" and not args.no_workloads:
        peaks = load_peaks()
        for row in variant_times(iters=20, hkvs=[(8, 128)], groups=[16, 32]):
            row.pop("cuda_core_us", None)
            row.pop("cuda_core_gbs", None)
            row["tcgen05_frac_of_hbm_peak"] = round(row["tcgen05_gbs"] / peaks["hbm_gbs"], 4)
            row["default_variant"] = "tcgen05"
            wide.append(row)
        multi = list(multi_token_times())

    # ---- the other workloads, device-timed (one GPU, default workload only)
    others = {}
    if world == 1 and args.workload == "llama8b" and not args.no_workloads:
        peaks = load_peaks()
        for name in OTHER_WORKLOADS:
            o = device_arm(name, K, W, rank, device, world, min_s=args.min_seconds / 2)
            others[name] = workload_entry(name, o, peaks, world)
            del o
            torch.cuda.empty_cache()
        dev_err |= pa_device_error()

    if rank == 0:
        peaks = load_peaks()
        gbs = bytes_all / (step_ms * 1e-3) / 1e9
        achieved = decode_bytes_last / (decode_ms * 1e-3) / 1e9
        line = {
            "metric": METRIC,
            "value": round(gbs, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": K,
            "warmup": W,
            "ms_per_step": round(step_ms / steps_timed, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded bf16 N(0,1) q/K/V; seeded lengths and shuffled block pool)",
            "config": workload_config(args.workload, steps_total(W, K), world),
            "run": {**summary, "timed_repeats": steps_timed // K, "steps_timed": steps_timed,
                    "timing": "the K steps (copy-on-write copies, fused cache write + decode + merge) recorded "
                              "once as a CUDA graph and replayed timed_repeats times back to back; one pair of "
                              "CUDA events around all of them; ms_per_step = their device time / steps_timed"},
            "decode_seqs_per_s": round(batch * world * steps_timed / (step_ms * 1e-3), 1),
            "frac_of_hbm_peak": round(gbs / world / peaks["hbm_gbs"], 4),
            # against the B200 data-sheet bandwidth (8 TB/s) rather than the measured copy
            "frac_of_spec_hbm": round(gbs / world / SPEC_HBM_GBS, 4),
            "spec_hbm_gbs": SPEC_HBM_GBS,
            "roofline": {
                "bound": "hbm",
                "kernel": "pa_decode (main + split-K merge), back-to-back launches",
                "achieved": round(achieved, 2),
                "peak": peaks["hbm_gbs"],
                "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "peak_source": peaks["source"],
                "traffic": captured_traffic(args.workload, args.variant, args.partition_tokens),
                "traffic_note": "dram read+write per launch of the main decode kernel from the committed "
                                "ncu capture; null unless that capture was taken on the current decode sources",
                "launches_timed": dec_launches,
            },
            "e2e": {
                "value": round(e2e_bytes_all / (e2e_ms * 1e-3) / 1e9, 2),
                "unit": "GB/s",
                "h2d_bytes_per_step": int(stage_bytes),
                "d2h_bytes_per_step": int(d2h_bytes),
                "ms_per_step": round(e2e_ms / K, 5),
                "steps_timed": K,
                "path": "per step: one CUDA graph holding the H2D copy of a pinned staging buffer "
                        "(metadata from the C++ allocator + the step's q/k/v) and the fused cache write + "
                        "decode + merge, whose kernels store the output rows straight into pinned host "
                        "memory across PCIe as they finish (zero-copy); then a sync; the allocator work "
                        "for the next step runs on the host while the GPU works",
                "with_d2h_copy": {
                    "value": round(e2e_copy_bytes_all / (e2e_copy_ms * 1e-3) / 1e9, 2),
                    "ms_per_step": round(e2e_copy_ms / K, 5),
                    "path": "the same steps with the output written on the device and one D2H copy "
                            "of it at the end of the graph",
                },
                "timing": f"one loop of 2K steps, blocks of {E2E_BLOCK} steps of each output path in "
                          "turn (equal lengths for both), CUDA events at the block boundaries; each "
                          "path's ms_per_step = its blocks' time / K",
            },
            "gpu_launches": launches * world,  # the step loop (value's timed region), every rank
            "clocks": clocks,
            "device_error_word": dev_err,
        }
        if others:
            line["workloads"] = others
        if wide:
            line["wide_columns"] = wide
        if multi:
            line["multi_token"] = multi
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------------------
# the oracle on host cores
# --------------------------------------------------------------------------
class OracleRunner:
    """The fp64 oracle decoding whole requests of a workload, one at a time.

    The requests' tables come from the oracle's own allocator model; their
    K/V blocks and queries are seeded bf16 N(0,1), built on the host outside
    the timed part.  Only the oracle decode call is timed.  ``first`` offsets
    the runner's walk through the requests (parallel runners decode
    different requests).
    """

    def __init__(self, name, first=0):
        from oracle.block_allocator import BlockAllocator

        self.name = name
        p = workloads.plan(name)
        self.shape = p.shape
        self.alloc = BlockAllocator(p.num_blocks, p.shape.block_size, p.initial_order)
        self.ids = workloads.populate(self.alloc, p)
        self.order = np.random.default_rng(workloads.seed_of(name)).permutation(len(self.ids))
        self.next = first

    def _request(self):
        s = self.shape
        sid = self.ids[self.order[self.next % len(self.ids)]]
        self.next += 1
        table = self.alloc.block_table(sid)
        n = self.alloc.seq_len(sid)
        blocks = workloads.bf16_normal((len(table), 2, s.num_kv_heads, s.block_size, s.head_dim),
                                       seed=int(sid) + 1).double().numpy()
        q = workloads.bf16_normal((1, s.num_q_heads, s.head_dim), seed=int(sid) + 7).double().numpy()
        return q, blocks, np.arange(len(table))[None, :], n

    def run(self, budget_s, min_requests=1):
        """Decode requests until budget_s of oracle time; (kv_bytes, requests, seconds)."""
        from threadpoolctl import threadpool_limits

        from oracle import paged_attention as opa

        s = self.shape
        kv_bytes, done, elapsed = 0, 0, 0.0
        with threadpool_limits(1):
            while done < min_requests or elapsed < budget_s:
                q, blocks, table, n = self._request()
                t0 = time.perf_counter()
                opa.decode(q, blocks, table, np.array([n]), 1.0 / math.sqrt(s.head_dim))
                elapsed += time.perf_counter() - t0
                kv_bytes += n * 2 * s.num_kv_heads * s.head_dim * 2
                done += 1
        return kv_bytes, done, elapsed


_ORACLE_BARRIER = None


def _oracle_pool_init(barrier):
    global _ORACLE_BARRIER
    _ORACLE_BARRIER = barrier


def _oracle_worker(job):
    """One host core's share: build the runner, wait for every worker, then
    warmup + steps rounds of per_step seconds; (kv_bytes, requests, seconds)
    summed over the timed rounds."""
    import torch

    # one core per worker: torch's own thread pool generates the requests'
    # inputs and is not covered by the BLAS limit inside OracleRunner.run
    torch.set_num_threads(1)
    name, first, per_step, warmup, steps = job
    runner = OracleRunner(name, first)
    _ORACLE_BARRIER.wait(timeout=600)  # all workers start together (torch imports first)
    for _ in range(warmup):
        runner.run(per_step)
    kv, n, el = 0, 0, 0.0
    for _ in range(steps):
        a, b, c = runner.run(per_step)
        kv, n, el = kv + a, n + b, el + c
    return kv, n, el


def oracle_all_cores(name, per_step, warmup=0, steps=1):
    """The oracle on every host core this process may use: one spawned
    worker per core (one NumPy thread each), each decoding its own requests
    for the same rounds.  Returns (kv_bytes, requests, seconds, workers): the
    bytes and requests summed over the workers, the seconds the slowest
    worker's oracle time."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor

    workers = len(os.sched_getaffinity(0))
    ctx = mp.get_context("spawn")  # never fork: a GPU context may exist in this process
    barrier = ctx.Barrier(workers)
    # a worker that dies breaks the executor (an error, not a wait); the
    # barrier and the result wait are bounded too
    limit = 900 + 4 * per_step * (warmup + steps)
    with ProcessPoolExecutor(workers, mp_context=ctx, initializer=_oracle_pool_init, initargs=(barrier,)) as ex:
        futs = [ex.submit(_oracle_worker, (name, w, per_step, warmup, steps)) for w in range(workers)]
        res = [f.result(timeout=limit) for f in futs]
    kv = sum(r[0] for r in res)
    n = sum(r[1] for r in res)
    el = max(r[2] for r in res)
    return kv, n, el, workers


def describe_oracle(name, requests, workers):
    s = workloads.plan(name).shape
    return (f"{requests} whole requests of the {name} workload (all {s.num_q_heads} query heads each), fp64 "
            f"NumPy oracle, {workers} processes x 1 thread")


def cpu_baseline(name, budget_s):
    kv, n, el, workers = oracle_all_cores(name, budget_s)
    return {"value": round(kv / el / 1e9, 4), "unit": "GB/s", "cores": workers, "kind": "oracle",
            "sample": describe_oracle(name, n, workers), "seqs_per_s": round(n / el, 3),
            "host_cores_available": len(os.sched_getaffinity(0))}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step = args.cpu_seconds / max(1, args.steps + args.warmup)
    kv, n, el, workers = oracle_all_cores(args.workload, per_step, args.warmup, args.steps)
    value = kv / el / 1e9
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * el / args.steps, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded bf16 N(0,1) K/V and q, upcast to f64)",
        "config": workload_config(args.workload, steps_total(args.warmup, args.steps),
                                  int(os.environ.get("WORLD_SIZE", "1"))),
        "run": {"note": "every host core runs the oracle on its own requests; each step decodes at least "
                        "one whole request per core; ms_per_step is the slowest core's oracle time / steps"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": workers, "kind": "oracle",
                         "sample": describe_oracle(args.workload, n, workers)},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# studies of the pages' context claims (not the headline line)
# --------------------------------------------------------------------------
MAX_CONTEXT = {"tiny": 65, "llama8b": 4096, "long": 32768, "beam": 2306, "mixed": 8192}


def study_memory_waste():
    """Slots held vs tokens stored: contiguous max-context reservation against
    the paged allocator's actual state, per workload (host only).

    "Paged attention in LLMs", sections "Why the memory gets wasted" and "Why
    this helps so much"; the quiz page's table row "Wasted memory".  The
    contiguous layout reserves the workload's maximum context per request and
    stores every beam's copy of a shared prefix; the paged numbers come from
    the C++ allocator after the workload's events.
    """
    import paged_kv_cache_354_b200 as pk

    for name in workloads.NAMES:
        p = workloads.plan(name)
        a = pk.PaAlloc(p.num_blocks, p.shape.block_size, p.initial_order)
        ids = workloads.populate(a, p)
        if p.append_tokens:
            a.append_batch(ids, p.append_tokens)
        st = a.stats()
        bs = p.shape.block_size
        reserved = len(ids) * MAX_CONTEXT[name]
        line = {
            "study": "memory_waste", "workload": name, "requests": len(ids), "block_size": bs,
            "tokens": st["tokens"],
            "contiguous_reserved_slots": reserved,
            "contiguous_waste_frac": round(1 - st["tokens"] / reserved, 4),
            "paged_logical_slots": st["logical_slots"],
            "paged_internal_waste_frac": round(1 - st["tokens"] / st["logical_slots"], 4),
            "paged_physical_slots": st["physical_blocks"] * bs,
            "paged_physical_over_tokens": round(st["physical_blocks"] * bs / st["tokens"], 4),
            "max_internal_waste_per_request": bs - 1,
        }
        print(json.dumps(line), flush=True)


def study_page_table(iters=30, names=("llama8b", "mixed", "long")):
    """pa_decode on the workload's scattered block tables vs on identity
    tables (each request's blocks physically consecutive, same lengths and
    pool format), and vs pa_decode_contiguous on a contiguous reservation per
    request (no block table at all; the quiz page's "Naive contiguous
    allocation"): the cost the block-table indirection adds to the kernel
    (quiz page, comparison table row "Kernel overhead": small, <5%)."""
    import torch

    import paged_kv_cache_354_b200 as pk
    from paged_kv_cache_354_b200.engine import PagedDecodeCache

    dev = torch.device("cuda", torch.cuda.current_device())
    for name in names:
        p = workloads.plan(name)
        s = p.shape
        res = {}
        for layout, order in (("scattered", p.initial_order), ("identity", np.arange(p.num_blocks))):
            cache = PagedDecodeCache(p.num_blocks, s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size,
                                     len(p.seq_lens), int(max(p.seq_lens)) + 2, initial_order=order, device=dev)
            gen = torch.Generator(device=dev)
            gen.manual_seed(workloads.seed_of(name))
            cache.pool.copy_(torch.randn(cache.pool.shape, generator=gen, device=dev).bfloat16())
            if layout == "scattered":
                ids = workloads.populate(cache.alloc, p)
            else:  # requests filled in order from an untouched pool (no churn)
                ids = list(range(len(p.seq_lens)))
                for sid in ids:
                    cache.alloc.add_seq(sid)
                    cache.alloc.append(sid, int(p.seq_lens[sid]))
            tables, lens = cache.alloc.block_tables(ids, cache.max_blocks)
            if layout == "identity":
                flat = np.concatenate([t[: -(-int(n) // s.block_size)] for t, n in zip(tables, lens)])
                assert np.array_equal(np.diff(flat), np.ones(len(flat) - 1)), "identity layout not consecutive"
            q = torch.randn((len(ids), s.num_q_heads, s.head_dim), generator=gen, device=dev).bfloat16()
            out = torch.empty_like(q)
            d_t, d_l = torch.as_tensor(tables, device=dev), torch.as_tensor(lens, device=dev)
            for _ in range(3):
                cache.decode(q, out, d_t, d_l)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(iters):
                cache.decode(q, out, d_t, d_l)
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) / iters * 1e3
            nbytes = decode_bytes(lens, s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size)[0]
            res[layout] = (us, nbytes / us / 1e3)
            del cache
            torch.cuda.empty_cache()
        # the same lengths in one contiguous run per request, 16-row tiles
        lens_c = np.asarray(p.seq_lens, dtype=np.int32)
        max_len = -(-int(lens_c.max()) // 16) * 16
        gen = torch.Generator(device=dev)
        gen.manual_seed(workloads.seed_of(name) + 1)
        kv = torch.randn((len(lens_c), 2, s.num_kv_heads, max_len, s.head_dim), generator=gen, device=dev,
                         dtype=torch.bfloat16)
        q = torch.randn((len(lens_c), s.num_q_heads, s.head_dim), generator=gen, device=dev).bfloat16()
        out = torch.empty_like(q)
        d_l = torch.as_tensor(lens_c, device=dev)
        ws = torch.empty(pk.pa_decode_contiguous_workspace_size(len(lens_c), s.num_q_heads, s.num_kv_heads,
                                                                 s.head_dim, max_len), dtype=torch.uint8, device=dev)
        scale = 1.0 / float(np.sqrt(s.head_dim))
        for _ in range(3):
            pk.pa_decode_contiguous(out, q, kv, d_l, scale, ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            pk.pa_decode_contiguous(out, q, kv, d_l, scale, ws)
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / iters * 1e3
        kv_bytes = int(lens_c.astype(np.int64).sum()) * 2 * s.num_kv_heads * s.head_dim * 2
        res["contiguous"] = (us, (kv_bytes + 2 * q.numel() * 2 + 4 * len(lens_c)) / us / 1e3)
        del kv
        torch.cuda.empty_cache()
        print(json.dumps({
            "study": "page_table_overhead", "workload": name,
            "scattered_us": round(res["scattered"][0], 2), "identity_us": round(res["identity"][0], 2),
            "contiguous_us": round(res["contiguous"][0], 2),
            "scattered_gbs": round(res["scattered"][1], 1), "identity_gbs": round(res["identity"][1], 1),
            "contiguous_gbs": round(res["contiguous"][1], 1),
            "overhead_frac": round(res["scattered"][0] / res["identity"][0] - 1, 4),
            "overhead_vs_contiguous_frac": round(res["scattered"][0] / res["contiguous"][0] - 1, 4),
            "paged_block_size": s.block_size, "contiguous_tile_rows": 16,
            "iters": iters}), flush=True)
    assert pk.pa_device_error() == 0


def multi_token_times(iters=30):
    """pa_decode_multi at the llama8b shape for T = 1, 2, 4 causal query
    tokens per request (speculative verification): KV bytes stay the same,
    the tensor-core tile widens from 4 to 16 (token, head) columns.  Yields
    one dict per T."""
    import torch

    import paged_kv_cache_354_b200 as pk

    dev = torch.device("cuda", torch.cuda.current_device())
    p, cache, ids, gen = build_cache("llama8b", 8, 0, dev)
    tables, lens = cache.alloc.block_tables(ids, cache.max_blocks)
    d_t, d_l = torch.as_tensor(tables, device=dev), torch.as_tensor(lens, device=dev)
    nbytes = decode_bytes(lens, cache.hq, cache.hkv, cache.d, cache.bs)[0]
    for T in (1, 2, 4):
        q = torch.randn((len(ids), T, cache.hq, cache.d), generator=gen, device=dev).bfloat16()
        out = torch.empty_like(q)
        ws = torch.empty(max(256, pk.pa_decode_multi_workspace_size(len(ids), T, cache.hq, cache.hkv, cache.d,
                                                                     cache.bs, cache.max_seq_len)),
                         dtype=torch.uint8, device=dev)

        def call():
            pk.pa_decode_multi(out, q, cache.pool, d_t, d_l, cache.max_seq_len, 1.0 / math.sqrt(cache.d), ws)

        for _ in range(3):
            call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            call()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / iters * 1e3
        extra_qo = 2 * len(ids) * (T - 1) * cache.hq * cache.d * 2
        yield {"workload": "llama8b", "query_tokens": T, "columns_per_kv_head": T * cache.hq // cache.hkv,
               "us": round(us, 2), "gbs": round((nbytes + extra_qo) / us / 1e3, 1),
               "frac_of_hbm_peak": round((nbytes + extra_qo) / us / 1e3 / load_peaks()["hbm_gbs"], 4),
               "tokens_per_s": round(len(ids) * T / us * 1e6, 1)}
    del cache
    torch.cuda.empty_cache()
    assert pk.pa_device_error() == 0


def study_multi_token(iters=30):
    for row in multi_token_times(iters):
        print(json.dumps({"study": "multi_token", **row}), flush=True)


def variant_times(iters=20, hkvs=None, groups=None, only=None):
    """The three consumers across GQA group sizes: pa_decode on the llama8b
    lengths and shuffled pool, Hkv in {8, 32}, head dim 128 and (Hkv 8) 64,
    groups 1, 2, 4, 8, 16, 32 -- mma.sync and tcgen05 for every group, CUDA
    cores for 1, 2, 4; CUDA events over back-to-back launches.  Yields one
    dict per (Hkv, head dim, group)."""
    import torch

    import paged_kv_cache_354_b200 as pk

    dev = torch.device("cuda", torch.cuda.current_device())
    p = workloads.plan("llama8b")
    gen = torch.Generator(device=dev)
    gen.manual_seed(workloads.seed_of("llama8b"))
    ws = torch.empty(64 << 20, dtype=torch.uint8, device=dev)
    for hkv, d in ((8, 128), (32, 128), (8, 64)):
        if hkvs and (hkv, d) not in hkvs:
            continue
        bs = 16
        pool = torch.randn((p.num_blocks, 2, hkv, bs, d), generator=gen, device=dev).bfloat16()
        alloc = pk.PaAlloc(p.num_blocks, bs, p.initial_order)
        ids = workloads.populate(alloc, p)
        tables, lens = alloc.block_tables(ids, -(-int(max(p.seq_lens)) // bs))
        d_t, d_l = torch.as_tensor(tables, device=dev), torch.as_tensor(lens, device=dev)
        for g in (1, 2, 4, 8, 16, 32):
            if groups and g not in groups:
                continue
            q = torch.randn((len(ids), hkv * g, d), generator=gen, device=dev).bfloat16()
            out = torch.empty_like(q)
            nbytes = decode_bytes(lens, hkv * g, hkv, d, bs)[0]
            res = {}
            for name, variant in (("mma", pk.PA_DECODE_MMA), ("cuda_core", pk.PA_DECODE_CUDA_CORE),
                                  ("tcgen05", pk.PA_DECODE_TCGEN05)):
                if (variant == pk.PA_DECODE_CUDA_CORE and g not in (1, 2, 4)) or (only and name != only):
                    continue

                def call():
                    pk.pa_decode(out, q, pool, d_t, d_l, int(lens.max()), 1.0 / math.sqrt(d), workspace=ws,
                                 variant=variant)

                for _ in range(3):
                    call()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(iters):
                    call()
                e1.record()
                torch.cuda.synchronize()
                res[name] = e0.elapsed_time(e1) / iters * 1e3
            yield {"workload": "llama8b lengths", "num_kv_heads": hkv, "head_dim": d, "group": g,
                   **{f"{k}_us": round(v, 1) for k, v in res.items()},
                   **{f"{k}_gbs": round(nbytes / v / 1e3, 1) for k, v in res.items()}, "iters": iters}
        del pool
        torch.cuda.empty_cache()
    assert pk.pa_device_error() == 0


def study_variants(iters=20, hkvs=None, groups=None, only=None):
    for row in variant_times(iters, hkvs, groups, only):
        print(json.dumps({"study": "variants", **row}), flush=True)


def study_read_bandwidth(iters=20):
    """What a plain contiguous read stream reaches on this GPU: torch's own
    bf16 sum (fp32 accumulate) over 2 GiB, for context beside the copy-based
    peak in MEASURED_PEAKS.json (which counts a read and a write per byte)."""
    import torch

    x = torch.empty(1024 ** 3, dtype=torch.bfloat16, device="cuda").normal_()
    for _ in range(3):
        torch.sum(x, dtype=torch.float32)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        torch.sum(x, dtype=torch.float32)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / iters
    print(json.dumps({"study": "read_bandwidth", "probe": "torch.sum bf16 -> fp32 over 2 GiB",
                      "gbs": round(x.numel() * 2 / ms / 1e6, 1), "ms": round(ms, 4),
                      "copy_peak_gbs": load_peaks()["hbm_gbs"]}), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama8b", choices=workloads.NAMES)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--variant", default="auto", choices=["auto", "mma", "cuda_core"],
                    help="decode consumer: auto (tensor cores for GQA groups >= 4), or forced")
    ap.add_argument("--study", choices=["memory-waste", "page-table", "multi-token", "read-bandwidth", "variants"],
                    help="print the study's JSON lines instead of the benchmark line")
    ap.add_argument("--study-workload", choices=["llama8b", "mixed", "long"], default=None,
                    help="page-table study: one workload only (default: all three)")
    ap.add_argument("--study-hkv", type=int, choices=[8, 32], default=None,
                    help="variants study: one KV-head count only (with --study-head-dim)")
    ap.add_argument("--study-head-dim", type=int, choices=[64, 128], default=128)
    ap.add_argument("--study-group", type=int, choices=[1, 2, 4, 8, 16, 32], default=None,
                    help="variants study: one GQA group only")
    ap.add_argument("--study-variant", choices=["mma", "cuda_core", "tcgen05"], default=None,
                    help="variants study: one consumer only")
    ap.add_argument("--study-iters", type=int, default=None, help="timed launches per study point")
    ap.add_argument("--partition-tokens", type=int, default=0,
                    help="0 = library's choice; -1 = balanced schedule; N > 0 = per-partition grid of "
                         "N-token partitions")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--min-seconds", type=float, default=MIN_TIMED_S,
                    help="device time each timed loop reaches (the K steps are repeated until it does)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the device-timed figures of the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.study == "memory-waste":
        study_memory_waste()
    elif args.study == "page-table":
        study_page_table(names=(args.study_workload,) if args.study_workload else ("llama8b", "mixed", "long"))
    elif args.study == "multi-token":
        study_multi_token()
    elif args.study == "read-bandwidth":
        study_read_bandwidth()
    elif args.study == "variants":
        study_variants(iters=args.study_iters or 20,
                       hkvs=[(args.study_hkv, args.study_head_dim)] if args.study_hkv else None,
                       groups=[args.study_group] if args.study_group else None, only=args.study_variant)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
