"""Benchmark of the paged decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the whole decode path over one batch: copy-on-write block
copies (when the step has any), the slot-mapped append of every sequence's new
token, and paged decode attention over the block tables.  Inputs sit in HBM when
the timed region starts; the KV bytes a step reads (about 1.2 GB for the default
workload) are far larger than the 126 MB L2, so no flush is needed between steps.

The metric is throughput in GB/s of algorithmic bytes: the K and V rows of every
context token, q and the output, block tables and lengths, plus the appended rows.
Whole-block over-reads and the context-split workspace traffic are not counted.
Sequences/s is reported beside it.

Under torchrun each rank runs its own batch (seed + rank) on its own GPU: the path
shards by sequence with no data exchange (weak scaling).  Timing is by CUDA events,
max over ranks.

--impl reference times the fp64 CPU oracle on the host cores instead (rank 0
only), on a bounded sample of sequences of the same workload per step.
"""
import argparse
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from paged_kv_cache_363_b200 import workloads as W  # noqa: E402

METRIC = "paged decode attention KV HBM GB/s (% of B200 peak) and sequences/sec"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2 ** 20


# ------------------------------------------------------------------ helpers shared with the tests

def rank_seed(seed, rank):
    """Each rank draws its own batch: same shapes and distributions, other values."""
    return int(seed) + 1000 * int(rank)


def reduce_max(x, device=None):
    """Max of a scalar over the ranks of the default process group (x itself if none)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


DECODE_SOURCES = ("pa_decode.cu", "pa_decode_common.cuh", "pa_decode_fma.cuh", "pa_decode_mma.cuh", "pa_ptx.cuh")
PREFILL_SOURCES = ("pa_prefill.cu", "pa_tcgen05.cuh", "pa_ptx.cuh")


def decode_source_hash(sources=None):
    """Hash of a kernel's code (ties a committed profile to the code it measured); the
    decode kernel's by default.  Comments and whitespace are left out, so rewording a
    comment keeps a profile valid; any change to the code does not."""
    import hashlib
    h = hashlib.sha256()
    for name in (DECODE_SOURCES if sources is None else sources):
        with open(os.path.join(ROOT, "paged_kv_cache_363_b200", "csrc", name)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        for line in text.splitlines():
            code = re.sub(r"//.*", "", line).split()
            if code:
                h.update((" ".join(code) + "\n").encode())
    return h.hexdigest()[:16]


def profiled_config(args):
    """True when this run's workload is the one the committed ncu summaries measured:
    the named workload at seed 0, automatic partitions, no overrides."""
    return args.seed == 0 and args.partition is None and not args.set


def profile_traffic(kernel, workload, sources=None):
    """dram bytes per launch from the committed ncu summary for this kernel and workload,
    if its recorded source hash still matches the kernel's sources; else None."""
    path = os.path.join(ROOT, "profiles", "%s_%s.md" % (kernel, workload))
    try:
        fields = {}
        with open(path) as f:
            for line in f:
                if ":" in line and line.startswith("- "):
                    k, v = line[2:].split(":", 1)
                    fields[k.strip()] = v.strip().strip("`")
        if (fields.get("source_sha256_16") or "").split(" ")[0] != decode_source_hash(sources):
            return None
        return float(fields["traffic_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while the timed region runs."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index, interval=0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.interval = interval
        self._stop = threading.Event()
        self._thread = None
        self.h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = int(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        except Exception:
            self.h = None

    def _sample(self):
        nv = self.nv
        self.samples.append(int(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)))
        try:
            bits = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
        except Exception:
            bits = int(nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h))
        for b, name in self.REASONS.items():
            if bits & b:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            time.sleep(self.interval)

    def __enter__(self):
        if self.h is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


L2_BYTES = 126e6


def l2_note(batch, logical_bytes):
    """How the timed steps stand to the 126 MB L2: the distinct K/V blocks a step reads."""
    wl = batch.wl
    elt = 4 if wl.dtype == "f32" else 2
    used = np.unique(batch.block_tables.cpu().numpy())
    unique = int((used >= 0).sum()) * wl.block_size * 2 * wl.num_kv_heads * wl.head_dim * elt
    if unique >= L2_BYTES:
        return "inputs larger than L2: %.0f MB of distinct KV per step (%.0f MB logical) vs 126 MB" % (
            unique / 1e6, logical_bytes / 1e6)
    return ("distinct KV %.0f MB per step fits the 126 MB L2 (shared blocks are re-read from L2); value counts "
            "the %.0f MB of logical bytes" % (unique / 1e6, logical_bytes / 1e6))


def partition_used(batch, wl):
    """Tokens per context partition that the last decode call used: the plan kernel writes
    its choice, in blocks, to word 2 of the workspace.  The automatic choice may be longer
    than the starting value pa_decode_partition_size reports."""
    import torch
    return int(batch.workspace[:4].view(torch.int32)[2].item()) * wl.block_size


def partition_entry(batch, wl, start):
    """The partition as requested (config's partition_size: 0 = automatic, as the reference
    line reports it) and as run: the starting value and the plan's final choice, in tokens."""
    return {"partition_size": wl.partition_size, "partition_start": start, "partition_used": partition_used(batch, wl)}


def workload_config(wl, partition, batch=None):
    cfg = {"workload": wl.name, "num_heads": wl.num_heads, "num_kv_heads": wl.num_kv_heads,
           "head_dim": wl.head_dim, "block_size": wl.block_size, "num_blocks": wl.num_blocks,
           "partition_size": partition, "seed": wl.seed}
    if isinstance(wl, W.CowWorkload):
        cfg.update(num_seqs=wl.num_seqs, prompts=wl.num_prompts, streams_per_prompt=wl.streams_per_prompt)
    elif isinstance(wl, W.PrefixWorkload):
        cfg.update(num_seqs=wl.num_seqs, prompts=wl.num_prompts, requests_per_prompt=wl.requests_per_prompt,
                   context_tokens=int(np.sum(wl.context_lens)), max_context_len=int(np.max(wl.context_lens)))
        if batch is not None:
            cfg.update(cached_prompt_tokens=int(batch.cached_tokens.sum()), written_prompt_tokens=batch.written_tokens,
                       unique_kv_mb=round(batch.unique_kv_bytes() / 1e6, 1),
                       allocator_us_per_request=round(batch.alloc_us_per_request, 2))
    elif isinstance(wl, W.BeamWorkload):
        cfg.update(num_seqs=wl.num_seqs, requests=wl.num_requests, beam_width=wl.beam_width,
                   beam_steps=wl.beam_steps, context_tokens=int(np.sum(wl.context_lens)),
                   max_context_len=int(np.max(wl.context_lens)))
        if batch is not None:
            cfg.update(copies_in_timed_step=int(batch.cow_pairs.shape[0]),
                       copies_per_beam_step=round(float(np.mean(batch.copies_per_step)), 2),
                       allocator_us_per_beam_step=round(float(np.median(batch.host_us_per_step)), 2))
    else:
        cfg.update(num_seqs=wl.num_seqs, context_tokens=int(np.sum(wl.context_lens)),
                   max_context_len=int(np.max(wl.context_lens)))
    return cfg


def parse_overrides(items):
    """KEY=VALUE workload overrides; VALUE is an int, a float, or a comma list."""
    def conv(x):
        for f in (int, float):
            try:
                return f(x)
            except ValueError:
                pass
        return x
    out = {}
    for it in items:
        k, v = it.split("=", 1)
        parts = [conv(x) for x in v.split(",")]
        out[k] = tuple(parts) if len(parts) > 1 else parts[0]
    return out


# ------------------------------------------------------------------ the oracle on the host cores

def _oracle_sample_inputs(wl, seqs, values):
    q, keys, vals, off = values
    ks = [keys[off[s]:off[s + 1]].float().cpu().numpy() for s in seqs]
    vs = [vals[off[s]:off[s + 1]].float().cpu().numpy() for s in seqs]
    B, Hkv, D = wl.block_size, wl.num_kv_heads, wl.head_dim
    nblk = [max(1, -(-len(k) // B)) for k in ks]
    kp = np.zeros((sum(nblk), Hkv, B, D), np.float32)
    vp = np.zeros_like(kp)
    tables = np.full((len(seqs), max(nblk)), -1, np.int32)
    base = 0
    for i in range(len(seqs)):
        L = len(ks[i])
        pad = nblk[i] * B - L
        kk = np.concatenate([ks[i], np.zeros((pad, Hkv, D), np.float32)])
        vv = np.concatenate([vs[i], np.zeros((pad, Hkv, D), np.float32)])
        kp[base:base + nblk[i]] = kk.reshape(nblk[i], B, Hkv, D).transpose(0, 2, 1, 3)
        vp[base:base + nblk[i]] = vv.reshape(nblk[i], B, Hkv, D).transpose(0, 2, 1, 3)
        tables[i, :nblk[i]] = np.arange(base, base + nblk[i])
        base += nblk[i]
    lens = np.array([len(k) for k in ks], np.int32)
    return q[list(seqs)].float().cpu().numpy(), kp, vp, tables, lens


def _seq_bytes(wl, seqs):
    elt = 4 if wl.dtype == "f32" else 2
    tok = int(sum(int(wl.context_lens[s]) for s in seqs))
    nblk = int(sum(-(-int(wl.context_lens[s]) // wl.block_size) for s in seqs))
    return tok * 2 * wl.num_kv_heads * wl.head_dim * elt + 2 * len(seqs) * wl.num_heads * wl.head_dim * elt + \
        4 * (nblk + len(seqs)) + len(seqs) * (4 * wl.num_kv_heads * wl.head_dim * elt + 8)


def cpu_model():
    """The host CPU's model name (first processor in /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def oracle_single_thread(wl, values, budget_s):
    """The oracle on one thread over the first sequences of the workload that fit the
    budget: (GB/s, sample text)."""
    from oracle import oracle
    qs, kp, vp, tb, ln = _oracle_sample_inputs(wl, [0], values)
    t0 = time.perf_counter()
    oracle.decode(qs, kp, vp, tb, ln, wl.scale, nthreads=1)
    per_seq = max(1e-4, time.perf_counter() - t0)
    n = int(max(1, min(wl.num_seqs, budget_s / per_seq)))
    seqs = list(range(n))
    inputs = _oracle_sample_inputs(wl, seqs, values)
    t0 = time.perf_counter()
    oracle.decode(*inputs, wl.scale, nthreads=1)
    t = time.perf_counter() - t0
    sample = "first %d of %d sequences of %s (%d context tokens), fp64, 1 thread" % (
        n, wl.num_seqs, wl.name, int(sum(int(wl.context_lens[s]) for s in seqs)))
    return _seq_bytes(wl, seqs) / t / 1e9, sample


def cpu_baseline_entry(wl, values, gbs, cores, sample, single_budget_s):
    """The cpu_baseline object: the multi-thread oracle figure, plus the same oracle on
    one thread and the CPU it ran on."""
    one_gbs, one_sample = oracle_single_thread(wl, values, single_budget_s)
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample,
            "cpu_model": cpu_model(),
            "single_thread": {"value": round(one_gbs, 4), "unit": "GB/s", "sample": one_sample}}


def oracle_leg(wl, budget_s, values, steps=1):
    """Times the fp64 oracle on the host cores over a sample of sequences per step.
    `values` are the generator's tensors (any device; the sample is copied to host).
    Returns (GB/s of the sample's algorithmic bytes, seqs/s, cores, sample text, seconds)."""
    from oracle import oracle
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    order = list(range(wl.num_seqs))
    # calibrate on one sequence, then size the per-step sample to the budget
    qs, kp, vp, tb, ln = _oracle_sample_inputs(wl, order[:1], values)
    t0 = time.perf_counter()
    oracle.decode(qs, kp, vp, tb, ln, wl.scale, nthreads=cores)
    per_seq = max(1e-4, time.perf_counter() - t0)
    n = int(max(1, min(wl.num_seqs, budget_s / per_seq)))
    seqs = order[:n]
    inputs = _oracle_sample_inputs(wl, seqs, values)
    t_total = 0.0
    for _ in range(steps):
        t0 = time.perf_counter()
        oracle.decode(*inputs, wl.scale, nthreads=cores)
        t_total += time.perf_counter() - t0
    nbytes = _seq_bytes(wl, seqs) * steps
    sample = "first %d of %d sequences of %s (%d context tokens) per step, fp64, %d threads" % (
        n, wl.num_seqs, wl.name, int(sum(int(wl.context_lens[s]) for s in seqs)), cores)
    return nbytes / t_total / 1e9, n * steps / t_total, cores, sample, t_total


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = W.make_workload(W.NAME_TO_ID[args.workload], seed=args.seed)
    if not isinstance(wl, W.DecodeWorkload):
        print(json.dumps({"impl": "reference", "unavailable": "oracle leg covers the decode workloads only"}))
        return 0
    total = args.steps + args.warmup
    per_step = min(2.0, 120.0 / max(1, total))
    try:
        import torch
        gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    except Exception:
        gen_dev = "cpu"
    values = W.decode_values(wl, gen_dev)
    # warm-up steps are untimed passes of the same sample
    oracle_leg(wl, per_step, values, steps=max(1, min(args.warmup, 3)))
    gbs, seqs_s, cores, sample, t = oracle_leg(wl, per_step, values, steps=args.steps)
    line = {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * t / args.steps, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, wl.partition_size), "seqs_per_s": round(seqs_s, 3),
            "cpu_baseline": cpu_baseline_entry(wl, values, gbs, cores, sample, per_step),
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------ the CUDA path

def companion_timing(batch, stream, reps=50, num_pairs=96):
    """Latency and GB/s of the companions alone: the step's slot-mapped append, a
    copy-on-write batch of `num_pairs` whole-block copies from blocks in use to free ones,
    and a swap of up to 128 blocks out to pinned host memory and back in.
    `us` is the median of per-call CUDA-event brackets; `us_back_to_back` the mean over
    `reps` calls queued without gaps."""
    import torch
    from paged_kv_cache_363_b200 import pa

    wl = batch.wl
    elt = 4 if wl.dtype == "f32" else 2
    used = np.unique(batch.block_tables.cpu().numpy())
    used = used[used >= 0]
    free = np.setdiff1d(np.arange(wl.num_blocks), used)
    n = int(min(num_pairs, len(used), len(free)))
    rng = np.random.default_rng(7)
    pairs = np.stack([rng.choice(used, n, replace=False), rng.choice(free, n, replace=False)], 1).astype(np.int64)
    pairs_d = torch.from_numpy(pairs).to(batch.device)
    row = wl.num_kv_heads * wl.head_dim * elt
    calls = {
        "reshape_and_cache": (lambda: pa.pa_reshape_and_cache(batch.new_k, batch.new_v, batch.k_cache, batch.v_cache,
                                                              batch.slot_mapping, stream=stream),
                              batch.new_k.shape[0] * (2 * row * 2 + 8), {"tokens": int(batch.new_k.shape[0])}),
        "copy_blocks": (lambda: pa.pa_copy_blocks(batch.k_cache, batch.v_cache, pairs_d, stream=stream),
                        n * 2 * (row * wl.block_size) * 2 + 16 * n, {"pairs": n}),
    }
    # swapping: whole blocks between the device pool and a pinned host pool, both ways
    ns = int(min(128, len(used), len(free)))
    kh = torch.empty((ns,) + tuple(batch.k_cache.shape[1:]), dtype=batch.k_cache.dtype).pin_memory()
    vh = torch.empty_like(kh).pin_memory()
    out_pairs = torch.from_numpy(np.stack([rng.choice(used, ns, replace=False), np.arange(ns)], 1)
                                 .astype(np.int64)).to(batch.device)
    in_pairs = torch.from_numpy(np.stack([np.arange(ns), rng.choice(free, ns, replace=False)], 1)
                                .astype(np.int64)).to(batch.device)
    swap_bytes = ns * 2 * row * wl.block_size
    calls["swap_out"] = (lambda: pa.pa_swap_blocks(kh, vh, batch.k_cache, batch.v_cache, out_pairs, stream=stream),
                         swap_bytes, {"pairs": ns, "direction": "device to pinned host"})
    calls["swap_in"] = (lambda: pa.pa_swap_blocks(batch.k_cache, batch.v_cache, kh, vh, in_pairs, stream=stream),
                        swap_bytes, {"pairs": ns, "direction": "pinned host to device"})
    flat_h = kh.view(-1)
    flat_d = torch.empty_like(flat_h, device=batch.device)
    calls["copy_engine_h2d_reference"] = (lambda: flat_d.copy_(flat_h, non_blocking=True), ns * row * wl.block_size,
                                          {"note": "one contiguous copy of one pool's swapped bytes (PCIe ceiling)"})
    out = {}
    for name, (fn, nbytes, extra) in calls.items():
        for _ in range(5):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in ev:
            a.record(stream)
            fn()
            b.record(stream)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(reps):
            fn()
        t1.record(stream)
        torch.cuda.synchronize(batch.device)
        med = statistics.median(a.elapsed_time(b) for a, b in ev)
        b2b = t0.elapsed_time(t1) / reps
        out[name] = dict(extra, bytes=nbytes, us=round(med * 1e3, 3), gbs=round(nbytes / (med * 1e-3) / 1e9, 1),
                         us_back_to_back=round(b2b * 1e3, 3), gbs_back_to_back=round(nbytes / (b2b * 1e-3) / 1e9, 1))
    return out


def plan_once_timing(batch, stream, dec_bytes, args):
    """A serving step runs decode attention once per layer over the same sequences: plan
    once (pa_decode_plan), then one pa_decode_run per layer.  Times the run alone, and
    the plan alone, with CUDA events; GB/s of the run over the same algorithmic bytes."""
    import torch
    from paged_kv_cache_363_b200 import pa

    wl = batch.wl
    part = batch.partition_size
    ws = batch.workspace_for(part)
    out = torch.empty_like(batch.q)
    plan = lambda: pa.pa_decode_plan(batch.block_tables, batch.context_lens, batch.max_context_len, wl.num_heads,
                                     batch.k_cache, ws, part, stream=stream)
    run = lambda: pa.pa_decode_run(out, batch.q, batch.k_cache, batch.v_cache, batch.block_tables,
                                   batch.context_lens, batch.max_context_len, wl.scale, ws, part, stream=stream)
    plan()
    for _ in range(max(3, args.warmup)):
        run()
    res = {}
    for name, fn in (("run", run), ("plan", plan)):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(100)]
        for a, b in ev:
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize(batch.device)
        res[name] = statistics.mean(a.elapsed_time(b) for a, b in ev)
    plan()   # leave a fresh plan
    torch.cuda.synchronize(batch.device)
    return {"run_us": round(res["run"] * 1e3, 3), "run_gbs": round(dec_bytes / (res["run"] * 1e-3) / 1e9, 1),
            "plan_us": round(res["plan"] * 1e3, 3),
            "note": "one plan per step, one run per layer; the run is the persistent decode kernel and the merge"}


def e2e_leg(stepper, args, world, dev):
    """Device time of `args.steps` host-fed steps (upload, kernels, read-back), max over ranks."""
    import torch
    import torch.distributed as dist

    for _ in range(args.warmup):
        stepper.submit()
    stepper.drain()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e_s = torch.cuda.Event(enable_timing=True)
    e_e = torch.cuda.Event(enable_timing=True)
    # the first upload is ordered after e_s: the copy stream waits for the compute stream
    e_s.record(stepper.stream)
    stepper.h2d_stream.wait_event(e_s)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        i = stepper.submit()
        stepper.host_inputs(i)            # the host may refill the buffer: its upload is done
    stepper.drain()
    e_e.record(stepper.stream)
    host_s = time.perf_counter() - t0
    torch.cuda.synchronize(dev)
    ms = reduce_max(e_s.elapsed_time(e_e), dev)
    if world > 1:
        dist.barrier()
    return {"ms": ms, "h2d": stepper.h2d_bytes, "d2h": stepper.d2h_bytes, "host_us": 1e6 * host_s / args.steps}


def make_run(name, seed, dev, overrides=None, partition=None):
    """Workload `name` at `seed`, its seeded values on `dev`, and its batch."""
    from paged_kv_cache_363_b200 import runner

    wl = W.make_workload(W.NAME_TO_ID[name], seed=seed, **(overrides or {}))
    if partition is not None:
        wl.partition_size = partition
    if isinstance(wl, W.CowWorkload):
        values = W.cow_values(wl, dev)
    elif isinstance(wl, W.PrefixWorkload):
        values = W.prefix_values(wl, dev)
    elif isinstance(wl, W.BeamWorkload):
        values = W.beam_values(wl, dev)
    elif isinstance(wl, W.PrefillWorkload):
        values = W.prefill_values(wl, dev)
    else:
        values = W.decode_values(wl, dev)
    return wl, values, runner.make_batch(wl, dev, values=values)


def time_decode_steps(batch, stream, steps, warmup, dev, world):
    """Device-resident decode steps: `warmup` untimed, then `steps` timed between a
    barrier + synchronize on both sides, each step's decode call bracketed by its own
    CUDA events on `stream`.  Whole-step and decode-call times are max over ranks."""
    import torch
    import torch.distributed as dist
    from paged_kv_cache_363_b200 import pa

    for _ in range(warmup):
        batch.step(stream)
    torch.cuda.synchronize(dev)
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clk:
        t_start.record(stream)
        for k in range(steps):
            batch.append(stream)
            ev_s[k].record(stream)
            batch.decode(stream=stream)
            ev_e[k].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    dec_ms = [a.elapsed_time(b) for a, b in zip(ev_s, ev_e)]
    return {"ms_max": reduce_max(t_start.elapsed_time(t_end), dev), "dec_ms": dec_ms,
            "dec_avg_max": reduce_max(statistics.mean(dec_ms), dev), "clocks": clk.summary(),
            "flags": pa.pa_device_status(), "out_ok": bool(torch.isfinite(batch.out.float()).all().item())}


def time_prefill_steps(batch, stream, steps, warmup, dev, world):
    """pa_prefill calls: `warmup` untimed, then `steps` timed, each bracketed by CUDA
    events on `stream`; whole-run and per-call times are max over ranks."""
    import torch
    import torch.distributed as dist
    from paged_kv_cache_363_b200 import pa

    for _ in range(warmup):
        batch.step(stream)
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clk:
        t0.record(stream)
        for a, b in evs:
            a.record(stream)
            batch.step(stream)
            b.record(stream)
        t1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    per = [a.elapsed_time(b) for a, b in evs]
    return {"ms_max": reduce_max(t0.elapsed_time(t1), dev), "per_ms": per,
            "avg_max": reduce_max(statistics.mean(per), dev), "clocks": clk.summary(),
            "flags": pa.pa_device_status(), "out_ok": bool(torch.isfinite(batch.out.float()).all().item())}


def bf16_peak():
    """The measured cuBLAS bf16 burst peak (TFLOP/s), else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (cuBLAS bf16 burst)"
    except Exception:
        return 1590.0, "fallback"


def decode_launches(batch, n_part):
    """Kernels one step launches: [copy-on-write copies], append, plan, persistent
    decode, [merge of split sequences]."""
    cow = 1 if getattr(batch, "cow_pairs", None) is not None and batch.cow_pairs.numel() else 0
    return cow + 1 + 2 + (1 if n_part > 1 else 0)


def side_workload(name, args, dev, world, rank):
    """One more workload measured in the same run as the headline: its own batch (seeded
    per rank), `steps` device-resident steps, the decode call's (or the prefill call's)
    roofline fraction against the measured peak."""
    import torch
    from paged_kv_cache_363_b200 import pa

    steps = max(5, min(args.steps, 20))
    wl, values, batch = make_run(name, rank_seed(args.seed, rank), dev)
    del values
    stream = torch.cuda.current_stream(dev)
    if isinstance(wl, W.PrefillWorkload):
        t = time_prefill_steps(batch, stream, steps, args.warmup, dev, world)
        flops = wl.flops()
        peak, kind = bf16_peak()
        achieved = flops / (t["avg_max"] * 1e-3) / 1e12
        return {"metric": "chunked prefill attention TFLOP/s (causal FLOPs)",
                "value": round(world * flops * steps / (t["ms_max"] * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "steps": steps, "ms_per_step": round(t["ms_max"] / steps, 5),
                "config": {"workload": wl.name, "num_seqs": wl.num_seqs, "num_heads": wl.num_heads,
                           "num_kv_heads": wl.num_kv_heads, "query_tokens": int(wl.query_lens.sum()),
                           "context_tokens": int(wl.context_lens.sum()), "seed": wl.seed},
                "roofline": {"bound": "tensor", "kernel": "prefill_tc_kernel", "achieved": round(achieved, 2),
                             "peak": peak, "peak_kind": kind, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                             "traffic": (profile_traffic("prefill_tc_kernel", wl.name, PREFILL_SOURCES)
                                         if wl.seed == 0 else None),
                             "algorithmic_flops_per_launch": flops, "avg_launch_us": round(t["avg_max"] * 1e3, 3)},
                "gpu_launches": steps, "clocks": t["clocks"], "device_status": t["flags"],
                "output_finite": t["out_ok"]}
    part = pa.pa_decode_partition_size(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
                                       batch.max_context_len, batch.partition_size)
    dec_bytes = batch.decode_bytes()
    step_bytes = dec_bytes + batch.append_bytes()
    t = time_decode_steps(batch, stream, steps, args.warmup, dev, world)
    peak, peak_kind = measured_hbm_peak()
    achieved = dec_bytes / (t["dec_avg_max"] * 1e-3) / 1e9
    roof = {"bound": "hbm", "kernel": "pa_decode (plan kernel + persistent decode kernel + merge)",
            "achieved": round(achieved, 2), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": profile_traffic("decode_persistent_kernel", wl.name) if wl.seed == 0 else None,
            "algorithmic_bytes_per_launch": dec_bytes, "avg_launch_us": round(t["dec_avg_max"] * 1e3, 3),
            "launch_us_p10_p50_p90": [round(float(np.percentile(t["dec_ms"], q)) * 1e3, 3) for q in (10, 50, 90)]}
    if isinstance(wl, W.CowWorkload):
        roof["note"] = ("logical bytes: the 4 streams of a prompt share its blocks, which are re-read from L2, "
                        "so the fraction can exceed 1")
    return {"value": round(world * step_bytes * steps / (t["ms_max"] * 1e-3) / 1e9, 2), "unit": "GB/s",
            "steps": steps, "ms_per_step": round(t["ms_max"] / steps, 5),
            "seqs_per_s": round(world * wl.num_seqs * steps / (t["ms_max"] * 1e-3), 1),
            "config": dict(workload_config(wl, part, batch), l2=l2_note(batch, dec_bytes),
                           **partition_entry(batch, wl, part)),
            "roofline": roof,
            "gpu_launches": decode_launches(batch, -(-batch.max_context_len // partition_used(batch, wl))) * steps,
            "clocks": t["clocks"],
            "device_status": t["flags"], "output_finite": t["out_ok"]}


SIDE_WORKLOADS = ("decode-gqa-bf16", "long-splitk-bf16", "cow-sampling-bf16", "prefill-chunk-bf16")


def side_workload_names(args):
    """Workloads measured after the headline in the same run: by default the GQA,
    long-context, copy-on-write and prefill workloads when the headline is the
    Llama-7B-shaped decode at its defaults; none for other headlines or overrides."""
    if args.workloads == "none":
        return []
    if args.workloads != "auto":
        names = [n for n in args.workloads.split(",") if n]
        for n in names:
            if n not in W.NAME_TO_ID:
                raise SystemExit("unknown workload %s" % n)
        return names
    if args.workload == "decode-mha-bf16" and profiled_config(args) and args.pool_blocks is None:
        return list(SIDE_WORKLOADS)
    return []


def run_prefill(args, wl, batch, dev, stream, world):
    """Chunked prefill: TFLOP/s of pa_prefill (causal FLOPs only) against the tensor peak."""
    import torch
    from paged_kv_cache_363_b200 import pa

    flops = wl.flops()
    t = time_prefill_steps(batch, stream, args.steps, args.warmup, dev, world)
    ms, avg = t["ms_max"], t["avg_max"]
    # end to end: each step uploads its query rows from pinned memory and reads the output back
    qh = batch.q.cpu().pin_memory()
    oh = torch.empty(batch.out.shape, dtype=batch.out.dtype).pin_memory()
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for k in range(args.warmup + args.steps):
        if k == args.warmup:
            e_s.record(stream)
        batch.q.copy_(qh, non_blocking=True)
        batch.step(stream)
        oh.copy_(batch.out, non_blocking=True)
    e_e.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max(e_s.elapsed_time(e_e), dev)
    peak, kind = bf16_peak()
    achieved = flops / (avg * 1e-3) / 1e12
    line = {
        "metric": "chunked prefill attention TFLOP/s over the paged KV cache (causal FLOPs)",
        "value": round(world * flops * args.steps / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload=wl.name, num_seqs=wl.num_seqs, num_heads=wl.num_heads, num_kv_heads=wl.num_kv_heads,
                       head_dim=wl.head_dim, block_size=wl.block_size, query_tokens=int(wl.query_lens.sum()),
                       context_tokens=int(wl.context_lens.sum()), seed=wl.seed,
                       l2="compute-bound; %.0f MB of KV read per step" % (
                           wl.context_lens.sum() * 2 * wl.num_kv_heads * wl.head_dim * 2 / 1e6),
                       parallelism="replicas: one batch per GPU (dp%d)" % world),
        "roofline": {"bound": "tensor", "kernel": "prefill_tc_kernel", "achieved": round(achieved, 2),
                     "peak": peak, "peak_kind": kind, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": (profile_traffic("prefill_tc_kernel", wl.name, PREFILL_SOURCES)
                                 if profiled_config(args) else None),
                     "algorithmic_flops_per_launch": flops, "avg_launch_us": round(avg * 1e3, 3)},
        "e2e": {"value": round(world * flops * args.steps / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": qh.numel() * qh.element_size(),
                "d2h_bytes_per_step": oh.numel() * oh.element_size(), "ms_per_step": round(e2e_ms / args.steps, 5)},
        "gpu_launches": args.steps,
        "clocks": t["clocks"],
        "device_status": t["flags"], "output_finite": t["out_ok"],
    }
    return line


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    from paged_kv_cache_363_b200 import pa, runner

    overrides = {} if args.pool_blocks is None else {"num_blocks": args.pool_blocks}
    overrides.update(parse_overrides(args.set))
    wl, values, batch = make_run(args.workload, rank_seed(args.seed, rank), dev, overrides, args.partition)
    if isinstance(wl, W.PrefillWorkload):
        stream = torch.cuda.current_stream(dev)
        line = run_prefill(args, wl, batch, dev, stream, world)
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(line))
        return 0
    part = pa.pa_decode_partition_size(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
                                       batch.max_context_len, batch.partition_size)
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)
    if pa.pa_device_status() != 0:
        raise SystemExit("device status flagged during set-up")

    dec_bytes = batch.decode_bytes()
    step_bytes = dec_bytes + batch.append_bytes()
    # ---- device-resident timing
    t = time_decode_steps(batch, stream, args.steps, args.warmup, dev, world)
    launches_per_step = decode_launches(batch, -(-batch.max_context_len // partition_used(batch, wl)))
    ms_max, dec_ms, dec_avg_max = t["ms_max"], t["dec_ms"], t["dec_avg_max"]
    out_ok, flags = t["out_ok"], t["flags"]

    e2e = None
    if not args.skip_e2e:
        # ---- end to end through the API: every step uploads its inputs from pinned host
        # memory in one copy and reads its output back; two buffers overlap the copies of
        # neighbouring steps with this step's kernels (depth 1 = no overlap, also reported)
        gbs = lambda ms: round(world * step_bytes * args.steps / (ms * 1e-3) / 1e9, 2)
        nbuf, graph = args.e2e_buffers, bool(args.e2e_graph)
        main_leg = e2e_leg(runner.HostStepper(batch, depth=nbuf, stream=stream, graph=graph), args, world, dev)
        serial = e2e_leg(runner.HostStepper(batch, depth=1, stream=stream), args, world, dev)
        e2e = {"value": gbs(main_leg["ms"]), "unit": "GB/s",
               "h2d_bytes_per_step": main_leg["h2d"], "d2h_bytes_per_step": main_leg["d2h"],
               "ms_per_step": round(main_leg["ms"] / args.steps, 5), "buffers": nbuf, "cuda_graph": graph,
               "host_us_per_submit": round(main_leg["host_us"], 2),
               "serial": {"value": gbs(serial["ms"]), "ms_per_step": round(serial["ms"] / args.steps, 5),
                          "buffers": 1, "cuda_graph": False}}

    companions = companion_timing(batch, stream) if not args.skip_e2e else None
    plan_once = plan_once_timing(batch, stream, dec_bytes, args) if not args.skip_e2e else None

    peak, peak_kind = measured_hbm_peak()
    achieved = dec_bytes / (dec_avg_max * 1e-3) / 1e9
    value = world * step_bytes * args.steps / (ms_max * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": dict(workload_config(wl, part, batch), l2=l2_note(batch, dec_bytes),
                       parallelism="replicas: one batch per GPU (dp%d)" % world, **partition_entry(batch, wl, part)),
        "seqs_per_s": round(world * wl.num_seqs * args.steps / (ms_max * 1e-3), 1),
        "pct_of_peak": round(100.0 * value / peak, 2),
        "roofline": {"bound": "hbm", "kernel": "pa_decode (plan kernel + persistent decode kernel + merge)",
                     "achieved": round(achieved, 2), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": (profile_traffic("decode_persistent_kernel", wl.name)
                                 if profiled_config(args) else None),
                     "algorithmic_bytes_per_launch": dec_bytes, "avg_launch_us": round(dec_avg_max * 1e3, 3),
                     "launch_us_p10_p50_p90": [round(float(np.percentile(dec_ms, q)) * 1e3, 3) for q in (10, 50, 90)]},
        "companions": companions,
        "plan_once": plan_once,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": t["clocks"],
        "device_status": flags, "output_finite": out_ok,
    }
    if world == 1 and not args.no_cpu_baseline and isinstance(wl, W.DecodeWorkload):
        gbs, seqs_s, cores, sample, _ = oracle_leg(wl, args.cpu_budget, values)
        line["cpu_baseline"] = cpu_baseline_entry(wl, values, gbs, cores, sample, args.cpu_budget / 4)
    # ---- the other workloads, each in its own timed region after the headline's
    side = side_workload_names(args)
    if side:
        del batch, values
        torch.cuda.empty_cache()
        line["workloads"] = {}
        for name in side:
            line["workloads"][name] = side_workload(name, args, dev, world, rank)
            torch.cuda.empty_cache()
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="decode-mha-bf16", choices=sorted(W.NAME_TO_ID))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--partition", type=int, default=None, help="context partition tokens (0 = automatic)")
    ap.add_argument("--cpu-budget", type=float, default=8.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true", help="skip the end-to-end leg (profiling runs)")
    ap.add_argument("--e2e-buffers", type=int, default=2,
                    help="host/device buffer pairs the end-to-end leg rotates (1 = no copy/compute overlap)")
    ap.add_argument("--e2e-graph", type=int, default=1, choices=(0, 1),
                    help="replay each buffer's kernels from a captured CUDA graph in the end-to-end leg")
    ap.add_argument("--pool-blocks", type=int, default=None,
                    help="override the pool size (profiling runs on a smaller device footprint)")
    ap.add_argument("--workloads", default="auto",
                    help="comma list of workloads measured after the headline in the same run (auto: GQA, long "
                         "context, copy-on-write and prefill after the default headline; none: skip)")
    ap.add_argument("--set", action="append", default=[], metavar="KEY=VALUE",
                    help="override a workload field, e.g. num_kv_heads=32 or lens=uniform,128,2048")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
