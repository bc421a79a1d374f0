"""Benchmark: paged decode attention on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--seed S]

Workload: one Llama-2-70B attention layer decode step -- 32 sequences x 64 heads x 128
dims, block_size 16, contexts uniform in [1, 2048], pool = blocks needed + 10 %, shuffled
free list, fp16, synthetic N(0, 1) data.  A step is the whole hot path: write each
sequence's newest K/V row into its slot (reshape_and_cache; no copy-on-write occurs in
this workload, so copy_blocks has nothing to do), then paged decode attention (partition
+ merge kernels).  With N GPUs every rank runs its own batch (seed + rank): weak
scaling, no collective on the data path; the timing is the max over ranks.

Metric: algorithmic KV bytes (every attended K and V row read once) / step time, in GB/s;
also tokens/s per layer (= sequences / step time) and % of the measured HBM copy peak.
"""
from __future__ import annotations

import argparse
import hashlib
import importlib.util
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402


def _load_accounting():
    """The package's byte / FLOP accounting (host arithmetic on sizes), loaded on its own so
    that the reference arm never loads the CUDA library the package __init__ opens."""
    spec = importlib.util.spec_from_file_location(
        "pa_accounting", os.path.join(ROOT, "paged_kv_cache_384_b200", "accounting.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


accounting = _load_accounting()

PRESET = "llama70b_fp16"
CONTEXT_DESC = {"llama70b_fp16": "uniform [1, 2048]",
                "chat_prefix_bf16": "2000 shared + lognormal(median 300, sigma 1) tail, 64 copy-on-write forks",
                "sliding_window_fp16": "32768 each, window 4096",
                "llama70b_gqa_fp16": "uniform [1, 2048], 64 query heads over 8 cached heads",
                "llama70b_int8": "uniform [1, 2048], INT8 cache written by quantise-on-write",
                "llama70b_fp8": "uniform [1, 2048], FP8 E4M3 cache written by quantise-on-write",
                "llama70b_gqa_int8": "uniform [1, 2048], 64 query heads over 8 cached heads, INT8 cache written by "
                                     "quantise-on-write",
                "llama70b_gqa_fp8": "uniform [1, 2048], 64 query heads over 8 cached heads, FP8 E4M3 cache written by "
                                    "quantise-on-write"}
METRIC = "paged decode attention KV GB/s (% of B200 HBM peak) and tokens/s per layer"
FALLBACK_HBM_GBS = 6650.0      # copy bandwidth measured earlier on this GPU type
FALLBACK_BF16_TFLOPS = 1590.0  # cuBLAS bf16 burst measured earlier on this GPU type
NOMINAL_HBM_GBS = 8000.0       # the ~8 TB/s HBM3e figure quoted for B200 (7.7 TB/s in HGX systems)


# ---------------------------------------------------------------------------------------
# helpers shared with the multi-rank tests
# ---------------------------------------------------------------------------------------
def rank_seed(seed: int, rank: int) -> int:
    """Each rank decodes its own batch (weak scaling)."""
    return seed + 1000 * rank


def reduce_max(value: float, dist=None) -> float:
    """Max over ranks of a per-rank time (identity without a process group)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_rank_step, steps: int, max_seconds: float) -> float:
    """Aggregate GB/s: bytes of every rank over the slowest rank's time."""
    return sum(bytes_per_rank_step) * steps / max_seconds / 1e9


def _peaks_file():
    with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
        return json.load(f)


def measured_peak():
    """HBM copy bandwidth (GB/s) of this GPU type and where it comes from."""
    try:
        return float(_peaks_file()["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError, TypeError):
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense fp16/bf16 tensor throughput (TFLOP/s, burst) and where it comes from."""
    try:
        return float(_peaks_file()["bf16_tflops"]), "measured (cuBLAS bf16 burst)"
    except (OSError, KeyError, ValueError, TypeError):
        return FALLBACK_BF16_TFLOPS, "fallback (cuBLAS bf16 burst measured earlier on this GPU type)"


def source_digest(kernel_source: str) -> str:
    """SHA-256 over a kernel's source file followed by the device headers beside it that the
    kernels include (pa_device.cuh, pa_decode_shared.cuh), so a record goes stale when any of
    them changes."""
    h = hashlib.sha256()
    with open(kernel_source, "rb") as f:
        h.update(f.read())
    here = os.path.dirname(kernel_source)
    for name in ("pa_device.cuh", "pa_decode_shared.cuh"):
        path = os.path.join(here, name)
        if os.path.exists(path):
            with open(path, "rb") as f:
                h.update(f.read())
    return h.hexdigest()


def kernel_traffic(kernel_source: str, record: str = "decode_partition_traffic.json", workload: str = None):
    """ncu DRAM bytes per launch of a kernel, if captured for this exact source and workload."""
    path = os.path.join(ROOT, "profiles", record)
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    sha = source_digest(kernel_source)
    if rec.get("source_sha256") != sha or rec.get("workload") != (PRESET if workload is None else workload):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi samples (every 100 ms) of SM clock, power and throttle reasons.

    ``mark()`` is called when the timed region starts; ``summary()`` keeps only samples
    taken after it (the timed region plus, when it is shorter than a second, an untimed
    soak of the same steps that follows it, so that there is something to sample).
    """

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.idx = device_id
        self.proc = None
        self.lines = []
        self.t_mark = None

    def __enter__(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="pa_clocks_", suffix=".csv")
        os.close(fd)
        try:
            # -f: nvidia-smi writes each sample line itself (a pipe would buffer them away)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def mark(self):
        import datetime
        self.t_mark = datetime.datetime.now()

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.send_signal(2)
            try:
                self.proc.wait(timeout=10)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
        try:
            with open(self.path) as f:
                self.lines = [l for l in f.read().splitlines() if l.strip()]
            os.unlink(self.path)
        except OSError:
            self.lines = []
        return False

    def summary(self):
        import datetime
        rows = []
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f")
                rows.append(dict(ts=ts, sm=float(f[1]), max=float(f[2]), power=float(f[3]),
                                 hw=f[5], hwt=f[6], swt=f[7], pcap=f[8]))
            except ValueError:
                continue
        if self.t_mark is not None:
            rows = [r for r in rows if r["ts"] >= self.t_mark]
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["max"] for r in rows),
                "samples": len(rows), "power_w_median": statistics.median(r["power"] for r in rows),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------------------
# 8-bit workloads: (the fp16 batch their cache is quantised from, code dtype)
EIGHT_BIT = {"llama70b_int8": ("llama70b_int8", torch.int8), "llama70b_fp8": ("llama70b_int8", torch.float8_e4m3fn),
             "llama70b_gqa_int8": ("llama70b_gqa_fp16", torch.int8),
             "llama70b_gqa_fp8": ("llama70b_gqa_fp16", torch.float8_e4m3fn)}


def build(seed: int, device, workload: str = PRESET, block_size=None):
    import paged_kv_cache_384_b200 as pa
    over = {} if block_size is None else {"block_size": block_size}
    big = workload == "sliding_window_fp16"          # 8.6 GB of cache: draw values on the GPU
    preset = EIGHT_BIT[workload][0] if workload in EIGHT_BIT else workload
    w = synth.build_workload(preset, seed, pa.BlockManager, device=device if big else "cpu", **over)
    ctx = w.context_lens.tolist()
    slots = pa.slot_mapping(w.block_tables, range(w.num_seqs), [c - 1 for c in ctx], w.block_size)
    host = dict(q=w.q.cpu(), k_new=w.k_new.cpu(), v_new=w.v_new.cpu(), slots=slots, block_tables=w.block_tables,
                context_lens=w.context_lens)
    dev = {k: v.to(device) for k, v in host.items()}
    dev["k_cache"] = w.k_cache.to(device)
    dev["v_cache"] = w.v_cache.to(device)
    dev["k_scale"] = dev["v_scale"] = None
    if workload in EIGHT_BIT:
        # The fp16 pool is quantised on the GPU by the library's own quantise-on-write
        # kernel, every slot as one row (untimed setup); steps then write the newest rows
        # through the same kernel.
        src_k, src_v = dev["k_cache"], dev["v_cache"]
        NB, bs, H, D = src_k.shape
        code = EIGHT_BIT[workload][1]
        dev["k_cache"] = torch.empty(NB, bs, H, D, dtype=code, device=device)
        dev["v_cache"] = torch.empty_like(dev["k_cache"])
        dev["k_scale"] = torch.empty(NB, bs, H, dtype=torch.float16, device=device)
        dev["v_scale"] = torch.empty_like(dev["k_scale"])
        all_slots = torch.arange(NB * bs, dtype=torch.int64, device=device)
        pa.reshape_and_cache_quant(src_k.view(NB * bs, H, D), src_v.view(NB * bs, H, D), dev["k_cache"],
                                   dev["v_cache"], dev["k_scale"], dev["v_scale"], all_slots)
        torch.cuda.synchronize(device)
        del src_k, src_v
        w.cache_dtype = "int8" if code == torch.int8 else "fp8"
    dev["out"] = torch.empty_like(dev["q"])
    dev["ws"] = pa.alloc_workspace(w.num_seqs, w.num_heads, w.head_dim, device)
    dev["pairs"] = w.copy_pairs.to(device)
    kv_bytes = accounting.decode_kv_bytes(ctx, w.num_kv_heads, w.head_dim, w.cache_dtype, w.window)
    return w, host, dev, kv_bytes


def step(pa, w, d, stream):
    """One pass of the hot path: append the newest rows, copy-on-write copies, decode."""
    if d["k_scale"] is not None:   # 8-bit cache: quantise-on-write
        pa.reshape_and_cache_quant(d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], d["k_scale"], d["v_scale"],
                                   d["slots"], stream=stream)
    else:
        pa.reshape_and_cache(d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], d["slots"], stream=stream)
    if d["pairs"].shape[0]:
        pa.copy_blocks(d["k_cache"], d["v_cache"], d["pairs"], stream=stream)
    pa.paged_attention_decode(d["out"], d["q"], d["k_cache"], d["v_cache"], d["block_tables"],
                              d["context_lens"], w.scale, w.window, d["k_scale"], d["v_scale"], workspace=d["ws"],
                              stream=stream)


class PackedInputs:
    """A step's per-request inputs packed into one pinned host buffer and one device
    buffer (256-byte aligned fields), so they cross PCIe in a single copy."""

    def __init__(self, host: dict, device):
        self.layout, off = {}, 0
        for k, t in host.items():
            n = t.numel() * t.element_size()
            self.layout[k] = (off, t.dtype, tuple(t.shape))
            off = (off + n + 255) // 256 * 256
        self.nbytes = off
        self.h = torch.zeros(off, dtype=torch.uint8).pin_memory()
        for k, t in host.items():
            o, _, _ = self.layout[k]
            n = t.numel() * t.element_size()
            self.h[o:o + n].copy_(t.contiguous().view(-1).view(torch.uint8))
        self.d = torch.empty(off, dtype=torch.uint8, device=device)

    def views(self):
        out = {}
        for k, (o, dt, shape) in self.layout.items():
            n = math.prod(shape) * torch.empty((), dtype=dt).element_size()
            out[k] = self.d[o:o + n].view(dt).view(shape)
        return out


def run_e2e(pa, w, d, host, args, device, stream, barrier):
    """Steps through the public API with inputs in pinned host memory and the result read
    back every step.  Two input/output buffer sets and a copy stream pipeline the
    transfers: the inputs of step i+1 cross PCIe while step i computes."""
    sets = [PackedInputs(host, device) for _ in range(2)]
    outs_h = [torch.empty(d["out"].shape, dtype=d["out"].dtype).pin_memory() for _ in range(2)]
    outs_d = [torch.empty_like(d["out"]) for _ in range(2)]
    copy = torch.cuda.Stream(device)
    h2d = sets[0].nbytes
    d2h = outs_h[0].numel() * outs_h[0].element_size()
    dd = [dict(d, **s.views()) for s in sets]
    for i in range(2):
        dd[i]["out"] = outs_d[i]

    def run(n):
        ready = [torch.cuda.Event() for _ in range(2)]     # inputs of set i on the device
        done = [torch.cuda.Event() for _ in range(2)]      # step on set i finished
        copy.wait_stream(stream)                           # no transfer starts before the timer
        with torch.cuda.stream(copy):
            sets[0].d.copy_(sets[0].h, non_blocking=True)
            ready[0].record(copy)
        for i in range(n):
            b = i % 2
            stream.wait_event(ready[b])
            step(pa, w, dd[b], stream)
            done[b].record(stream)
            with torch.cuda.stream(copy):
                if i + 1 < n:                               # prefetch the next step's inputs
                    nb = (i + 1) % 2
                    if i >= 1:
                        copy.wait_event(done[nb])
                    sets[nb].d.copy_(sets[nb].h, non_blocking=True)
                    ready[nb].record(copy)
                copy.wait_event(done[b])
                outs_h[b].copy_(outs_d[b], non_blocking=True)  # read the result back
        stream.wait_stream(copy)

    run(args.warmup)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run(args.steps)
    e1.record(stream)
    barrier()
    return e0.elapsed_time(e1) / 1e3, h2d, d2h


def launches_per_step(d) -> int:
    return 1 + (1 if d["pairs"].shape[0] else 0) + 2


# ---------------------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------------------
def cpu_oracle_rate(w, seqs, threads=1, repeats=1):
    """Time the fp64 oracle (plain C, ``threads`` worker threads over the independent
    (sequence, head) pairs) on the given sequences of the workload."""
    import oracle  # the CPU-baseline legs are the one place the benchmark runs the oracle
    sel = list(seqs)
    kv = accounting.decode_kv_bytes([int(w.context_lens[s]) for s in sel], w.num_kv_heads, w.head_dim,
                                    w.cache_dtype, w.window)
    q, bt, cl = w.q[sel], w.block_tables[sel], w.context_lens[sel]
    t0 = time.perf_counter()
    for _ in range(repeats):
        oracle.paged_decode(q, w.k_cache, w.v_cache, bt, cl, w.scale, w.window, threads=threads)
    dt = (time.perf_counter() - t0) / repeats
    return kv / dt / 1e9, dt, kv


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def run_reference(args):
    """The oracle as it stands on the host cores, same workload/metric; rank 0 only.  The
    batch is laid out by the oracle's own block manager, so nothing of the product library
    is loaded.  A step is the whole 32-sequence batch on every core, unless one step would
    make the run take more than about two minutes; then a strided sample of the sequences,
    stated in ``config``."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from oracle.block_manager import BlockManager as OracleBM
    w = synth.build_workload(PRESET, args.seed, OracleBM)
    cores = host_cores()
    sel = list(range(w.num_seqs))
    _, probe, _ = cpu_oracle_rate(w, sel, threads=cores)
    stride = 1
    while stride < w.num_seqs and probe / stride * (args.steps + args.warmup) > 120.0:
        stride *= 2
    sel = list(range(0, w.num_seqs, stride))
    for _ in range(max(0, args.warmup - 1)):
        cpu_oracle_rate(w, sel, threads=cores)
    times, kv = [], 0
    for _ in range(args.steps):
        _, dt, kv = cpu_oracle_rate(w, sel, threads=cores)
        times.append(dt)
    t = sum(times) / len(times)
    value = kv / t / 1e9
    if stride == 1:
        desc = f"the whole {PRESET} batch (32 sequences) per step, fp64 C oracle on {cores} threads"
    else:
        desc = (f"sequences 0,{stride},...({len(sel)} of 32) of the {PRESET} batch per step, fp64 C oracle "
                f"on {cores} threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * t, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": PRESET, "num_seqs": len(sel), "num_heads": w.num_heads, "head_dim": w.head_dim,
                   "block_size": w.block_size, "num_blocks": w.num_blocks, "window": w.window,
                   "context": CONTEXT_DESC[PRESET], "seed": args.seed,
                   "sample": "whole batch" if stride == 1 else f"every {stride}th sequence"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def timed_steps(pa, w, d, stream, steps) -> float:
    """Seconds for ``steps`` steps, CUDA events on the launching stream."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step(pa, w, d, stream)
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / 1e3


def decode_kernel_ms(pa, w, d, stream, steps):
    """Average (attention kernel, merge kernel) ms per step, from the events the library
    records around its own launches."""
    pa.profile_enable(True)
    pa.profile_read(reset=True)
    for _ in range(steps):
        step(pa, w, d, stream)
    part_ms, merge_ms, calls = pa.profile_read(reset=True)
    pa.profile_enable(False)
    return part_ms / max(calls, 1), merge_ms / max(calls, 1)


def decode_kernel_name(w) -> str:
    if w.num_kv_heads * 4 > w.num_heads:
        return "decode_partition_kernel"
    return "decode_gqa_tc8_kernel" if w.cache_dtype in ("int8", "fp8") else "decode_gqa_tc_kernel"


# The other decode workloads of the method, measured after the metric's own workload in a
# default run so that their numbers sit in the same record: the prefix-sharing chat batch,
# the INT8 and FP8 caches, the 32k-token sliding window at block sizes 8 / 16 / 32, and the
# grouped-query Llama-2-70B layer (64 query heads over 8 cached heads) with fp16, INT8 and FP8
# caches.
SECONDARY = (("chat_prefix_bf16", None), ("llama70b_int8", None), ("llama70b_fp8", None),
             ("sliding_window_fp16", 8), ("sliding_window_fp16", 16), ("sliding_window_fp16", 32),
             ("llama70b_gqa_fp16", None), ("llama70b_gqa_int8", None), ("llama70b_gqa_fp8", None))
SECONDARY_STEPS = 100


def measure_secondary(pa, name, bs, seed, device, stream, peak):
    w, _host, d, kv = build(seed, device, name, bs)
    for _ in range(5):
        step(pa, w, d, stream)
    torch.cuda.synchronize(device)
    sec = timed_steps(pa, w, d, stream, SECONDARY_STEPS)
    part, merge = decode_kernel_ms(pa, w, d, stream, SECONDARY_STEPS)
    errs = pa.device_error(clear=True)
    ms = 1e3 * sec / SECONDARY_STEPS
    rec = {"workload": name, "block_size": w.block_size, "cache_dtype": w.cache_dtype, "steps": SECONDARY_STEPS,
           "context": CONTEXT_DESC.get(name, ""), "kv_bytes_per_step": kv,
           "ms_per_step": round(ms, 4), "kv_gbs": round(kv / sec * SECONDARY_STEPS / 1e9, 2),
           "frac": round(kv / sec * SECONDARY_STEPS / 1e9 / peak, 4),
           "frac_of_nominal": round(kv / sec * SECONDARY_STEPS / 1e9 / NOMINAL_HBM_GBS, 4),
           "kernel": decode_kernel_name(w), "kernel_ms": round(part, 4), "merge_ms": round(merge, 4),
           "kernel_gbs": round(kv / part / 1e6, 2), "kernel_frac": round(kv / part / 1e6 / peak, 4),
           "tokens_per_s_per_layer": round(w.num_seqs / (ms / 1e3), 1), "device_errors": errs}
    if name == "chat_prefix_bf16":
        # The shared 2000-token prefix is read by all 256 sequences but held once, and it
        # stays in L2: the logical bytes above exceed what HBM can deliver.  The roofline of
        # this workload is the DRAM traffic the kernel causes (ncu byte counters, captured
        # for this exact source) against the distinct rows it must read at least once.
        unique = accounting.decode_unique_kv_bytes(w.block_tables.tolist(), w.context_lens.tolist(), w.block_size,
                                                   w.num_kv_heads, w.head_dim, w.cache_dtype, w.window)
        dram = kernel_traffic(os.path.join(ROOT, "paged_kv_cache_384_b200", "csrc", "pa_decode.cu"),
                              "decode_partition_traffic_chat_prefix_bf16.json", name)
        rec.update({"unique_kv_bytes": unique, "unique_gbs_kernel": round(unique / part / 1e6, 2),
                    "dram_bytes_per_launch": dram,
                    "dram_gbs_kernel": None if dram is None else round(dram / part / 1e6, 2),
                    "dram_frac": None if dram is None else round(dram / part / 1e6 / peak, 4),
                    "unique_over_dram": None if dram is None else round(unique / dram, 4)})
    del w, d
    torch.cuda.empty_cache()
    return rec


def run_ours(args):
    import paged_kv_cache_384_b200 as pa
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w, host, d, kv_bytes = build(rank_seed(args.seed, rank), device, args.workload, args.block_size)
    stream = torch.cuda.current_stream(device)
    peak, peak_kind = measured_peak()

    def barrier():
        if dist is not None:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize(device)

    # ---- warm-up, then the timed region: K steps between two events ----
    for _ in range(args.warmup):
        step(pa, w, d, stream)
    barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(device)
    smi_id = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    with ClockSampler(smi_id) as clocks:
        clocks.mark()
        start.record(stream)
        for _ in range(args.steps):
            step(pa, w, d, stream)
        end.record(stream)
        barrier()
        sec = start.elapsed_time(end) / 1e3
        soak = max(0, int((1.0 - sec) / max(sec / args.steps, 1e-6)))  # same steps, untimed
        for _ in range(soak):
            step(pa, w, d, stream)
        torch.cuda.synchronize(device)
    sec_max = reduce_max(sec, dist)
    all_bytes = [kv_bytes] * world if dist is None else None
    if dist is not None:
        t = torch.tensor([float(kv_bytes)], dtype=torch.float64, device=device)
        gathered = [torch.zeros_like(t) for _ in range(world)]
        dist.all_gather(gathered, t)
        all_bytes = [float(x.item()) for x in gathered]
    value = whole_job_gbs(all_bytes, args.steps, sec_max)
    ms_step = 1e3 * sec_max / args.steps
    tokens_per_s = world * w.num_seqs * args.steps / sec_max
    device_errors = pa.device_error(clear=True)
    pa.device_error(clear=True)

    # ---- roofline: the attention kernel alone (library events around it) ----
    part_avg, merge_avg = decode_kernel_ms(pa, w, d, stream, args.steps)
    achieved = kv_bytes / (part_avg / 1e3) / 1e9
    traffic = kernel_traffic(os.path.join(ROOT, "paged_kv_cache_384_b200", "csrc", "pa_decode.cu"))

    # ---- end to end through the public API with host buffers ----
    e2e_sec, h2d, d2h = run_e2e(pa, w, d, host, args, device, stream, barrier)
    e2e_sec = reduce_max(e2e_sec, dist)
    e2e_value = whole_job_gbs(all_bytes, args.steps, e2e_sec)

    # ---- CPU baseline: the oracle on this batch, rank 0 at N = 1 only ----
    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline and args.workload == PRESET:
        cores = host_cores()
        rate, dt, _ = cpu_oracle_rate(w, range(w.num_seqs), threads=cores, repeats=3)
        rate1, dt1, _ = cpu_oracle_rate(w, range(w.num_seqs), threads=1)
        cpu = {"value": round(rate, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"the full {PRESET} batch (32 sequences), fp64 C oracle, {cores} threads over the "
                         f"(sequence, head) pairs, {dt:.2f} s per batch (mean of 3)",
               "single_core": {"value": round(rate1, 4), "unit": "GB/s", "cores": 1, "seconds": round(dt1, 2)}}

    launches = launches_per_step(d) * args.steps
    cache_dtype, nseq, nheads, hd = w.cache_dtype, w.num_seqs, w.num_heads, w.head_dim
    bsz, nblk, win, kernel_name = w.block_size, w.num_blocks, w.window, decode_kernel_name(w)
    workloads = workloads_clocks = None
    if world == 1 and args.workload == PRESET and not args.no_workloads:
        del w, d, host   # free this batch before the next ones are built
        torch.cuda.empty_cache()
        workloads = []
        with ClockSampler(smi_id) as wclocks:
            wclocks.mark()
            for name, bs in SECONDARY:
                workloads.append(measure_secondary(pa, name, bs, rank_seed(args.seed, rank), device, stream, peak))
        workloads_clocks = wclocks.summary()

    if dist is not None:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {"fp16": "f16", "bf16": "bf16", "fp32": "f32", "int8": "i8", "fp8": "fp8_e4m3"}[cache_dtype],
        "data": "synthetic",
        "config": {"workload": args.workload, "num_seqs": nseq, "num_heads": nheads, "head_dim": hd,
                   "block_size": bsz, "num_blocks": nblk, "window": win,
                   "context": CONTEXT_DESC.get(args.workload, ""),
                   "kv_bytes_per_step_per_gpu": kv_bytes, "seed": args.seed,
                   "l2": "inputs larger than L2 (KV per step >> 126 MB), no flush", "parallelism": f"replicas x{world}"},
        "tokens_per_s_per_layer": round(tokens_per_s, 1),
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "pct_of_nominal_hbm": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": peak_kind,
                     "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                     "nominal_peak": NOMINAL_HBM_GBS,
                     "kernel": kernel_name,
                     "partition_ms": round(part_avg, 4),
                     "merge_ms": round(merge_avg, 4)},
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
        "device_errors": device_errors,
        "workloads": workloads,
        "workloads_clocks": workloads_clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_swap(args):
    """Preemption swap of the Llama-2-70B layer batch: the blocks of the last 8 of the 32
    sequences move to a page-locked host pool (swap-out) and back (swap-in), one
    swap_blocks launch per direction.  The host-link ceiling is measured live: one copy
    of the same bytes per direction between contiguous pinned and device buffers."""
    import paged_kv_cache_384_b200 as pa
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    w = synth.build_workload(PRESET, args.seed, pa.BlockManager)
    gk, gv = w.k_cache.to(device), w.v_cache.to(device)
    ctx = w.context_lens.tolist()
    victims = range(w.num_seqs - 8, w.num_seqs)
    blocks = [int(w.block_tables[s, j]) for s in victims for j in range(-(-ctx[s] // w.block_size))]
    n = len(blocks)
    hk = torch.empty((n,) + tuple(gk.shape[1:]), dtype=gk.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_pairs = torch.tensor([[b, i] for i, b in enumerate(blocks)], dtype=torch.int64)
    in_pairs = out_pairs.flip(1).contiguous()
    d_out, d_in = out_pairs.to(device), in_pairs.to(device)
    block_bytes = gk[0].numel() * gk.element_size()
    bytes_step = 2 * 2 * n * block_bytes                    # K and V, out and back in
    stream = torch.cuda.current_stream(device)

    def step():
        pa.swap_blocks(gk, gv, hk, hv, d_out, stream=stream)
        pa.swap_blocks(hk, hv, gk, gv, d_in, stream=stream)

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / 1e3 / reps

    # host-link ceiling: contiguous copies of the same bytes, one per direction
    flat_d = torch.empty(n * block_bytes * 2, dtype=torch.uint8, device=device)
    flat_h = torch.empty(n * block_bytes * 2, dtype=torch.uint8).pin_memory()

    def link():
        flat_h.copy_(flat_d, non_blocking=True)
        flat_d.copy_(flat_h, non_blocking=True)
    link_gbs = bytes_step / timed(link, 5) / 1e9

    # the per-block alternative: one copy-engine transfer per block and pool
    def per_block():
        for s_, t_ in out_pairs.tolist():
            hk[t_].copy_(gk[s_], non_blocking=True)
            hv[t_].copy_(gv[s_], non_blocking=True)
        for s_, t_ in in_pairs.tolist():
            gk[t_].copy_(hk[s_], non_blocking=True)
            gv[t_].copy_(hv[s_], non_blocking=True)
    per_block_gbs = bytes_step / timed(per_block, 2) / 1e9

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(device)
    smi_id = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    with ClockSampler(smi_id) as clocks:
        clocks.mark()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(device)
    sec = e0.elapsed_time(e1) / 1e3
    value = bytes_step * args.steps / sec / 1e9

    # end to end: pairs handed over in pinned host memory each step (read by the kernel)
    h_out, h_in = out_pairs.pin_memory(), in_pairs.pin_memory()

    def e2e_step():
        pa.swap_blocks(gk, gv, hk, hv, h_out, stream=stream)
        pa.swap_blocks(hk, hv, gk, gv, h_in, stream=stream)
    e2e_sec = timed(e2e_step, args.steps)
    ok = torch.equal(gk[blocks[0]], hk[0].to(device)) and pa.device_error(clear=True) == 0
    line = {
        "metric": "KV block swap GB/s (GPU <-> page-locked host pool, out + in)", "value": round(value, 2),
        "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sec / args.steps, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": "swap_llama70b_fp16", "preempted_seqs": 8, "blocks_swapped": n,
                   "block_bytes": block_bytes, "bytes_per_step": bytes_step, "seed": args.seed,
                   "l2": "inputs larger than L2, no flush"},
        "roofline": {"bound": "host_link", "achieved": round(value, 2), "peak": round(link_gbs, 2), "unit": "GB/s",
                     "frac": round(value / link_gbs, 4), "traffic": None,
                     "peak_source": "measured live: one contiguous pinned copy per direction, same bytes"},
        "per_block_copy_engine_gbs": round(per_block_gbs, 2),
        "cpu_baseline": None,
        "e2e": {"value": round(bytes_step / e2e_sec / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": bytes_step // 2 + 2 * out_pairs.numel() * 8,
                "d2h_bytes_per_step": bytes_step // 2},
        "gpu_launches": 2 * args.steps, "clocks": clocks.summary(), "verified": bool(ok),
    }
    print(json.dumps(line), flush=True)
    return 0


PREFILL = {  # name: (prompts, prompt/chunk tokens, cached tokens before the chunk, q heads, kv heads)
    "prefill_llama70b_fp16": (4, 2048, 0, 64, 64),
    "prefill_llama70b_gqa_fp16": (4, 2048, 0, 64, 8),
    "chunked_prefill_llama70b_fp16": (8, 512, 1536, 64, 64),
    "prefill_llama70b_int8": (4, 2048, 0, 64, 64),
    "prefill_llama70b_fp8": (4, 2048, 0, 64, 64),
}
PREFILL_CODES = {"prefill_llama70b_int8": torch.int8, "prefill_llama70b_fp8": torch.float8_e4m3fn}


def run_prefill(args):
    """Prompt processing of one Llama-2-70B attention layer: each sequence's new tokens
    are written into the paged cache (reshape_and_cache) and attend causally to it
    (paged_attention_prefill).  The prompt batch holds 8192 tokens (the engine's
    max_num_batched_tokens on the deployment page).  Metric: attention FLOP/s, where a
    query row that attends n tokens costs 4 * n * head_dim FLOPs (QK^T and PV)."""
    import paged_kv_cache_384_b200 as pa
    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    S, qn, cached, Hq, Hkv = PREFILL[args.workload]
    D, bs = 128, args.block_size or 16
    ctx = qn + cached
    nblk = -(-ctx // bs)
    g = torch.Generator(device=device).manual_seed(args.seed)
    NB = int(math.ceil(1.1 * S * nblk))
    perm = torch.randperm(NB, generator=g, device=device)
    bt = perm[: S * nblk].view(S, nblk).to(torch.int32).contiguous()
    kc = torch.randn(NB, bs, Hkv, D, generator=g, device=device, dtype=torch.float16)
    vc = torch.randn(NB, bs, Hkv, D, generator=g, device=device, dtype=torch.float16)
    T = S * qn
    q = torch.randn(T, Hq, D, generator=g, device=device, dtype=torch.float16)
    k_new = torch.randn(T, Hkv, D, generator=g, device=device, dtype=torch.float16)
    v_new = torch.randn(T, Hkv, D, generator=g, device=device, dtype=torch.float16)
    pos = torch.arange(cached, ctx, device=device).repeat(S)
    seq = torch.arange(S, device=device).repeat_interleave(qn)
    slots = (bt[seq, pos // bs].long() * bs + pos % bs).contiguous()
    cu = torch.arange(0, T + 1, qn, dtype=torch.int32, device=device)
    cl = torch.full((S,), ctx, dtype=torch.int32, device=device)
    out = torch.empty_like(q)
    scale = 1 / math.sqrt(D)
    stream = torch.cuda.current_stream(device)
    flops = accounting.prefill_flops([ctx] * S, [qn] * S, Hq, D)  # causal: position p sees p + 1 tokens
    code = PREFILL_CODES.get(args.workload)
    ks = vs = None
    if code is not None:
        # 8-bit cache: the fp16 pool quantised by the library's quantise-on-write (untimed
        # setup); each step then quantises the new rows into it
        ks = torch.empty(NB, bs, Hkv, dtype=torch.float16, device=device)
        vs = torch.empty_like(ks)
        kq, vq = torch.empty(kc.shape, dtype=code, device=device), torch.empty(vc.shape, dtype=code, device=device)
        all_slots = torch.arange(NB * bs, dtype=torch.int64, device=device)
        pa.reshape_and_cache_quant(kc.view(NB * bs, Hkv, D), vc.view(NB * bs, Hkv, D), kq, vq, ks, vs, all_slots)
        torch.cuda.synchronize(device)
        kc, vc = kq, vq

    def attn():
        pa.paged_attention_prefill(out, q, kc, vc, bt, cu, cl, qn, scale, stream=stream, k_scale=ks, v_scale=vs)

    def step():
        if code is not None:
            pa.reshape_and_cache_quant(k_new, v_new, kc, vc, ks, vs, slots, stream=stream)
        else:
            pa.reshape_and_cache(k_new, v_new, kc, vc, slots, stream=stream)
        attn()

    def timed(fn, reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / 1e3 / reps

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    props = torch.cuda.get_device_properties(device)
    smi_id = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    with ClockSampler(smi_id) as clocks:
        clocks.mark()
        sec = timed(step, args.steps)
        attn_sec = timed(attn, args.steps)
    peak, peak_kind = measured_tensor_peak()  # fp16 and bf16 run at the same tensor rate
    # end to end: q and the new K/V rows from pinned host memory, the output read back
    hq, hk, hv = q.cpu().pin_memory(), k_new.cpu().pin_memory(), v_new.cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        k_new.copy_(hk, non_blocking=True)
        v_new.copy_(hv, non_blocking=True)
        step()
        hout.copy_(out, non_blocking=True)
    e2e_step()
    torch.cuda.synchronize(device)
    e2e_sec = timed(e2e_step, max(3, args.steps // 4))
    nbytes = lambda t: t.numel() * t.element_size()
    errs = pa.device_error(clear=True)
    line = {
        "metric": "paged prefill attention TFLOP/s (causal, 4*n*head_dim FLOPs per query row)",
        "value": round(flops / sec / 1e12, 2), "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * sec, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": args.workload, "prompts": S, "new_tokens_per_seq": qn, "cached_before": cached,
                   "cache": {None: "fp16", torch.int8: "int8 + fp16 scales",
                             torch.float8_e4m3fn: "fp8 e4m3 + fp16 scales"}[code],
                   "num_q_heads": Hq, "num_kv_heads": Hkv, "head_dim": D, "block_size": bs, "seed": args.seed,
                   "step": "reshape_and_cache of the new K/V rows + paged_attention_prefill",
                   "l2": "K/V and q per step larger than L2, no flush"},
        "tokens_per_s": round(T / sec, 1),
        "roofline": {"bound": "tensor", "achieved": round(flops / attn_sec / 1e12, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(flops / attn_sec / 1e12 / peak, 4),
                     "traffic": kernel_traffic(os.path.join(ROOT, "paged_kv_cache_384_b200", "csrc", "pa_prefill_tc.cu"),
                                               "prefill_tc_traffic.json", args.workload),
                     "peak_source": peak_kind, "kernel": "prefill_tc_kernel",
                     "kernel_ms": round(1e3 * attn_sec, 4)},
        "cpu_baseline": None,
        "e2e": {"value": round(flops / e2e_sec / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": nbytes(q) + nbytes(k_new) + nbytes(v_new), "d2h_bytes_per_step": nbytes(out)},
        "gpu_launches": 2 * args.steps, "clocks": clocks.summary(), "device_errors": errs,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other decode workloads that a default run measures after the metric's own")
    ap.add_argument("--workload", default=PRESET, choices=["llama70b_fp16", "chat_prefix_bf16", "sliding_window_fp16",
                                                           "llama70b_gqa_fp16", "llama70b_int8", "llama70b_fp8",
                                                           "llama70b_gqa_int8", "llama70b_gqa_fp8", "swap_llama70b_fp16",
                                                           *PREFILL],
                    help="secondary workloads are for study; the metric is quoted on the default")
    ap.add_argument("--block-size", type=int, default=None)
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)  # timing rule: at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "swap_llama70b_fp16":
        return run_swap(args)
    if args.workload in PREFILL:
        return run_prefill(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
