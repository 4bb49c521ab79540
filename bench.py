"""Benchmark of the paged decode step on B200: KV GB/s (fraction of HBM peak) and seq-steps/s.

One step = ``pa_write_kv`` of each sequence's new token, then ``pa_decode`` over
the block-paged cache (all kernels of the hot path), on seeded synthetic data.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

N > 1 is launched by torchrun (one rank per GPU): each rank owns an independent
batch of the same shape (weak scaling, no data-path collective); timing is the
max over ranks.  ``--impl reference`` times the fp64 CPU oracle on host cores
on a bounded sample of the same workload.  Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "paged decode attention KV GB/s (fraction of HBM peak) and seq-steps/s, 1×B200"
DEFAULT_WORKLOAD = "llama2_7b_decode"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
SEEDS = {"tiny_decode": 1, "llama2_7b_decode": 2, "gqa_llama3_decode": 3, "long_context_splitk": 4,
         "shared_prefix_step": 5}


# Block operations on a Llama-2-7B-shaped pool (32 kv heads, 16-token blocks,
# head_dim 128, fp16: 128 KiB per block and cache).  copy_blocks is the
# copy-on-write copy inside the device pool; swap_out / swap_in move blocks to
# and from a pinned host pool (preemption).
BLOCK_OPS = {"copy_blocks": 2048, "swap_out": 1024, "swap_in": 1024}
BLOCK_POOL = {"num_blocks": 8192, "num_kv_heads": 32, "block_size": 16, "head_dim": 128, "dtype": "fp16"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.NAMED))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--op", default="decode", choices=["decode", "prefill"] + sorted(BLOCK_OPS),
                    help="decode step (default), paged prefill, or one of the block operations")
    ap.add_argument("--prefill-workload", default="llama2_7b_prefill", choices=sorted(W.PREFILL_NAMED))
    ap.add_argument("--pairs", type=int, default=None, help="block pairs per step (block operations)")
    ap.add_argument("--partition-tokens", type=int, default=0)
    ap.add_argument("--cascade", default="auto", choices=["auto", "on", "off"],
                    help="decode through pa_decode_cascade (prefix groups found on the host from the step's tables); "
                         "auto: when the batch has groups and no fixed partition is asked for")
    ap.add_argument("--cascade-chunk", type=int, default=0,
                    help="tokens per cascade job along the context (0: the library's default, 320)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-seconds", type=float, default=10.0,
                    help="seconds of oracle work per CPU leg (single thread, then all cores)")
    ap.add_argument("--l2-flush", default="auto", choices=["auto", "on", "off"],
                    help="auto: write a scratch buffer larger than L2 before every timed step when the step's "
                         "distinct bytes would fit in L2, else time steps back to back (inputs larger than L2)")
    ap.add_argument("--no-graph", action="store_true",
                    help="time direct library calls instead of replays of a CUDA graph of the step")
    ap.add_argument("--iters", type=int, default=100, help="per-iteration timings (median, p10, p90)")
    ap.add_argument("--num-seqs", type=int, default=None, help="override (llama2/gqa workloads; profiling)")
    ap.add_argument("--num-blocks", type=int, default=None, help="override (llama2/gqa workloads; profiling)")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def make_workload(name: str, rank: int, num_seqs=None, num_blocks=None):
    kw = {}
    if num_seqs is not None:
        kw["num_seqs"] = num_seqs
    if num_blocks is not None:
        kw["num_blocks"] = num_blocks
    return W.NAMED[name](seed=SEEDS[name] + 1000 * rank, **kw)


def step_bytes(wl, st):
    """Algorithmic bytes of one decode call: K and V of exactly the live tokens, q, out,
    the table entries read and the lengths (partial-block slack not counted)."""
    elem = 2
    kv = W.kv_bytes(st, wl.num_kv_heads, wl.head_dim, elem)
    qo = 2 * st.num_seqs * wl.num_q_heads * wl.head_dim * elem
    nblk = int(sum(-(-int(L) // wl.block_size) for L in st.context_lens))
    return kv, kv + qo + 4 * nblk + 4 * st.num_seqs


def recorded_traffic(workload: str, path: str | None = None):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary, or (None, reason)
    when the kernel sources changed since the capture or the workload was not captured.  ``path``
    selects a record of another decode path (``"cascade"``), kept under that key with its own sources."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "decode_traffic.json")) as f:
            rec = json.load(f)
        if path is not None:
            rec = rec[path]
        h = hashlib.sha256()
        for rel in rec["kernel_sources"]:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["kernel_sources_sha256"]:
            return None, "kernel changed since the ncu capture"
        w = rec["workloads"].get(workload)
        if w is None:
            return None, "no ncu capture for this workload"
        return int(w["dram_bytes_per_launch"]), w["kernel"] + ": " + w["how"]
    except (OSError, KeyError, ValueError) as e:
        return None, f"no traffic record ({type(e).__name__})"


def cascade_wanted(mode: str, num_groups: int, partition_tokens: int) -> bool:
    """Whether the decode step runs through pa_decode_cascade: always with ``on``; with ``auto`` when the
    host found prefix groups in the step's tables and no fixed partition was asked for (a partition
    length is a parameter of pa_decode's split, which the cascade plan does not take)."""
    return mode == "on" or (mode == "auto" and num_groups > 0 and partition_tokens == 0)


def max_over_ranks(values, device=None):
    """Elementwise maximum of per-rank timings (ms) over all ranks; identity on one rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_rate_gbs(bytes_per_rank_step: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: every rank moves bytes_per_rank_step per step; time = slowest rank."""
    return world * bytes_per_rank_step * steps / (max_ms / 1e3) / 1e9


def summarize_ms(times_ms):
    """Median, p10, p90 and mean (microseconds) of per-iteration times given in milliseconds."""
    a = np.asarray(times_ms, dtype=np.float64) * 1e3
    if a.size == 0:
        return None
    return {"median_us": round(float(np.median(a)), 3), "p10_us": round(float(np.percentile(a, 10)), 3),
            "p90_us": round(float(np.percentile(a, 90)), 3), "mean_us": round(float(a.mean()), 3), "n": int(a.size)}


def flush_needed(mode: str, distinct_bytes: int, l2_bytes: int) -> bool:
    """Whether timed steps must be separated by an L2 flush: always ("on"), never ("off"), or when
    the bytes one step reads (each distinct byte once) are not several times the L2 ("auto")."""
    if mode == "on":
        return True
    if mode == "off":
        return False
    return distinct_bytes < 4 * l2_bytes


def l2_note(flush: bool, distinct_bytes: int, l2_bytes: int, flush_bytes: int) -> str:
    size = f"{distinct_bytes / 1e6:.1f} MB of distinct inputs per step against a {l2_bytes / 1e6:.0f} MB L2"
    if flush:
        return (f"flushed: a {flush_bytes / 2**20:.0f} MiB scratch write and read-back before every timed step "
                f"({size})")
    return f"no flush: {size}, steps back to back"


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only) in a thread."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device, period_s: float = 0.01):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            import torch
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = repr(e)
        self.t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        n = self.nvml
        get_reasons = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            n.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append((time.perf_counter(), n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM),
                                     int(get_reasons(self.h))))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t.start()
        return self

    def stop(self):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"error": self.err}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        use = inside if len(inside) >= 3 else self.samples
        if not use:
            return {"error": "no samples"}
        mask = 0
        for s in use:
            mask |= s[2]
        return {"sm_mhz": statistics.median(s[1] for s in use), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(k for k, v in self.REASONS.items() if mask & v and k != "gpu_idle"),
                "samples": len(use), "window": "timed region" if use is inside else "whole run"}


def cpu_oracle_rate(wl, st, seconds: float):
    """Times the fp64 C oracle (single thread) on the first sequences of the step, about
    ``seconds`` of work; returns (GB/s of KV it processed, description)."""
    import oracle
    kc, vc = oracle.write_kv(st.k_new, st.v_new, wl.k_cache, wl.v_cache, st.slot_mapping, wl.block_size)
    order = np.arange(st.num_seqs)
    done_bytes, elapsed, n = 0, 0.0, 0
    per_seq = wl.num_kv_heads * wl.head_dim * 2 * 2
    while elapsed < seconds and n < st.num_seqs:
        s = order[n:n + 1]
        t = time.perf_counter()
        oracle.decode(st.q[s], kc, vc, st.block_tables[s], st.context_lens[s], wl.scale, wl.dtype)
        elapsed += time.perf_counter() - t
        done_bytes += int(st.context_lens[s].sum()) * per_seq
        n += 1
    return done_bytes / elapsed / 1e9, n, elapsed


def cpu_oracle_rate_parallel(wl, st, seconds: float):
    """Times the OpenMP build of the fp64 C oracle on all host cores: batches of one sequence per
    thread, rotating through the step, until about ``seconds`` have passed; returns
    (GB/s of KV it processed, threads, description)."""
    import oracle
    kc, vc = oracle.write_kv(st.k_new, st.v_new, wl.k_cache, wl.v_cache, st.slot_mapping, wl.block_size)
    threads = oracle.parallel_threads()
    per_seq = wl.num_kv_heads * wl.head_dim * 2 * 2
    batch = max(1, min(threads, st.num_seqs))
    done_bytes, elapsed, calls, seqs = 0, 0.0, 0, 0
    while elapsed < seconds:
        idx = (np.arange(batch) + calls * batch) % st.num_seqs
        t = time.perf_counter()
        oracle.decode(st.q[idx], kc, vc, st.block_tables[idx], st.context_lens[idx], wl.scale, wl.dtype,
                      parallel=True)
        elapsed += time.perf_counter() - t
        done_bytes += int(st.context_lens[idx].sum()) * per_seq
        calls += 1
        seqs += batch
    return done_bytes / elapsed / 1e9, threads, (
        f"{seqs} sequence passes ({calls} calls of {batch} sequences, rotating through the {st.num_seqs} of one "
        f"step), {elapsed:.1f} s, {threads} OpenMP threads over (sequence, query head)")


def cpu_baseline(wl, st, seconds: float):
    """The oracle timed on the host: all cores (the reported value) and one thread beside it."""
    rate1, nseq, secs = cpu_oracle_rate(wl, st, seconds)
    rate_n, threads, sample_n = cpu_oracle_rate_parallel(wl, st, seconds)
    return {"value": round(rate_n, 4), "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample_n,
            "host_cores_in_affinity": len(os.sched_getaffinity(0)),
            "single_thread": {"value": round(rate1, 4), "unit": "GB/s", "cores": 1,
                              "sample": f"first {nseq} of {st.num_seqs} sequences of one step, {secs:.1f} s"}}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    wl = make_workload(args.workload, 0)
    st = wl.steps[0]
    import oracle
    kc, vc = oracle.write_kv(st.k_new, st.v_new, wl.k_cache, wl.v_cache, st.slot_mapping, wl.block_size)
    per_seq = wl.num_kv_heads * wl.head_dim * 2 * 2
    threads = oracle.parallel_threads()
    # one step = the oracle on all host cores over a sample of one sequence per thread (rotating through
    # the batch), so the work per step stays bounded whatever the workload
    sample = max(1, min(threads, st.num_seqs))
    times, nbytes = [], []
    for i in range(args.warmup + args.steps):
        idx = (np.arange(sample) + i * sample) % st.num_seqs
        t = time.perf_counter()
        oracle.decode(st.q[idx], kc, vc, st.block_tables[idx], st.context_lens[idx], wl.scale, wl.dtype,
                      parallel=True)
        dt = time.perf_counter() - t
        if i >= args.warmup:
            times.append(dt)
            nbytes.append(int(st.context_lens[idx].sum()) * per_seq)
    total_t = sum(times)
    value = sum(nbytes) / total_t / 1e9
    desc = f"{sample} of {st.num_seqs} sequences per step, rotating; {threads} OpenMP threads"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total_t / len(times), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "description": wl.description, "sample": desc},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": desc, "host_cores_in_affinity": len(os.sched_getaffinity(0))},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def block_op_pairs(op: str, pairs: int, num_blocks: int, host_blocks: int, seed: int):
    """(source, destination) pairs: distinct destinations, none of them a source of another pair."""
    rng = np.random.default_rng(seed)
    if op == "copy_blocks":
        ids = rng.permutation(num_blocks)[: 2 * pairs]
        return np.stack([ids[:pairs], ids[pairs:]], axis=1).astype(np.int64)
    dev = rng.permutation(num_blocks)[:pairs]
    host = rng.permutation(host_blocks)[:pairs]
    pair = (dev, host) if op == "swap_out" else (host, dev)
    return np.stack(pair, axis=1).astype(np.int64)


def oracle_copy_rate(op: str, seconds: float):
    """The oracle's block copy on host arrays: GB/s of block bytes moved (K and V), bounded sample."""
    import oracle
    g = BLOCK_POOL
    nb, pairs = 256, 64
    rng = np.random.default_rng(17)
    shape = (nb, g["num_kv_heads"], g["block_size"], g["head_dim"])
    k = rng.integers(0, 1 << 16, size=shape, dtype=np.uint16)
    v = rng.integers(0, 1 << 16, size=shape, dtype=np.uint16)
    m = block_op_pairs("copy_blocks", pairs, nb, nb, 3)
    per_pair = 2 * int(np.prod(shape[1:])) * 2
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle.copy_blocks(k, v, k, v, m)
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    secs = time.perf_counter() - t0
    return n * pairs * per_pair / secs / 1e9, f"{n} calls of {pairs} pairs on a {nb}-block host pool, {secs:.1f} s"


def run_block_op(args):
    """Times copy_blocks / swap_out / swap_in through the C ABI; prints one JSON line."""
    import torch
    import torch.distributed as dist

    import paged_kv_cache_457_b200 as pa

    rank, world, local_rank = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    pa.load_library()
    g = BLOCK_POOL
    op = args.op
    pairs = args.pairs or BLOCK_OPS[op]
    nb = args.num_blocks or g["num_blocks"]
    shape = (g["num_kv_heads"], g["block_size"], g["head_dim"])
    block_bytes = int(np.prod(shape)) * 2
    gen = torch.Generator(device=device).manual_seed(100 + rank)
    k_cache = torch.randint(-32768, 32767, (nb,) + shape, dtype=torch.int16, device=device, generator=gen)
    v_cache = torch.randint(-32768, 32767, (nb,) + shape, dtype=torch.int16, device=device, generator=gen)
    k_cache, v_cache = k_cache.view(torch.float16), v_cache.view(torch.float16)
    host_blocks = pairs
    m_np = block_op_pairs(op, pairs, nb, host_blocks, 7 + rank)
    mapping = torch.from_numpy(m_np).to(device)
    if op == "copy_blocks":
        call = lambda mp: pa.copy_blocks(k_cache, v_cache, mp)  # noqa: E731
        host_k = host_v = None
    else:
        host_k = torch.empty((host_blocks,) + shape, dtype=torch.float16, pin_memory=True)
        host_v = torch.empty((host_blocks,) + shape, dtype=torch.float16, pin_memory=True)
        if op == "swap_out":
            call = lambda mp: pa.swap_blocks(k_cache, v_cache, host_k, host_v, mp)  # noqa: E731
        else:
            call = lambda mp: pa.swap_blocks(host_k, host_v, k_cache, v_cache, mp, device=device)  # noqa: E731
    moved = 2 * pairs * block_bytes  # K and V blocks per step
    torch.cuda.synchronize()
    sampler = ClockSampler(device).start()
    for _ in range(args.warmup):
        call(mapping)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = pa.launch_count()
    wall0 = time.perf_counter()
    e0.record()
    for _ in range(args.steps):
        call(mapping)
    e1.record()
    torch.cuda.synchronize()
    wall1 = time.perf_counter()
    launches = pa.launch_count() - launches0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.stop()
    ms = e0.elapsed_time(e1) / args.steps

    # End to end: the mapping comes from pinned host memory each step, the status word goes back.
    host_map = torch.from_numpy(m_np).pin_memory()
    status_host = torch.zeros(1, dtype=torch.int32, pin_memory=True)
    dmap = torch.empty_like(mapping)

    def e2e_step():
        dmap.copy_(host_map, non_blocking=True)
        call(dmap)
        status_host.copy_(torch.zeros(1, dtype=torch.int32, device=device), non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(args.steps):
        e2e_step()
    f1.record()
    torch.cuda.synchronize()
    e2e_ms = f0.elapsed_time(f1) / args.steps

    # The link's own rate for the swap legs: one contiguous pinned copy of the same bytes.
    link = None
    if op != "copy_blocks":
        flat_dev = k_cache.view(-1)[: moved // 2]
        flat_host = torch.empty(moved // 2, dtype=torch.float16, pin_memory=True)
        for _ in range(3):
            (flat_host.copy_(flat_dev, non_blocking=True) if op == "swap_out"
             else flat_dev.copy_(flat_host, non_blocking=True))
        torch.cuda.synchronize()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record()
        for _ in range(args.steps):
            (flat_host.copy_(flat_dev, non_blocking=True) if op == "swap_out"
             else flat_dev.copy_(flat_host, non_blocking=True))
        c1.record()
        torch.cuda.synchronize()
        link = (moved // 2 * 2) / (c0.elapsed_time(c1) / args.steps / 1e3) / 1e9
    status = pa.device_status()
    ms, e2e_ms = max_over_ranks([ms, e2e_ms], device)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, sample = oracle_copy_rate(op, min(args.cpu_sample_seconds, 5.0))
        cpu = {"value": round(rate, 3), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample}
    if rank == 0:
        value = world * moved / (ms / 1e3) / 1e9
        if op == "copy_blocks":
            peak, peak_kind = measured_peak()
            achieved = 2 * moved / (ms / 1e3) / 1e9  # read + write, as the copy peak counts them
            roof = {"bound": "hbm", "kernel": "copy_blocks_kernel", "achieved": round(achieved, 1),
                    "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                    "traffic": None, "algorithmic_bytes": 2 * moved, "ms_per_launch": round(ms, 5)}
        else:
            achieved = moved / (ms / 1e3) / 1e9
            roof = {"bound": "host link", "kernel": "copy_blocks_kernel", "achieved": round(achieved, 1),
                    "peak": round(link, 1), "peak_kind": "measured in this run: one contiguous pinned "
                    + ("device-to-host" if op == "swap_out" else "host-to-device") + " copy of the same bytes",
                    "unit": "GB/s", "frac": round(achieved / link, 4), "traffic": None,
                    "algorithmic_bytes": moved, "ms_per_launch": round(ms, 5)}
        line = {
            "metric": f"{op} block bytes moved GB/s, 1×B200", "value": round(value, 2), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u16",
            "data": "synthetic",
            "config": {"workload": f"{op}: {pairs} block pairs, Llama-2-7B pool geometry",
                       "num_blocks": nb, "num_kv_heads": g["num_kv_heads"], "block_size": g["block_size"],
                       "head_dim": g["head_dim"], "storage_dtype": g["dtype"], "pairs": pairs,
                       "bytes_moved_per_step": moved, "parallelism": f"dp{world} (independent pools per GPU)",
                       "l2": f"no flush: {moved / 2**20:.0f} MiB moved per step, larger than the 126 MB L2"},
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": round(world * moved / (e2e_ms / 1e3) / 1e9, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": int(m_np.nbytes), "d2h_bytes_per_step": 4,
                    "ms_per_step": round(e2e_ms, 4)},
            "gpu_launches": int(launches), "clocks": sampler.summary(wall0, wall1), "device_status": status,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (cuBLAS bf16 burst; fp16 has the same nominal rate)"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def oracle_prefill_rate(case, seconds: float):
    """The oracle on the shortest sequences of the case, one after another, until `seconds` pass."""
    import oracle
    qs, lens = case.query_start, case.context_lens
    order = np.argsort(lens)
    flops, done, t0 = 0, 0, time.perf_counter()
    for s in order:
        s = int(s)
        n = int(qs[s + 1] - qs[s])
        L = int(lens[s])
        oracle.prefill(case.q[qs[s]:qs[s + 1]], case.k_cache, case.v_cache, case.block_tables[s:s + 1],
                       np.array([0, n], np.int32), lens[s:s + 1], case.scale, case.dtype)
        flops += 4 * case.head_dim * case.num_q_heads * (n * (L - n) + n * (n + 1) // 2)
        done += 1
        if time.perf_counter() - t0 >= seconds:
            break
    secs = time.perf_counter() - t0
    return flops / secs / 1e12, f"{done} of {case.num_seqs} sequences (shortest first), {secs:.1f} s, single thread"


def run_prefill_op(args):
    """Times pa_prefill on a named prefill configuration; prints one JSON line."""
    import torch
    import torch.distributed as dist

    import paged_kv_cache_457_b200 as pa

    rank, world, local_rank = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    pa.load_library()
    case = W.PREFILL_NAMED[args.prefill_workload](seed=6 + 100 * rank if args.prefill_workload == "llama2_7b_prefill"
                                                  else 7 + 100 * rank)
    tdt = torch.float16 if case.dtype == "fp16" else torch.bfloat16

    def dev_bits(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(tdt)

    kc, vc, q = dev_bits(case.k_cache), dev_bits(case.v_cache), dev_bits(case.q)
    tables = torch.from_numpy(case.block_tables).to(device)
    qs = torch.from_numpy(case.query_start).to(device)
    lens = torch.from_numpy(case.context_lens).to(device)
    out = torch.empty_like(q)
    mql = case.max_query_len
    flops = 4 * case.head_dim * case.num_q_heads * case.attended_pairs

    def step(qq=q, ss=qs, ll=lens, tt=tables):
        pa.prefill(qq, kc, vc, tt, ss, ll, case.scale, mql, out=out)

    torch.cuda.synchronize()
    sampler = ClockSampler(device).start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = pa.launch_count()
    wall0 = time.perf_counter()
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    wall1 = time.perf_counter()
    launches = pa.launch_count() - launches0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.stop()
    ms = e0.elapsed_time(e1) / args.steps
    status = pa.device_status()

    def measure_e2e():
        # end to end: q and the batch metadata from pinned host memory, the output back to pinned host memory
        hq_ = torch.from_numpy(case.q.view(np.int16)).pin_memory()
        hmeta = [torch.from_numpy(a).pin_memory() for a in (case.query_start, case.context_lens, case.block_tables)]
        out_host = torch.empty(out.shape, dtype=torch.int16).pin_memory()
        # double-buffered: step k's copies in and out overlap step k-1's kernel (two copy streams)
        bufs = [dict(q=torch.empty_like(q), qs=torch.empty_like(qs), lens=torch.empty_like(lens),
                     tables=torch.empty_like(tables), out=torch.empty_like(out)) for _ in range(2)]
        out_hosts = [out_host, torch.empty(out.shape, dtype=torch.int16).pin_memory()]
        h2d_stream, d2h_stream = torch.cuda.Stream(device), torch.cuda.Stream(device)
        compute = torch.cuda.current_stream(device)
        ready = [torch.cuda.Event() for _ in range(2)]
        computed = [torch.cuda.Event() for _ in range(2)]
        drained = [torch.cuda.Event() for _ in range(2)]
        for b in range(2):
            computed[b].record(compute)
            drained[b].record(compute)
        counter = [0]

        def e2e_step():
            b = counter[0] & 1
            counter[0] += 1
            buf = bufs[b]
            with torch.cuda.stream(h2d_stream):
                h2d_stream.wait_event(computed[b])
                buf["q"].view(torch.int16).copy_(hq_, non_blocking=True)
                buf["qs"].copy_(hmeta[0], non_blocking=True)
                buf["lens"].copy_(hmeta[1], non_blocking=True)
                buf["tables"].copy_(hmeta[2], non_blocking=True)
                ready[b].record(h2d_stream)
            compute.wait_event(ready[b])
            compute.wait_event(drained[b])
            pa.prefill(buf["q"], kc, vc, buf["tables"], buf["qs"], buf["lens"], case.scale, mql, out=buf["out"])
            computed[b].record(compute)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(computed[b])
                out_hosts[b].copy_(buf["out"].view(torch.int16), non_blocking=True)
                drained[b].record(d2h_stream)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(compute)
        h2d_stream.wait_event(f0)
        d2h_stream.wait_event(f0)
        for _ in range(args.steps):
            e2e_step()
        for b in range(2):
            compute.wait_event(drained[b])
        f1.record(compute)
        torch.cuda.synchronize()
        return f0.elapsed_time(f1) / args.steps, hq_.numel() * 2 + sum(t.numel() * t.element_size() for t in hmeta), \
            out_host.numel() * 2

    if args.no_e2e:
        e2e_ms, h2d, d2h = None, 0, 0
        ms = max_over_ranks([ms], device)[0]
    else:
        e2e_ms, h2d, d2h = measure_e2e()
        ms, e2e_ms = max_over_ranks([ms, e2e_ms], device)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, sample = oracle_prefill_rate(case, min(args.cpu_sample_seconds, 10.0))
        cpu = {"value": round(rate, 6), "unit": "TFLOP/s", "cores": 1, "kind": "oracle", "sample": sample}
    if rank == 0:
        peak, peak_kind = measured_tensor_peak()
        achieved = flops / (ms / 1e3) / 1e12
        line = {
            "metric": "paged causal prefill attention TFLOP/s (fraction of tensor peak), 1×B200",
            "value": round(world * achieved, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": case.dtype, "data": "synthetic",
            "tokens_per_s": round(world * int(case.query_start[-1]) / (ms / 1e3), 1),
            "config": {"workload": case.name, "description": case.description, "num_seqs": case.num_seqs,
                       "new_tokens": int(case.query_start[-1]), "attended_pairs": case.attended_pairs,
                       "num_q_heads": case.num_q_heads, "num_kv_heads": case.num_kv_heads,
                       "head_dim": case.head_dim, "block_size": case.block_size,
                       "parallelism": f"dp{world} (independent batches per GPU)",
                       "l2": "no flush: K/V of the batch exceed the 126 MB L2"},
            "roofline": {"bound": "tensor", "kernel": "prefill_tc_kernel", "achieved": round(achieved, 1),
                         "peak": peak, "peak_kind": peak_kind, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                         "traffic": None, "algorithmic_flops": flops, "ms_per_launch": round(ms, 5)},
            "cpu_baseline": cpu,
            "e2e": None if e2e_ms is None else {
                    "value": round(world * flops / (e2e_ms / 1e3) / 1e12, 2), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "ms_per_step": round(e2e_ms, 4),
                    "how": "q and metadata copied in, the output read back, double-buffered on two copy streams "
                           "that overlap the previous step's kernel; bound by the host link (~150 MB each way)"},
            "gpu_launches": int(launches), "clocks": sampler.summary(wall0, wall1), "device_status": status,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "prefill":
        return run_prefill_op(args)
    if args.op != "decode":
        return run_block_op(args)

    import torch
    import torch.distributed as dist

    import paged_kv_cache_457_b200 as pa

    rank, world, local_rank = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    pa.load_library()

    wl = make_workload(args.workload, rank, args.num_seqs, args.num_blocks)
    if len(wl.steps) != 1:
        steps_used = wl.steps[1:2]  # steady-state decode step of the multi-step workload
    else:
        steps_used = wl.steps
    st = steps_used[0]
    tdt = torch.float16 if wl.dtype == "fp16" else torch.bfloat16

    def dev_bits(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(tdt)

    k_cache = dev_bits(wl.k_cache)
    v_cache = dev_bits(wl.v_cache)
    if len(wl.steps) != 1:  # bring the cache to the state before the timed step
        for prev in wl.steps[:1]:
            pa.write_kv(dev_bits(prev.k_new), dev_bits(prev.v_new), k_cache, v_cache,
                        torch.from_numpy(prev.slot_mapping).to(device))
    q = dev_bits(st.q)
    k_new = dev_bits(st.k_new)
    v_new = dev_bits(st.v_new)
    slots = torch.from_numpy(st.slot_mapping).to(device)
    tables = torch.from_numpy(st.block_tables).to(device)
    lens = torch.from_numpy(st.context_lens).to(device)
    out = torch.empty_like(q)
    mcl = st.max_context_len
    part = args.partition_tokens
    ws_bytes = pa.decode_workspace_size(st.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
                                        mcl, part)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device)

    # Shared leading blocks: the host finds the groups from the step's tables (as a scheduler would) and the
    # cascade path reads each group's shared tiles once.
    groups = pa.find_prefix_groups(st.block_tables, st.context_lens, wl.block_size)
    use_cascade = cascade_wanted(args.cascade, groups.num_groups, part)
    if use_cascade:
        plan = pa.cascade_plan(st.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.block_size, mcl, groups,
                               chunk_tokens=args.cascade_chunk)
        plan_dev = plan.to(device)
        cws = torch.empty(max(pa.cascade_workspace_size(plan, wl.head_dim), 16), dtype=torch.uint8, device=device)

    def decode_into(q_, tables_, lens_, out_, plan_dev_=None):
        if use_cascade:
            pa.decode_cascade(q_, k_cache, v_cache, tables_, lens_, wl.scale, plan,
                              plan_dev if plan_dev_ is None else plan_dev_, out=out_, workspace=cws)
        else:
            pa.decode(q_, k_cache, v_cache, tables_, lens_, wl.scale, max_context_len=mcl, out=out_,
                      partition_tokens=part, workspace=ws)

    def step():
        pa.write_kv(k_new, v_new, k_cache, v_cache, slots)
        decode_into(q, tables, lens, out)

    def decode_only():
        decode_into(q, tables, lens, out)

    kv_b, alg_b = step_bytes(wl, st)
    uniq_kv = W.unique_kv_bytes(st, wl.num_kv_heads, wl.head_dim, wl.block_size)
    alg_unique = alg_b - kv_b + uniq_kv  # shared prefix blocks counted once: what must come from HBM
    l2_bytes = int(torch.cuda.get_device_properties(device).L2_cache_size)
    flush = flush_needed(args.l2_flush, alg_unique, l2_bytes)
    flush_bytes = max(512 * 2**20, 4 * l2_bytes)
    flush_buf = torch.empty(flush_bytes, dtype=torch.uint8, device=device) if flush else None
    torch.cuda.synchronize()
    assert pa.device_status() == 0, "device status after setup"

    # The step as a CUDA graph (default): one replay re-runs the library's kernels with the captured
    # arguments, so the host's per-call cost (argument checks, ctypes) is paid once, at capture.
    reference_out = None
    launches_per_step = 3
    if not args.no_graph:
        step()
        torch.cuda.synchronize()
        reference_out = out.clone()
        graph = torch.cuda.CUDAGraph()
        n0 = pa.launch_count()
        with torch.cuda.graph(graph):
            step()
        launches_per_step = pa.launch_count() - n0
        run_step = graph.replay
    else:
        run_step = step

    def prime():
        # a GPU-side wait ahead of the timed region, so the host enqueues the timed steps while the GPU is
        # busy: the clock then measures the GPU's work, not the host's launch rate
        torch.cuda._sleep(50_000_000)

    flush_sink = torch.zeros(1, dtype=torch.int32, device=device)

    def flush_l2(i):
        # write a buffer several times the L2, then read it back: the read pass evicts the written lines
        # (their write-back to HBM happens here, not inside the timed step), so L2 holds only clean
        # lines of the scratch buffer when the step starts
        flush_buf.fill_(i & 0x7f)
        pa.read_bandwidth_probe(flush_buf, flush_sink)

    def timed_per_iteration(fn, n, cold):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        prime()
        for i in range(n):
            if cold:
                flush_l2(i)
            evs[i][0].record()
            fn()
            evs[i][1].record()
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    sampler = ClockSampler(device).start()
    for _ in range(args.warmup):
        run_step()
    torch.cuda.synchronize()
    if reference_out is not None:
        assert torch.equal(out, reference_out), "graph replay differs from the direct call"
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = pa.launch_count()
    wall0 = time.perf_counter()
    if flush:
        step_times = timed_per_iteration(run_step, args.steps, cold=True)
        elapsed_ms = float(sum(step_times))
    else:
        prime()
        t_start.record()
        for _ in range(args.steps):
            run_step()
        t_end.record()
        torch.cuda.synchronize()
        elapsed_ms = t_start.elapsed_time(t_end)
        step_times = None
    wall1 = time.perf_counter()
    launches = pa.launch_count() - launches0
    if flush:
        launches -= args.steps  # the flush's read-back pass between steps is not part of a step
    if not args.no_graph:
        launches = launches_per_step * args.steps  # replays do not pass through the host-side counter
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.stop()

    # pa_decode alone (split + merge kernels), the roofline's kernel: back to back, then per iteration with
    # and without an L2 flush before each call
    if not args.no_graph:
        dgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(dgraph):
            decode_only()
        run_decode = dgraph.replay
    else:
        run_decode = decode_only
    for _ in range(3):
        run_decode()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    prime()
    d0.record()
    for _ in range(args.steps):
        run_decode()
    d1.record()
    torch.cuda.synchronize()
    dec_b2b_ms = d0.elapsed_time(d1) / args.steps
    if flush_buf is None:
        flush_buf = torch.empty(flush_bytes, dtype=torch.uint8, device=device)
    cold = timed_per_iteration(run_decode, args.iters, cold=True)
    warm = timed_per_iteration(run_decode, args.iters, cold=False)
    dec_ms = float(np.mean(cold)) if flush else dec_b2b_ms
    del flush_buf
    status = pa.device_status()

    # read-only streaming rate of this GPU, measured now by the library's own probe kernel
    probe_bytes = max(2 * 2**30, 8 * l2_bytes)
    probe_buf = torch.empty(probe_bytes, dtype=torch.uint8, device=device)
    sink = torch.zeros(1, dtype=torch.int32, device=device)
    for _ in range(3):
        pa.read_bandwidth_probe(probe_buf, sink)
    probe_ms = timed_per_iteration(lambda: pa.read_bandwidth_probe(probe_buf, sink), 20, cold=False)
    read_peak = probe_bytes / (min(probe_ms) / 1e3) / 1e9
    del probe_buf

    # ---- end to end through the public API: pinned host inputs -> device -> step -> host output
    e2e = None
    if not args.no_e2e:
        # A step's inputs packed into one pinned buffer (each at a 256-byte offset) and moved by one copy,
        # as a serving loop would: one transfer per step instead of one per tensor keeps the host ahead.
        parts = [("q", st.q, q), ("k", st.k_new, k_new), ("v", st.v_new, v_new), ("slots", st.slot_mapping, slots),
                 ("tables", st.block_tables, tables), ("lens", st.context_lens, lens)]
        if use_cascade:
            parts.append(("plan", plan.plan, plan_dev))
        offsets, total = {}, 0
        for n, arr, _ in parts:
            offsets[n] = total
            total += -(-np.ascontiguousarray(arr).nbytes // 256) * 256
        host_packed = torch.zeros(total, dtype=torch.uint8).pin_memory()
        for n, arr, _ in parts:
            raw = np.ascontiguousarray(arr).view(np.uint8).reshape(-1)
            host_packed[offsets[n]:offsets[n] + raw.size].copy_(torch.from_numpy(raw))
        out_host = torch.empty(out.shape, dtype=torch.int16).pin_memory()
        h2d = total
        d2h = out_host.numel() * out_host.element_size()

        def views(packed):
            v = {}
            for n, arr, like in parts:
                nb = np.ascontiguousarray(arr).nbytes
                v[n] = packed[offsets[n]:offsets[n] + nb].view(like.dtype).view(like.shape)
            return v
        # Two sets of device inputs and outputs: step k's inputs are copied in on one stream and its
        # output read back on another while the compute stream runs step k-1, as a serving loop would.
        packs = [torch.empty(total, dtype=torch.uint8, device=device) for _ in range(2)]
        bufs = [dict(views(packs[i]), out=torch.empty_like(out), packed=packs[i]) for i in range(2)]
        out_hosts = [out_host, torch.empty(out.shape, dtype=torch.int16).pin_memory()]
        h2d_stream, d2h_stream = torch.cuda.Stream(device), torch.cuda.Stream(device)
        compute = torch.cuda.current_stream(device)
        ready = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer b copied in
        computed = [torch.cuda.Event() for _ in range(2)]  # step on buffer b done (its inputs free)
        drained = [torch.cuda.Event() for _ in range(2)]   # output of buffer b copied out
        for b in range(2):
            computed[b].record(compute)
            drained[b].record(compute)
        counter = [0]

        def e2e_step():
            b = counter[0] & 1
            counter[0] += 1
            buf = bufs[b]
            with torch.cuda.stream(h2d_stream):
                h2d_stream.wait_event(computed[b])
                buf["packed"].copy_(host_packed, non_blocking=True)
                ready[b].record(h2d_stream)
            compute.wait_event(ready[b])
            compute.wait_event(drained[b])
            pa.write_kv(buf["k"], buf["v"], k_cache, v_cache, buf["slots"])
            decode_into(buf["q"], buf["tables"], buf["lens"], buf["out"], buf.get("plan"))
            computed[b].record(compute)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(computed[b])
                out_hosts[b].copy_(buf["out"].view(torch.int16), non_blocking=True)
                drained[b].record(d2h_stream)

        for _ in range(max(3, args.warmup // 4)):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(compute)
        h2d_stream.wait_event(e0)
        d2h_stream.wait_event(e0)
        for _ in range(args.steps):
            e2e_step()
        for b in range(2):  # the last outputs are on the host before the clock stops
            compute.wait_event(drained[b])
        e1.record(compute)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1)], device)[0]
        e2e = {"value": round(job_rate_gbs(kv_b, world, args.steps, e2e_ms), 2), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e2e_ms / args.steps, 4),
               "how": "each step's inputs copied from one pinned host buffer (one copy per step) and its output "
                      "read back, on two copy streams, double-buffered so that they overlap the previous step's "
                      "kernels" + ("; the cascade plan is among the copied inputs (built on the host once for the "
                                   "batch's groups, as a scheduler rebuilds it only when a group changes)"
                                   if use_cascade else "")}

    elapsed_ms, dec_ms, read_peak_neg = max_over_ranks([elapsed_ms, dec_ms, -read_peak], device)
    read_peak = -read_peak_neg  # the slowest rank's probe

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, st, args.cpu_sample_seconds)

    if rank == 0:
        ms_step = elapsed_ms / args.steps
        value = job_rate_gbs(kv_b, world, args.steps, elapsed_ms)
        value_distinct = job_rate_gbs(uniq_kv, world, args.steps, elapsed_ms)
        peak, peak_kind = measured_peak()
        achieved = alg_unique / (dec_ms / 1e3) / 1e9
        traffic, traffic_note = recorded_traffic(wl.name, "cascade" if use_cascade else None)
        shared = uniq_kv != kv_b
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "storage_dtype": wl.dtype, "data": "synthetic",
            "seq_steps_per_s": round(world * st.num_seqs / (ms_step / 1e3), 1),
            "distinct_kv_gbs": round(value_distinct, 2),
            "frac_of_hbm_peak": round(value_distinct / world / peak, 4),
            "frac_of_read_only_peak": round(value_distinct / world / read_peak, 4),
            "frac_of_8tbs": round(value_distinct / world / NOMINAL_HBM_GBS, 4),
            "config": {"workload": wl.name, "description": wl.description, "num_seqs": st.num_seqs,
                       "num_q_heads": wl.num_q_heads, "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
                       "block_size": wl.block_size, "max_context_len": mcl,
                       "split": (f"cascade plan: {plan.info.num_prefix_jobs} prefix jobs (a group's shared tiles), "
                                 f"{plan.info.num_jobs - plan.info.num_prefix_jobs} suffix jobs, "
                                 f"{plan.info.num_pieces} partial states to combine") if use_cascade else
                                (f"chunks of {part} tokens" if part else
                                 "one block per (sequence, kv head) segment, no workspace (small batch)"
                                 if ws_bytes == 0 else
                                 "balanced tile stream cut into chunks, one queue of chunks shared by the warps"),
                       "kv_bytes_per_step": kv_b, "distinct_kv_bytes_per_step": uniq_kv,
                       "parallelism": f"dp{world} (independent batches per GPU)",
                       "timing": ("per-step CUDA events, L2 flushed before each step" if flush else
                                  "one CUDA event pair around all steps, back to back")
                       + ((f"; each step a replay of a CUDA graph of pa_write_kv + "
                           f"{'pa_decode_cascade' if use_cascade else 'pa_decode'}") if not args.no_graph
                          else "; direct library calls"),
                       "path": (f"pa_decode_cascade: {groups.num_groups} prefix groups found on the host "
                                f"(sizes {sorted(set(np.diff(groups.offsets).tolist()))}, shared blocks "
                                f"{sorted(set(groups.prefix_blocks.tolist()))}), each shared tile read once per group"
                                if use_cascade else "pa_decode"),
                       "l2": l2_note(flush, alg_unique, l2_bytes, flush_bytes)},
            "step_timing": summarize_ms(step_times) if step_times else None,
            "roofline": {"bound": "hbm", "kernel": ("pa_decode_cascade (partial + combine kernels)" if use_cascade
                                                    else "pa_decode (split + merge kernels)"),
                         "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic, "traffic_note": traffic_note,
                         "algorithmic_bytes": alg_unique,
                         "algorithmic_bytes_note": ("K/V of the distinct physical rows read (a prefix block named by "
                                                    "several tables counted once) + q + out + table entries + lengths"
                                                    if shared else "K/V of the live tokens + q + out + table entries "
                                                    "+ lengths"),
                         "ms_per_launch": round(dec_ms, 5),
                         "launch_timing": "mean of per-call times, L2 flushed before each call" if flush else
                                          "back-to-back calls, mean",
                         "peaks": {
                             "measured_copy": {"gbs": peak, "frac": round(achieved / peak, 4),
                                               "source": "MEASURED_PEAKS.json hbm_gbs (read+write copy)"},
                             "read_only_probe": {"gbs": round(read_peak, 1), "frac": round(achieved / read_peak, 4),
                                                 "source": "pa_read_bandwidth_probe over "
                                                           f"{probe_bytes / 2**30:.1f} GiB, best of 20, this run"},
                             "nominal_8tbs": {"gbs": NOMINAL_HBM_GBS, "frac": round(achieved / NOMINAL_HBM_GBS, 4)}},
                         "logical_bytes": alg_b if shared else None,
                         "logical_rate_note": (f"{alg_b / (dec_ms / 1e3) / 1e9:.1f} GB/s counting every table's "
                                               "reads of the shared prefix; not a fraction of any peak (repeat reads "
                                               "of a block come from L2)") if shared else None},
            "decode_timing": {"back_to_back_us": round(dec_b2b_ms * 1e3, 3), "cold_l2": summarize_ms(cold),
                              "warm_l2": summarize_ms(warm)},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches),
            "clocks": sampler.summary(wall0, wall1), "device_status": status,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
