"""Benchmark of one paged decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config 2] [--mode fused|fused_single|split|single|cascade]
                    [--partition P]   (default 1024 tokens; 512 for config 4)
    python bench.py --config 4 --kv int8 [--channel-scales]   (other 8-bit caches)
    python bench.py --config 5 --mode cascade   (shared prefix attended once)
    python bench.py --op copy_blocks [--config 2] [--pairs 4096]
    python bench.py --op prefill [--pconfig 1|2] [--kv e4m3|e5m2|int8]

A step is one pass of the whole hot path over one batch: slot mapping of the
new tokens, cache write of their K/V rows, and decode attention.  The default
mode ("fused") makes it one pa_decode_append call: the split-KV decode kernel
stores the new tokens itself, then the reduce kernel merges the partitions
(2 launches).  "split" / "single" run pa_slot_mapping + pa_cache_write and
then pa_decode_split_reduce / pa_decode (4 / 3 launches); "cascade" runs them
and then pa_decode_shared_prefix.  The default workload is the Qwen3-8B-shaped
decode step: 64 sequences, 32 query / 8 KV heads, head_dim 128, bf16, lengths
U[512, 4096], 16-token blocks in a shuffled pool.  Its K/V (~585 MB) is larger
than L2 (126 MB), so no L2 flush is needed between steps.

Output: one JSON line on rank 0.  ``value`` is KV GB/s of the whole job
(algorithmic step bytes of all ranks / max-over-ranks step time); ``e2e`` is
the same with the step's inputs copied from pinned host memory and its output
read back inside the timed region; ``roofline`` is for the attention launch
(decode kernel + reduce kernel, event-timed together) against the measured HBM
copy bandwidth, with ``traffic`` the DRAM bytes of those launches from the
committed ncu record (profiles/decode_traffic.json) while its kernel sources
are unchanged;
``cpu_baseline`` times the CPU oracle on a bounded sample.

``--impl reference`` times the CPU oracle itself as the reference arm (rank 0
only; other ranks exit without work).

Multi-GPU: independent replicas (the decode path needs no exchange), one
process per GPU under torchrun; weak scaling.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV GB/s & tokens/s per step; % of B200 HBM roofline"
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 7700.0  # B200 HBM3e, nominal (HGX)


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:  # noqa: BLE001
        return 1590.0, "fallback"


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_HBM_GBS, "fallback"


# the sources the decode and reduce kernels are compiled from: a recorded
# traffic figure is only reported while these are unchanged
DECODE_SOURCES = ("pa_decode.cu", "pa_decode_mma.cu", "pa_device.cuh", "pa_internal.h", "pa_tmap.h")


def kernel_source_hash(sources=DECODE_SOURCES) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_369_b200", "csrc")
    for name in sources:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def same_run_copy_gbs(device, stream, nbytes: int = 512 * 1024 * 1024, reps: int = 10) -> float:
    """A device-to-device copy of nbytes (larger than L2), timed with CUDA
    events on `stream` in this process: read + write bytes per second, the
    same-run ceiling next to the measured copy peak."""
    import torch

    src = torch.ones(nbytes, dtype=torch.uint8, device=device)
    dst = torch.empty_like(src)
    with torch.cuda.stream(stream):
        for _ in range(3):
            dst.copy_(src)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            dst.copy_(src)
        e1.record(stream)
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1) / reps
    del src, dst
    return 2.0 * nbytes / (ms * 1e-3) / 1e9


def recorded_traffic(cfg: int, mode: str, path=None, key=None):
    """DRAM bytes per attention launch from the committed ncu summary, if it
    was taken on the current kernel sources (else None).  `key` names an
    entry directly (e.g. a prefill workload)."""
    path = path or os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:  # noqa: BLE001
        return None
    key = key or f"config{cfg}_{mode}"
    ent = rec.get(key)
    if not ent or ent.get("kernel_hash") != kernel_source_hash(tuple(ent.get("sources", DECODE_SOURCES))):
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and throttle reasons from NVML, sampled in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.period = period_s
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001
            self.ok = False

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        try:
            mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        except Exception:  # noqa: BLE001
            mask = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
        for bit, name in self.REASONS.items():
            if mask & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank float over the process group (identity without one)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def workload_config(w, cfg: int, mode: str, P: int) -> dict:
    return {
        "workload": w.name, "config_id": cfg, "num_seqs": w.num_seqs,
        "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
        "block_size": w.block_size, "kv_dtype": w.kv_dtype, "act_dtype": w.act_dtype,
        "seq_len_mean": float(w.seq_lens.mean()), "seq_len_min": int(w.seq_lens.min()),
        "seq_len_max": int(w.seq_lens.max()), "num_blocks": w.num_blocks, "seed": w.seed,
        "mode": mode, "partition_size": P if mode in ("split", "fused", "cascade") else None,
        "l2": "inputs larger than L2: no flush" if w.kv_bytes_logical() > 256e6
        else "L2 flushed (256 MB write) between steps",
    }


# ---------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------

def oracle_units(w):
    """(sequence, KV head) units of the workload, each with its query heads."""
    return [(s, h) for s in range(w.num_seqs) for h in range(w.num_kv_heads)]


def time_oracle_units(w, kc, vc, units, budget_s=None):
    """Run the oracle's decode over the query heads of the given units; return
    (seconds, KV bytes those units read once, units done)."""
    import oracle

    g = w.group
    done = 0
    kv_bytes = 0
    t0 = time.perf_counter()
    for (s, kvh) in units:
        pairs = np.array([(s, kvh * g + i) for i in range(g)], dtype=np.int32)
        oracle.decode_for(w, kc, vc, pairs)
        kv_bytes += int(w.seq_lens[s]) * 2 * w.head_dim * w.kv_elem_bytes()
        done += 1
        if budget_s is not None and time.perf_counter() - t0 > budget_s:
            break
    return time.perf_counter() - t0, kv_bytes, done


def time_oracle_units_threads(w, kc, vc, units, threads: int, budget_s: float):
    """The same per-unit oracle calls spread over `threads` host threads (the
    C oracle keeps no shared state, and ctypes releases the GIL for the call);
    each thread takes units until the budget is spent.  Returns (seconds,
    KV bytes, units done)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor

    oracle.lib()  # loaded before the threads start
    g = w.group
    it = iter(units)
    lock = threading.Lock()
    t0 = time.perf_counter()

    def worker(_):
        b = n = 0
        while time.perf_counter() - t0 <= budget_s:
            with lock:
                u = next(it, None)
            if u is None:
                break
            s, kvh = u
            pairs = np.array([(s, kvh * g + i) for i in range(g)], dtype=np.int32)
            oracle.decode_for(w, kc, vc, pairs)
            b += int(w.seq_lens[s]) * 2 * w.head_dim * w.kv_elem_bytes()
            n += 1
        return b, n

    with ThreadPoolExecutor(max_workers=threads) as ex:
        res = list(ex.map(worker, range(threads)))
    return time.perf_counter() - t0, sum(r[0] for r in res), sum(r[1] for r in res)


def cpu_baseline(w, budget_s: float = 15.0):
    import oracle

    t0 = time.perf_counter()
    kc, vc = oracle.caches_for(w)
    build_s = time.perf_counter() - t0
    units = oracle_units(w)
    rng = np.random.default_rng(0)
    order = rng.permutation(len(units))
    sample = [units[i] for i in order]
    secs, kv_bytes, done = time_oracle_units(w, kc, vc, sample, budget_s)
    out = {
        "value": kv_bytes / secs / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
        "sample": f"{done} of {len(units)} (sequence, KV head) units of the same workload, "
                  f"fp64 C oracle, one thread ({secs:.1f} s; pools built in {build_s:.1f} s, untimed)",
    }
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    if cores > 1:
        secs_n, bytes_n, done_n = time_oracle_units_threads(w, kc, vc, sample, cores, budget_s / 2)
        out["all_cores"] = {
            "value": bytes_n / secs_n / 1e9, "unit": "GB/s", "cores": cores,
            "sample": f"{done_n} of {len(units)} units over {cores} threads ({secs_n:.1f} s)"}
    return out


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import workload

    w = workload.config(args.config, kv_dtype=args.kv, channel_scales=args.channel_scales)
    import oracle

    kc, vc = oracle.caches_for(w)
    units = oracle_units(w)
    for i in range(args.warmup):
        time_oracle_units(w, kc, vc, [units[i % len(units)]])
    tot_s, tot_b = 0.0, 0
    for i in range(args.steps):
        secs, b, _ = time_oracle_units(w, kc, vc, [units[(args.warmup + i) % len(units)]])
        tot_s += secs
        tot_b += b
    value = tot_b / tot_s / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_s / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.config, args.mode, args.partition),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": "each step: the query heads of one (sequence, KV head) unit "
                                   "of the workload, fp64 C oracle, one thread"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# copy-on-write block copy (pa_copy_blocks), one launch per step
# ---------------------------------------------------------------------------

def run_copy_blocks(args):
    """Time pa_copy_blocks on the pool shape of a named workload: ``--pairs``
    disjoint (src, dst) block pairs drawn from a seeded permutation, K and V
    pools alike.  Algorithmic bytes: every copied byte read once and written
    once."""
    import torch

    import workload
    import paged_kv_cache_369_b200 as pa

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    w = workload.config(args.config, draw_kv=False)
    from paged_kv_cache_369_b200 import pool_torch_dtype

    dt = pool_torch_dtype(w.kv_dtype)
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    kc = torch.empty(shape, dtype=dt, device=device)
    vc = torch.empty(shape, dtype=dt, device=device)
    kc.view(torch.uint8).fill_(0x3C)
    vc.view(torch.uint8).fill_(0x3C)
    n = min(args.pairs, w.num_blocks // 2)
    perm = np.random.default_rng(w.seed).permutation(w.num_blocks)
    pairs = torch.from_numpy(np.stack([perm[:n], perm[n:2 * n]], 1).astype(np.int32)).to(device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    block_bytes = w.num_kv_heads * w.block_size * w.head_dim * w.kv_elem_bytes()
    moved = 2 * 2 * n * block_bytes  # K and V, read + write
    stream = torch.cuda.Stream(device)
    flush = None if moved > 256e6 else torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            pa.pa_copy_blocks(kc, vc, pairs, err, stream)
    torch.cuda.synchronize(device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(device.index or 0)
    clocks.start()
    with torch.cuda.stream(stream):
        for a, b in ev:
            a.record(stream)
            pa.pa_copy_blocks(kc, vc, pairs, err, stream)
            b.record(stream)
            if flush is not None:
                flush.fill_(1)
    torch.cuda.synchronize(device)
    clocks.stop()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    value = moved / (ms * 1e-3) / 1e9
    peak, peak_kind = measured_hbm_peak()
    line = {
        "metric": "pa_copy_blocks GB/s (copy-on-write block copy, read + write)",
        "value": value, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.kv_dtype, "data": "synthetic pools, seeded block pairs",
        "config": {"workload": f"copy {n} blocks of {block_bytes} B per pool ({w.name} pool shape)",
                   "pairs": n, "block_bytes_per_pool": block_bytes, "num_blocks": w.num_blocks,
                   "l2": "copied bytes larger than L2: no flush" if flush is None
                   else "L2 flushed (256 MB write) between steps"},
        "roofline": {"bound": "hbm", "achieved": value, "peak": peak, "unit": "GB/s",
                     "frac": value / peak, "traffic": None,
                     "kernel": "copy_blocks_kernel", "algorithmic_bytes_per_launch": moved,
                     "peak_source": f"{peak_kind} HBM copy bandwidth"},
        "gpu_launches": args.steps, "clocks": clocks.summary(),
        "device_error": int(err.item()),
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# chunked prefill (pa_prefill), one attention launch per step
# ---------------------------------------------------------------------------

def run_prefill(args):
    """Time pa_prefill on a named 512-token-chunk workload.  A step is the
    chunk's cache append (slot mapping + cache write) and the attention
    launch; ``value`` counts the useful flops of q.K and P.V under the causal
    mask (4 * d * Hq per attended (query, key) pair)."""
    import torch

    import workload
    from paged_kv_cache_369_b200.runner import PagedPrefill

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    w = workload.prefill_config(args.pconfig, kv_dtype=args.kv)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        pre = PagedPrefill(w, device=str(device), stream=stream)
        for _ in range(args.warmup):
            pre.step()
    torch.cuda.synchronize(device)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(device.index or 0)
    clocks.start()
    with torch.cuda.stream(stream):
        for e0, e1, e2 in ev:
            e0.record(stream)
            pre.write_chunk()
            e1.record(stream)
            pre.attend()
            e2.record(stream)
    torch.cuda.synchronize(device)
    clocks.stop()
    step_ms = statistics.mean(a.elapsed_time(c) for a, _, c in ev)
    attn_ms = statistics.mean(b.elapsed_time(c) for _, b, c in ev)
    flops = w.flops()
    value = flops / (step_ms * 1e-3) / 1e12
    achieved = flops / (attn_ms * 1e-3) / 1e12
    peak, kind = measured_tensor_peak()
    line = {
        "metric": "chunked-prefill attention TFLOP/s (useful causal flops)",
        "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.act_dtype,
        "data": "synthetic: seeded N(0,1) q/K/V, shuffled block pool",
        "config": {"workload": w.name, "num_seqs": w.num_seqs, "chunk": int(w.max_query_len),
                   "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
                   "head_dim": w.head_dim, "kv_dtype": w.kv_dtype,
                   "context_mean": float((w.seq_lens - w.chunk_lens).mean()),
                   "seed": w.seed, "l2": "K/V re-read across query tiles is meant to hit L2; no flush"},
        "attention_us": attn_ms * 1e3, "cache_write_us": (step_ms - attn_ms) * 1e3,
        "tokens_per_s": w.num_tokens / (step_ms * 1e-3),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "traffic": recorded_traffic(0, "", key=f"prefill_pconfig{args.pconfig}_{w.kv_dtype}"),
                     "kernel": "prefill_kernel (tcgen05)",
                     "algorithmic_flops_per_launch": flops,
                     "peak_source": f"{kind} dense bf16 (cuBLAS burst, MEASURED_PEAKS.json bf16_tflops)"},
        "gpu_launches": 3 * args.steps, "clocks": clocks.summary(), "device_error": pre.error(),
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------

def time_device_steps(dec, stream, steps: int, fused: bool, flush=None):
    """Event-timed decode steps on `stream` with inputs resident in HBM.
    Returns (step ms without the L2 flushes, attention ms, cache-write ms)
    averaged over the steps.  The caller has warmed up and synchronised."""
    import torch

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    flush_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)] \
        if flush is not None else None
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for i in range(steps):
            e0, e1, e2 = ev[i]
            e0.record(stream)
            if fused:
                e1.record(stream)
                dec.step()  # one call: new tokens stored by the attention launch
            else:
                dec.write_new()
                e1.record(stream)
                dec.attend()
            e2.record(stream)
            if flush is not None:
                flush_ev[i][0].record(stream)
                flush.fill_(1)
                flush_ev[i][1].record(stream)
        t_end.record(stream)
    t_end.synchronize()
    total_ms = t_start.elapsed_time(t_end)
    flush_ms = sum(a.elapsed_time(b) for a, b in flush_ev) if flush_ev else 0.0
    step_ms = (total_ms - flush_ms) / steps
    attn_ms = statistics.mean(e1.elapsed_time(e2) for _, e1, e2 in ev)
    write_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1, _ in ev)
    return step_ms, attn_ms, write_ms


def time_graph_steps(dec, stream, steps: int, flush=None, barrier=None):
    """`steps` decode steps captured back to back in one CUDA graph (no
    events between them, so a step's first launch overlaps the previous
    step's last through programmatic dependent launch, and no host launch
    overhead), replayed once untimed and then once between two events on
    `stream`, with `barrier` (a rank barrier + device synchronise) on both
    sides of the timed replay.  With an L2 flush after every step, the
    flushes are timed in a graph of their own and subtracted.  Returns ms per
    step."""
    import torch

    def timed(body):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            body()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            g.replay()  # the first replay uploads the graph; not timed
        if barrier is not None:
            barrier()
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        if barrier is not None:
            barrier()
        e1.synchronize()
        ms = e0.elapsed_time(e1)
        del g
        return ms

    def steps_body():
        for _ in range(steps):
            dec.step()
            if flush is not None:
                flush.fill_(1)

    total = timed(steps_body)
    if flush is not None:
        def flush_body():
            for _ in range(steps):
                flush.fill_(1)
        total -= timed(flush_body)
    return total / steps


E2E_INPUTS = ("q", "k_new", "v_new", "block_tables", "seq_lens")


def time_end_to_end(dec, stream, device, steps: int, flush=None):
    """Decode steps end to end: every step copies its inputs (q, the new K/V
    rows, block tables, lengths) from pinned host memory and reads its output
    back into pinned host memory.  The copies of step i + 1's inputs and of
    step i - 1's output run on two copy streams while step i attends: inputs
    and outputs are double-buffered on the device, and events order each
    buffer's copy-in -> step -> copy-out -> reuse.  Returns (ms per step from
    the first input copy to the last output copy, H2D bytes per step, D2H
    bytes per step)."""
    import torch

    host = {n: getattr(dec, n).cpu().pin_memory() for n in E2E_INPUTS}
    keep = {n: getattr(dec, n) for n in E2E_INPUTS + ("out",)}
    bufs = [dict(keep), {n: torch.empty_like(t) for n, t in keep.items()}]
    host_out = [torch.empty_like(dec.out, device="cpu").pin_memory() for _ in range(2)]
    h2d_bytes = sum(t.numel() * t.element_size() for t in host.values())
    d2h_bytes = host_out[0].numel() * host_out[0].element_size()
    h2d_s, d2h_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer b landed
    ev_done = [torch.cuda.Event() for _ in range(2)]  # step on buffer b finished
    ev_out = [torch.cuda.Event() for _ in range(2)]   # output of buffer b read back
    e_s = torch.cuda.Event(enable_timing=True)
    e_e = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    e_s.record(h2d_s)
    for i in range(steps):
        b = i & 1
        buf = bufs[b]
        if i >= 2:
            h2d_s.wait_event(ev_done[b])  # step i - 2 no longer reads these inputs
        with torch.cuda.stream(h2d_s):
            for n in E2E_INPUTS:
                buf[n].copy_(host[n], non_blocking=True)
        ev_in[b].record(h2d_s)
        stream.wait_event(ev_in[b])
        if i >= 2:
            stream.wait_event(ev_out[b])  # step i - 2's output has been read back
        for n, t in buf.items():
            setattr(dec, n, t)
        with torch.cuda.stream(stream):
            dec.step()
            ev_done[b].record(stream)
            if flush is not None:
                flush.fill_(1)
        d2h_s.wait_event(ev_done[b])
        with torch.cuda.stream(d2h_s):
            host_out[b].copy_(buf["out"], non_blocking=True)
        ev_out[b].record(d2h_s)
    e_e.record(d2h_s)
    torch.cuda.synchronize(device)
    for n, t in keep.items():
        setattr(dec, n, t)
    return e_s.elapsed_time(e_e) / steps, h2d_bytes, d2h_bytes


def per_config_measurements(device, stream, steps: int, warmup: int):
    """Attention time, roofline fraction and clocks of the other named decode
    workloads, each in its default launch configuration: config 3 as a fused
    single-pass step, config 4 as a fused step with the 512-token partitions
    it prescribes, config 5 with its shared prefix attended once (cascade,
    768-token partitions).  Each is timed like the headline, on its own."""
    import torch

    import workload
    from paged_kv_cache_369_b200.runner import (PagedDecode, algorithmic_cascade_bytes,
                                                default_mode, default_partition_size)

    peak, _ = measured_hbm_peak()
    res = {}
    for cfg, mode in ((3, default_mode(3)), (4, default_mode(4)), (5, "cascade")):
        w = workload.config(cfg)
        P = default_partition_size(w, cfg)
        with torch.cuda.stream(stream):
            dec = PagedDecode(w, device=str(device), mode=mode, partition_size=P, stream=stream)
            for _ in range(warmup):
                dec.step()
        torch.cuda.synchronize(device)
        dec.dev_err.zero_()
        fused = mode.startswith("fused")
        attn_bytes = w.step_bytes() if fused else algorithmic_cascade_bytes(w)
        clocks = ClockSampler(device.index if device.index is not None else 0)
        clocks.start()
        step_ms = time_graph_steps(dec, stream, steps)
        clocks.stop()
        _, ev_attn_ms, write_ms = time_device_steps(dec, stream, steps, fused)
        attn_ms = step_ms if fused else ev_attn_ms
        achieved = attn_bytes / (attn_ms * 1e-3) / 1e9
        res[f"config{cfg}"] = {
            "workload": w.name, "mode": mode, "partition_size": P, "steps": steps,
            "us_per_step": step_ms * 1e3, "attention_us": attn_ms * 1e3,
            "cache_write_us": None if fused else write_ms * 1e3,
            "algorithmic_bytes_per_launch": attn_bytes, "achieved_gbs": achieved,
            "frac": achieved / peak, "tokens_per_s": w.num_seqs / (step_ms * 1e-3),
            "gpu_launches": steps * dec.launches_per_step(), "clocks": clocks.summary(),
            "traffic": recorded_traffic(cfg, mode), "device_error": dec.error(),
        }
        del dec
        torch.cuda.empty_cache()
    return res

def run_ours(args):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_env()
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=device)

    import workload
    from paged_kv_cache_369_b200.runner import (PagedDecode, algorithmic_cascade_bytes,
                                                algorithmic_decode_bytes)

    w = workload.config(args.config, kv_dtype=args.kv, channel_scales=args.channel_scales)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        dec = PagedDecode(w, device=str(device), mode=args.mode, partition_size=args.partition,
                          stream=stream)
    fused = args.mode.startswith("fused")
    step_bytes = w.step_bytes()
    # the fused attention launch also reads the new rows and stores them
    attn_bytes = step_bytes if fused else algorithmic_decode_bytes(w)
    if args.mode == "cascade":  # the shared prefix is read once, not once per sequence
        attn_bytes = algorithmic_cascade_bytes(w)
    flush = None
    if w.kv_bytes_logical() <= 256e6:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)

    # ---- device-resident timing ------------------------------------------
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            dec.step()
            if flush is not None:
                flush.fill_(1)
    barrier()
    dec.dev_err.zero_()
    clocks = ClockSampler(device.index if device.index is not None else 0)
    clocks.start()
    step_ms_local = time_graph_steps(dec, stream, args.steps, flush, barrier)
    clocks.stop()
    # the same steps issued one by one, each bracketed by events: the split of a
    # step into cache write and attention, and the cost of per-step launches
    barrier()
    ev_step_ms_local, ev_attn_ms, write_ms = time_device_steps(dec, stream, args.steps, fused, flush)
    barrier()
    err = dec.error()
    step_ms = max_over_ranks(step_ms_local, device)
    # attention time per step: the whole graph-timed step where the step is
    # the attention launches alone (a fused step stores the new tokens inside
    # them); else the event-timed attention launches
    attn_ms = step_ms_local if fused else ev_attn_ms
    total_bytes = sum_over_ranks(float(step_bytes), device)
    value = total_bytes / (step_ms * 1e-3) / 1e9

    # ---- end to end: pinned host inputs in, output out, every step --------
    e2e_steps = max(1, min(args.steps, 200))
    barrier()
    e2e_ms_local, h2d, d2h = time_end_to_end(dec, stream, device, e2e_steps, flush)
    barrier()
    e2e_ms = max_over_ranks(e2e_ms_local, device)
    e2e_value = total_bytes / (e2e_ms * 1e-3) / 1e9
    copy_gbs = same_run_copy_gbs(device, stream)

    result = None
    if rank == 0:
        peak, peak_kind = measured_hbm_peak()
        achieved = attn_bytes / (attn_ms * 1e-3) / 1e9
        traffic = recorded_traffic(args.config, args.mode)
        result = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.kv_dtype if w.kv_dtype not in ("e4m3", "e5m2", "int8")
            else f"{w.kv_dtype} KV / {w.act_dtype} q, f32 math",
            "data": "synthetic: seeded N(0,1) q/K/V, shuffled block pool, no dataset",
            "config": workload_config(w, args.config, args.mode, args.partition),
            "us_per_step": step_ms * 1e3,
            "tokens_per_s": world * w.num_seqs / (step_ms * 1e-3),
            "attention_us": attn_ms * 1e3,
            "cache_write_us": None if fused else write_ms * 1e3,
            "timing": "the K timed steps run as one CUDA graph (captured launches, programmatic "
                      "dependent launch between them) between two events on the launch stream",
            "event_timed": {"us_per_step": ev_step_ms_local * 1e3, "attention_us": ev_attn_ms * 1e3,
                            "note": "the same K steps launched one by one from Python with events "
                                    "around every step's launches"},
            "kv_bytes_per_step": w.kv_bytes_logical(),
            "step_bytes": step_bytes,
            "roofline": {
                "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic,
                "kernel": {
                    "fused": "pa_decode_append: decode kernel storing the new tokens + split reduce kernel",
                    "fused_single": "pa_decode_append: single-pass decode kernel storing the new tokens",
                    "split": "pa_decode_split_reduce: decode partition kernel + split reduce kernel",
                    "single": "pa_decode: single-pass decode kernel",
                    "cascade": "pa_decode_shared_prefix: prefix pass (tcgen05) + tail decode + merge"}[args.mode],
                "peak_source": f"{peak_kind} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6.65 TB/s",
                "algorithmic_bytes_per_launch": attn_bytes,
                "same_run_copy_gbs": copy_gbs,
                "frac_of_same_run_copy": achieved / copy_gbs,
                "frac_of_spec": achieved / SPEC_HBM_GBS,
            },
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps, "ms_per_step": e2e_ms,
                    "copies": "every step: its inputs H2D from pinned memory and its output "
                              "D2H, on two copy streams overlapping the neighbouring steps' "
                              "kernels (double-buffered)"},
            "gpu_launches": args.steps * dec.launches_per_step(),
            "clocks": clocks.summary(),
            "device_error": err,
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_per_config and args.config == 2 and args.mode == "fused" \
                and args.kv is None:
            del dec
            torch.cuda.empty_cache()
            result["per_config"] = per_config_measurements(device, stream, args.per_config_steps,
                                                           min(args.warmup, 10))
        if world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget)
        print(json.dumps(result), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", type=int, default=2, choices=(1, 2, 3, 4, 5))
    ap.add_argument("--mode", choices=("fused", "fused_single", "split", "single", "cascade"),
                    default=None,
                    help="default: fused_single for config 3, else fused; cascade: the "
                         "shared-prefix decode (config 5's common prefix attended once)")
    ap.add_argument("--partition", type=int, default=None,
                    help="split-KV partition in tokens (default: 512 for config 4, as it "
                         "prescribes, 768 for config 5, else 1024)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip timing the other named workloads (configs 3, 4, 5) after the "
                         "headline line's own measurement")
    ap.add_argument("--per-config-steps", type=int, default=300)
    ap.add_argument("--op", choices=("decode", "copy_blocks", "prefill"), default="decode",
                    help="decode: the decode step (default); copy_blocks: pa_copy_blocks alone; "
                         "prefill: a chunked-prefill step")
    ap.add_argument("--pconfig", type=int, default=1, choices=(1, 2),
                    help="named chunked-prefill workload for --op prefill")
    ap.add_argument("--pairs", type=int, default=4096, help="block pairs for --op copy_blocks")
    ap.add_argument("--kv", choices=("e4m3", "e5m2", "int8"), default=None,
                    help="replace the workload's cache format by this 8-bit one (per-tensor scale)")
    ap.add_argument("--channel-scales", action="store_true",
                    help="per-channel scales for the 8-bit cache (the cache write is then its own "
                         "call: --mode fused becomes split)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.mode is None or args.partition is None:
        from paged_kv_cache_369_b200.runner import default_mode, default_partition_size
        if args.mode is None:
            args.mode = default_mode(args.config)
        if args.partition is None:
            args.partition = default_partition_size(None, args.config)
    if args.channel_scales:
        if args.kv is None and args.config != 4:
            ap.error("--channel-scales needs an 8-bit cache (--kv or config 4)")
        if args.mode.startswith("fused"):
            args.mode = "split" if args.mode == "fused" else "single"
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "copy_blocks":
        return run_copy_blocks(args)
    if args.op == "prefill":
        return run_prefill(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
