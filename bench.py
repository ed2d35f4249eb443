"""Benchmark of one serving step of the paged KV cache hot path on B200.

A step is the whole hot path over one batch: slot mapping of the step's new tokens, the
cache write of their K/V, and paged attention of their queries over the cache (decode and
chunk kernels plus the split-KV reduce).  The request metadata, the step's Q/K/V and the
earlier tokens' K/V (already written into the pool) are resident in HBM before the timed
region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Prints one JSON line (rank 0).  `value` is KV-read GB/s of the whole step (algorithmic KV
bytes the step's attention reads / step time, summed over ranks); `tokens_per_s` is query
tokens per second.  Under torchrun every rank runs its own copy of the batch (weak scaling,
no collective on the data path); times are the max over ranks.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "long70b_decode"
# workloads measured alongside the main one in the same run (same metric, reported under
# "variants"): the long-context decode's FP8 E4M3 cache
VARIANTS = {"long70b_decode": {"fp8": "long70b_decode_fp8"}}
METRIC = "paged-attn KV-read GB/s (% of HBM peak) and query tokens/s per batch step"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20


# ---------------------------------------------------------------- helpers (no GPU needed)
def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    ap.add_argument("--sliding-window", type=int, default=0,
                    help="attend to the last W keys only (0 = full causal attention)")
    ap.add_argument("--local-chunk", type=int, default=0,
                    help="chunked local attention: a query at position p sees keys "
                         "floor(p / C) * C .. p (0 = off)")
    ap.add_argument("--no-alloc", action="store_true",
                    help="skip timing the device block allocation")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the workload's variants (e.g. the FP8 cache of long70b_decode)")
    ap.add_argument("--cpu-budget-s", type=float, default=10.0,
                    help="seconds of oracle time per CPU-baseline leg (single-threaded and "
                         "all host cores)")
    ap.add_argument("--flush", choices=["auto", "always", "never"], default="auto",
                    help="L2 flush between timed steps (auto: only when the step's KV bytes "
                         "are under 4x the 126 MB L2)")
    ap.add_argument("--kv-split-tokens", type=int, default=0,
                    help="force the KV partition (keys per split); 0 = planner's choice")
    ap.add_argument("--cascade", choices=["auto", "on", "off"], default="auto",
                    help="cascade attention over the block-table prefix every request shares "
                         "(auto: when it spans at least 256 tokens and 8 requests)")
    return ap.parse_args(argv)


def first_key(pos, window: int = 0, local_chunk: int = 0):
    """First key a query at position pos sees: 0 for full causal attention, pos - W + 1 with a
    sliding window W, floor(pos / C) * C with local chunks of C keys; the later of these."""
    pos = np.asarray(pos, dtype=np.int64)
    lo = np.zeros_like(pos)
    if window > 0:
        lo = np.maximum(lo, pos - window + 1)
    if local_chunk > 0:
        lo = np.maximum(lo, pos // local_chunk * local_chunk)
    return lo


def visible_keys(wl, window: int = 0, local_chunk: int = 0) -> np.ndarray:
    """Keys each request's rows read: from the first key its first new token sees (at
    position ctx - q_len) to the end of its context.  The first key never decreases with the
    position, so later rows read a subset."""
    ctx = wl.seq_lens.astype(np.int64)
    return ctx - first_key(ctx - wl.q_lens.astype(np.int64), window, local_chunk)


def kv_bytes(wl, window: int = 0, local_chunk: int = 0) -> int:
    """Algorithmic KV bytes the step's attention reads: every request's visible keys of K
    and V once per kv head (the GQA group shares one read)."""
    return int(np.sum(visible_keys(wl, window, local_chunk))) * 2 * wl.num_kv_heads * \
        wl.head_size * wl.dtype_bytes


def decode_kv_bytes(wl, window: int = 0, local_chunk: int = 0, prefix: int = 0) -> int:
    """KV bytes the decode kernel reads: the visible keys of every decode-kind request, less
    a shared prefix of `prefix` keys that cascade attention reads in its own pass."""
    G = wl.num_q_heads // wl.num_kv_heads
    ql = wl.q_lens
    dec = (ql > 0) & (ql * G <= 8)
    keys = visible_keys(wl, window, local_chunk)[dec] - prefix
    return int(np.sum(keys)) * 2 * wl.num_kv_heads * wl.head_size * wl.dtype_bytes


def prefix_pass_work(wl, prefix: int) -> tuple:
    """(KV bytes, FLOPs) of the cascade prefix pass: the prefix's keys read once per kv head,
    and every query row of the step against all of them (4 D FLOPs per (row, key))."""
    nbytes = prefix * 2 * wl.num_kv_heads * wl.head_size * wl.dtype_bytes
    flops = wl.num_tokens * wl.num_q_heads * prefix * 4 * wl.head_size
    return nbytes, flops


def chunk_flops(wl, window: int = 0, local_chunk: int = 0) -> int:
    """Algorithmic FLOPs of the chunk-kind requests: 4 D per unmasked (query, key) pair per q
    head (Q K^T and P V); query i of a request with q_len new tokens sits at position
    p = ctx - q_len + i and sees the keys first_key(p) .. p."""
    G = wl.num_q_heads // wl.num_kv_heads
    total = 0
    for ctx, ql in zip(wl.seq_lens.astype(np.int64), wl.q_lens.astype(np.int64)):
        if ql > 0 and ql * G > 8:
            pos = ctx - ql + np.arange(ql, dtype=np.int64)
            total += int(np.sum(pos + 1 - first_key(pos, window, local_chunk)))
    return total * wl.num_q_heads * 4 * wl.head_size


def launches_for_plan(plan: dict, head_size: int) -> int:
    """Kernels of ours per step, as pa_attention launches them: slot mapping and write, the
    split-counter clear (split decode requests, or chunk splits the tcgen05 kernel merges
    itself: head_size 128 and at most 4 splits), the cascade prefix pass, the decode and/or
    chunk kernel, and the split reduce (chunk splits not merged in the chunk kernel)."""
    fused = head_size == 128 and plan["chunk_max_splits"] <= 4
    clear = plan["decode_max_splits"] > 1 or (plan["chunk_max_splits"] > 1 and fused)
    reduce = plan["chunk_max_splits"] > 1 and not fused
    prefix = plan.get("prefix_splits", 0) > 0
    return 2 + int(clear) + int(prefix) + int(plan["num_decode_seqs"] > 0) + \
        int(plan["num_chunk_seqs"] > 0) + int(reduce)


def cascade_prefix_tokens(wl, mode: str = "auto") -> int:
    """Tokens of the block-table prefix every request of the step shares, to be read once by
    cascade attention; 0 when cascade is off (auto: a prefix of at least 256 tokens over at
    least 8 requests, every one of them a decode)."""
    if mode == "off":
        return 0
    from paged_kv_cache_421_b200 import _binding as B
    G = wl.num_q_heads // wl.num_kv_heads
    ql = wl.q_lens
    live = ql > 0
    if not np.all(ql[live] * G <= 8):
        return 0
    P = 16 * B.pa_common_prefix_blocks(wl.block_table, wl.seq_lens, wl.qsl)
    if mode == "auto" and (P < 256 or int(np.sum(live)) < 8):
        return 0
    return P


def unique_kv_bytes(wl) -> int:
    used = set()
    for r in range(wl.num_seqs):
        used.update(wl.block_table[r, :-(-int(wl.seq_lens[r]) // 16)].tolist())
    return len(used) * 2 * 16 * wl.num_kv_heads * wl.head_size * wl.dtype_bytes


def load_peaks() -> tuple:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def load_tensor_peak() -> tuple:
    """Dense bf16 tensor peak (TFLOP/s): the measured burst figure (the chunk kernel runs tens
    of microseconds, far from the power-capped sustained regime)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def _code_only(text: str) -> str:
    """Source text without comments and blank-line or indentation differences, so that a
    comment edit does not retire a recorded measurement of unchanged code."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.strip() for line in text.splitlines() if line.strip())


def source_digest(*names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "paged_kv_cache_421_b200", "csrc", n)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


# the sources each recorded kernel's code comes from (a change to any voids its record)
KERNEL_SOURCES = {
    "decode_kernel": ("pa_decode.cu", "pa_decode_epi.cuh", "pa_common.cuh"),
    "decode_tc8_kernel": ("pa_decode_tc.cu", "pa_decode_epi.cuh", "pa_tc.cuh", "pa_common.cuh"),
}


def decode_kernel_name(wl) -> str:
    """The decode kernel a workload runs on: tcgen05 for an FP8 cache at head_size 128."""
    return "decode_tc8_kernel" if (wl.kv_dtype != 0 and wl.head_size == 128) else "decode_kernel"


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu summary, if it
    was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path) or kernel not in KERNEL_SOURCES:
        return None
    digest = source_digest(*KERNEL_SOURCES[kernel])
    for line in open(path):
        parts = line.split()
        if len(parts) == 4 and parts[0] == kernel and parts[1] == workload and parts[2] == digest:
            return float(parts[3])
    return None


def median_clock(samples):
    loaded = [s for s in samples if s["util"] is None or s["util"] > 0] or samples
    mhz = [s["sm"] for s in loaded]
    return statistics.median(mhz) if mhz else None


class ClockSampler:
    """nvidia-smi clock/throttle sampling while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "utilization.gpu")

    def __init__(self, index: int, path: str):
        self.path, self.index, self.proc = path, index, None

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        samples, reasons = [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 10:
                continue
            try:
                sm, smax = float(p[1]), float(p[2])
            except ValueError:
                continue
            util = float(p[9]) if p[9].replace(".", "").isdigit() else None
            samples.append({"sm": sm, "max": smax, "util": util})
            for n, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": median_clock(samples), "sm_max_mhz": max(s["max"] for s in samples),
                "reasons": sorted(reasons), "samples": len(samples)}


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity on one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sub_workload_rows(wl, n_req: int):
    """Metadata of the first n_req requests of a step (for bounded CPU samples)."""
    qsl = wl.qsl[:n_req + 1].copy()
    return wl.block_table[:n_req], wl.seq_lens[:n_req], qsl


# ---------------------------------------------------------------- CPU oracle timing
def oracle_step_timer(wl, window: int = 0, local_chunk: int = 0):
    """Build the oracle's cache (untimed) and return a function that times the oracle over
    the first n requests of the step: slot mapping, cache write of their new tokens and
    attention of their queries, the attention single-threaded (threads None) or on the
    OpenMP build (threads n, 0 = every host core).  Returns (seconds, kv_bytes)."""
    import oracle
    from paged_kv_cache_421_b200 import workloads as W
    oracle.build()
    n_el = oracle.cache_elems(wl.num_blocks, 16, wl.num_kv_heads, wl.head_size)
    dt = np.uint16 if wl.kv_dtype == W.BF16 else np.uint8
    cache = np.full(n_el, W.CACHE_FILL_BF16 if dt == np.uint16 else W.CACHE_FILL_FP8, dt)
    ks = None if wl.k_scale is None else wl.k_scale.cpu().numpy()
    vs = None if wl.v_scale is None else wl.v_scale.cpu().numpy()
    hslots = oracle.slot_mapping(wl.hist_block_table, wl.hist_seq_lens, wl.hist_qsl, 16)
    oracle.write_kv(cache, wl.kv_dtype, wl.num_blocks, 16, wl.num_kv_heads, wl.head_size,
                    W.bits(wl.k_hist), W.bits(wl.v_hist), hslots, ks, vs)
    q_bits, k_bits, v_bits = W.bits(wl.q), W.bits(wl.k_new), W.bits(wl.v_new)
    per_tok = 2 * wl.num_kv_heads * wl.head_size * wl.dtype_bytes

    def run(n_req: int, threads=None):
        bt, sl, qsl = sub_workload_rows(wl, n_req)
        T = int(qsl[-1])
        t0 = time.perf_counter()
        slots = oracle.slot_mapping(bt, sl, qsl, 16)
        oracle.write_kv(cache, wl.kv_dtype, wl.num_blocks, 16, wl.num_kv_heads, wl.head_size,
                        k_bits[:T], v_bits[:T], slots, ks, vs)
        oracle.attention_paged(cache, wl.kv_dtype, wl.num_blocks, 16, wl.num_kv_heads,
                               wl.head_size, q_bits[:T], wl.num_q_heads, bt, sl, qsl, wl.scale,
                               ks, vs, window=window, local_chunk=local_chunk, threads=threads)
        ctx = sl.astype(np.int64)
        keys = ctx - first_key(ctx - np.diff(qsl), window, local_chunk)
        return time.perf_counter() - t0, int(np.sum(keys)) * per_tok
    return run


def _grow_sample(run, wl, budget_s: float, threads):
    """Time the oracle on the leading requests, growing the sample until one run takes about
    budget_s.  Returns (requests, seconds, kv bytes)."""
    n = 1
    sec, nbytes = run(n, threads)
    while sec < budget_s and n < wl.num_seqs:
        est = max(1, int(n * min(8.0, budget_s / max(sec, 1e-3))))
        n = min(wl.num_seqs, max(n + 1, est))
        sec, nbytes = run(n, threads)
    return n, sec, nbytes


def cpu_baseline(wl, budget_s: float, window: int = 0, local_chunk: int = 0) -> dict:
    """The oracle as it stands, timed on this host: single-threaded, and its OpenMP build over
    (request, kv head) units on every core this process may use.  The line's value is the
    all-core one; the single-threaded one is reported beside it."""
    import oracle
    run = oracle_step_timer(wl, window, local_chunk)
    n1, sec1, nb1 = _grow_sample(run, wl, budget_s, None)
    cores = oracle.threads_in_use(0)
    nn, secn, nbn = _grow_sample(run, wl, budget_s, 0)
    what = "slot mapping, cache write and fp64 attention"
    return {"value": round(nbn / secn / 1e9, 6), "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"first {nn} of {wl.num_seqs} requests of the step ({what}, {secn:.1f} s, "
                      f"C oracle built with OpenMP, {cores} threads over (request, kv head))",
            "single_thread": {
                "value": round(nb1 / sec1 / 1e9, 6), "unit": "GB/s", "cores": 1,
                "sample": f"first {n1} of {wl.num_seqs} requests of the step ({what}, "
                          f"{sec1:.1f} s, single-threaded C oracle)"}}


# ---------------------------------------------------------------- device step
class DeviceStep:
    def __init__(self, wl, device, kv_split_tokens: int = 0, sliding_window: int = 0,
                 local_chunk: int = 0, cascade: str = "auto"):
        import torch
        self.kv_split_tokens = kv_split_tokens
        self.window = sliding_window
        self.local_chunk = local_chunk
        self.prefix = (cascade_prefix_tokens(wl, cascade)
                       if not (sliding_window or local_chunk) else 0)
        from paged_kv_cache_421_b200 import ops
        from paged_kv_cache_421_b200 import workloads as W
        self.wl, self.dev, self.ops, self.torch = wl, device, ops, torch
        self.cache = ops.PagedKVCache(wl.num_blocks, wl.num_kv_heads, wl.head_size, wl.kv_dtype,
                                      k_scale=wl.k_scale, v_scale=wl.v_scale, device=device)
        if wl.kv_dtype == W.BF16:
            self.cache.buffer.view(torch.int16).fill_(W.CACHE_FILL_BF16)
        else:
            self.cache.buffer.fill_(W.CACHE_FILL_FP8)

        def i32(a):
            return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(device)
        hb, hs, hq = i32(wl.hist_block_table), i32(wl.hist_seq_lens), i32(wl.hist_qsl)
        Th = int(wl.hist_qsl[-1])
        if Th:
            hslots = ops.slot_mapping(hb, hs, hq, Th)
            ops.write_kv(self.cache, wl.k_hist.to(device).contiguous(),
                         wl.v_hist.to(device).contiguous(), hslots)
        self.bt, self.sl, self.qsl = i32(wl.block_table), i32(wl.seq_lens), i32(wl.qsl)
        self.q = wl.q.to(device).contiguous()
        self.k = wl.k_new.to(device).contiguous()
        self.v = wl.v_new.to(device).contiguous()
        T = wl.num_tokens
        self.slots = torch.empty(T, dtype=torch.int32, device=device)
        self.out = torch.empty(T, wl.num_q_heads, wl.head_size, dtype=torch.float32,
                               device=device)
        nb = ops.workspace_bytes_for(self.cache, wl.seq_lens, wl.qsl, wl.num_q_heads,
                                     wl.max_blocks_per_seq, kv_split_tokens,
                                     sliding_window=sliding_window, local_chunk=local_chunk,
                                     common_prefix_tokens=self.prefix)
        self.workspace = torch.empty(max(nb, 256), dtype=torch.uint8, device=device)
        self.plan = ops.B.pa_plan_attention(
            wl.seq_lens, wl.qsl, wl.num_q_heads, wl.num_kv_heads, wl.head_size,
            wl.max_blocks_per_seq,
            torch.cuda.get_device_properties(device).multi_processor_count,
            self.workspace.numel(), kv_split_tokens=kv_split_tokens,
            sliding_window=sliding_window, local_chunk=local_chunk,
            common_prefix_tokens=self.prefix, kv_dtype=self.cache.kv_dtype)
        torch.cuda.synchronize(device)

    def launches_per_step(self) -> int:
        return launches_for_plan(self.plan, self.wl.head_size)

    def run(self, events=None, q=None, k=None, v=None, bt=None, sl=None, qsl=None, out=None):
        B = self.ops.B
        wl = self.wl
        out = self.out if out is None else out
        bt = self.bt if bt is None else bt
        sl = self.sl if sl is None else sl
        qsl = self.qsl if qsl is None else qsl
        T = wl.num_tokens
        B.pa_slot_mapping(bt, bt.shape[1], sl, qsl, wl.num_seqs, T, 16, self.slots)
        B.pa_write_kv(self.cache.handle, self.k if k is None else k, self.v if v is None else v,
                      self.slots, T)
        B.pa_attention_ex(self.cache.handle, self.q if q is None else q, wl.num_q_heads, bt,
                          bt.shape[1], sl, qsl, wl.seq_lens, wl.qsl, wl.num_seqs, T, wl.scale,
                          out, self.workspace, self.workspace.numel(),
                          kv_split_tokens=self.kv_split_tokens, events=events,
                          sliding_window=self.window, local_chunk=self.local_chunk,
                          common_prefix_tokens=self.prefix)


def queue_ahead_ms(steps: int) -> float:
    """Length of the device-side wait in front of K timed steps: about 1 ms of host time per
    step to enqueue, at least 20 ms."""
    return min(200.0, max(20.0, 1.0 * steps))


def queue_ahead(stream, steps: int):
    """A device-side wait on `stream`, so that the host enqueues the timed steps while the
    device waits and the timed region holds device time only (a host slower than a step would
    otherwise leave the device idle between launches)."""
    import torch
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(queue_ahead_ms(steps) * 2.0e6))  # cycles at about 2 GHz


def time_step(step, args, flush_l2: bool, flush, stream, world: int, local: int, device,
              clock_path: str):
    """Warm up, then time K steps of `step`: once between one pair of CUDA events on the
    launching stream (the headline; consecutive kernels overlap their prologues through
    programmatic dependent launch, which events recorded between kernels would prevent; with
    an L2 flush each step gets its own event pair so the flush stays outside), then the same K
    steps again with events around every kernel for the per-kernel durations.  Clocks are
    sampled during the first pass.  Times are the max over ranks."""
    import torch
    import torch.distributed as dist

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for _ in range(max(args.warmup, 0)):
        step.run()
    torch.cuda.synchronize(device)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    st_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
    for e in ev:  # torch creates events lazily: record once so the library gets real handles
        for x in e:
            x.record()
    clocks = ClockSampler(local, clock_path)
    clocks.start()
    time.sleep(0.3)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fl_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(device)
    queue_ahead(stream, args.steps)
    t_start.record(stream)
    for i in range(args.steps):
        if flush_l2:
            flush.zero_()
            fl_ev[i][0].record(stream)
        step.run()
        if flush_l2:
            fl_ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    clk = clocks.stop()
    timed = (sum(a.elapsed_time(b) for a, b in fl_ev) if flush_l2
             else t_start.elapsed_time(t_end))
    ms_per_step = max_over_ranks(timed, world, device) / args.steps
    barrier()
    torch.cuda.synchronize(device)
    queue_ahead(stream, args.steps)
    for i in range(args.steps):
        if flush_l2:
            flush.zero_()
        st_ev[i][0].record(stream)
        step.run(events=ev[i])
        st_ev[i][1].record(stream)
    torch.cuda.synchronize(device)
    barrier()
    t = {"ms_per_step": ms_per_step,
         "ms_per_step_events": statistics.mean(a.elapsed_time(b) for a, b in st_ev),
         "decode": None, "chunk": None, "reduce": None, "clocks": clk}
    if step.plan["num_decode_seqs"]:
        t["decode"] = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in ev),
                                     world, device)
    # the chunk slot times the chunk kernel, or the prefix pass of a cascade step
    if step.plan["num_chunk_seqs"] or step.plan.get("prefix_splits", 0):
        t["chunk"] = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
    # the split reduce runs only for chunk splits the chunk kernel does not merge itself
    # (decode splits merge inside the decode kernel)
    if step.plan["chunk_max_splits"] > 1 and not (step.wl.head_size == 128 and
                                                  step.plan["chunk_max_splits"] <= 4):
        t["reduce"] = statistics.mean(e[4].elapsed_time(e[5]) for e in ev)
    return t


def decode_roofline(wl, workload: str, dec_ms: float, window: int, local_chunk: int,
                    prefix: int = 0) -> dict:
    """HBM roofline of the decode kernel: algorithmic KV bytes of one launch / its mean
    CUDA-event duration, against the measured copy peak."""
    peak, peak_kind = load_peaks()
    dec_bytes = decode_kv_bytes(wl, window, local_chunk, prefix)
    achieved = dec_bytes / (dec_ms * 1e-3) / 1e9
    kernel = decode_kernel_name(wl)
    return {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 1),
            "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
            # the record holds full-context launches: a window, local chunks or a cascade
            # prefix change what the kernel reads
            "traffic": (recorded_traffic(kernel, workload)
                        if not (window or local_chunk or prefix) else None),
            "peak_kind": peak_kind, "bytes_per_launch": dec_bytes,
            "ms_per_launch": round(dec_ms, 4)}


def dtype_name(wl) -> str:
    from paged_kv_cache_421_b200 import workloads as W
    return "bf16" if wl.kv_dtype == W.BF16 else "fp8_e4m3-kv/f16-mma"


def measure_variant(name: str, args, world: int, local: int, device, flush, stream) -> dict:
    """One variant workload (e.g. the FP8 cache of the main workload), timed like the main
    one: whole-step KV GB/s and the decode kernel's roofline."""
    import tempfile

    import torch
    from paged_kv_cache_421_b200 import workloads as W
    wl = W.CONFIGS[name](device=device)
    step = DeviceStep(wl, device, args.kv_split_tokens, args.sliding_window, args.local_chunk,
                      args.cascade)
    nbytes = kv_bytes(wl, args.sliding_window, args.local_chunk)
    flush_l2 = args.flush == "always" or (args.flush == "auto" and nbytes < 4 * L2_BYTES)
    t = time_step(step, args, flush_l2, flush, stream, world, local, device,
                  os.path.join(tempfile.gettempdir(), f"pa_clocks_{os.getpid()}_{name}.csv"))
    res = {"workload": name, "value": round(world * nbytes / (t["ms_per_step"] * 1e-3) / 1e9, 2),
           "unit": "GB/s", "ms_per_step": round(t["ms_per_step"], 4),
           "tokens_per_s": round(world * wl.num_tokens / (t["ms_per_step"] * 1e-3), 1),
           "dtype": dtype_name(wl), "kv_bytes_per_step": nbytes,
           "kernel_ms": {"decode": t["decode"], "chunk": t["chunk"], "reduce": t["reduce"]},
           "roofline": (decode_roofline(wl, name, t["decode"], args.sliding_window,
                                        args.local_chunk) if t["decode"] else None),
           "gpu_launches": step.launches_per_step() * args.steps, "clocks": t["clocks"]}
    del step
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()
    return res


def run_device_bench(args, rank, world, local):
    import tempfile

    import torch
    import torch.distributed as dist
    from paged_kv_cache_421_b200 import workloads as W

    device = torch.device(f"cuda:{local}")
    torch.cuda.set_device(device)
    wl = W.CONFIGS[args.workload](device=device)
    step = DeviceStep(wl, device, args.kv_split_tokens, args.sliding_window, args.local_chunk,
                      args.cascade)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    nbytes = kv_bytes(wl, args.sliding_window, args.local_chunk)
    flush_l2 = args.flush == "always" or (args.flush == "auto" and nbytes < 4 * L2_BYTES)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    stream = torch.cuda.current_stream(device)
    t = time_step(step, args, flush_l2, flush, stream, world, local, device,
                  os.path.join(tempfile.gettempdir(), f"pa_clocks_{os.getpid()}_{rank}.csv"))
    ms_per_step, ms_per_step_events = t["ms_per_step"], t["ms_per_step_events"]
    dec_ms, chunk_ms, reduce_ms, clk = t["decode"], t["chunk"], t["reduce"], t["clocks"]

    # ---- device block allocation for this step's requests (allocate_slots on a queue holding
    # the whole pool), timed apart from the step: the queue state is restored before each call
    alloc = None
    if not args.no_alloc:
        from paged_kv_cache_421_b200 import ops
        ql_d = torch.from_numpy(np.ascontiguousarray(wl.q_lens, np.int32)).to(device)
        comp_d = torch.from_numpy(np.ascontiguousarray(wl.seq_lens - wl.q_lens, np.int32)).to(device)
        queue = ops.BlockQueue(torch.arange(wl.num_blocks, dtype=torch.int32, device=device))
        saved = queue.state.clone()
        abt = torch.full((wl.num_seqs, wl.max_blocks_per_seq), -1, dtype=torch.int32, device=device)
        taken = ops.allocate_slots(abt, comp_d, ql_d, queue)
        # calls enqueued back to back, so the events see device time rather than host launch
        # gaps; the pool holds enough free blocks for all of them (else the state is restored
        # before each call with an 8-byte device copy, counted in the time)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_alloc = max(args.steps, 10)
        per_call = int(taken.clamp(min=0).sum().item())
        restore = per_call * (n_alloc + 1) > wl.num_blocks
        queue.state.copy_(saved)
        a0.record(stream)
        for i in range(n_alloc):
            if restore:
                queue.state.copy_(saved)
            ops.allocate_slots(abt, comp_d, ql_d, queue, out=taken)
        a1.record(stream)
        torch.cuda.synchronize(device)
        alloc = {"us_per_call": round(1e3 * a0.elapsed_time(a1) / n_alloc, 2),
                 "requests": wl.num_seqs, "blocks_taken": per_call,
                 "state_restored_each_call": restore}

    # ---- end-to-end: host inputs (pinned) -> device -> step -> output back to the host
    e2e = None
    if not args.no_e2e:
        # the step's host inputs packed back to back in one pinned buffer: one H2D copy per
        # step, then device views of it are handed to the C ABI
        parts = [wl.q.cpu().view(torch.uint8).reshape(-1),
                 wl.k_new.cpu().view(torch.uint8).reshape(-1),
                 wl.v_new.cpu().view(torch.uint8).reshape(-1),
                 torch.from_numpy(np.ascontiguousarray(wl.block_table, np.int32)).view(torch.uint8).reshape(-1),
                 torch.from_numpy(np.ascontiguousarray(wl.seq_lens, np.int32)).view(torch.uint8).reshape(-1),
                 torch.from_numpy(np.ascontiguousarray(wl.qsl, np.int32)).view(torch.uint8).reshape(-1)]
        offs, total = [], 0
        for t in parts:
            offs.append(total)
            total += (t.numel() + 255) // 256 * 256
        hbuf = torch.zeros(total, dtype=torch.uint8).pin_memory()
        for o, t in zip(offs, parts):
            hbuf[o:o + t.numel()] = t
        # two device input buffers and two output buffers: step i+1's inputs go up and step
        # i's output comes back on copy streams while step i computes (every step still copies
        # its inputs from pinned host memory and reads its output back to the host)
        dbufs = [torch.empty(total, dtype=torch.uint8, device=device) for _ in range(2)]
        douts = [torch.empty_like(step.out) for _ in range(2)]
        houts = [torch.empty(step.out.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
        up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)

        def dview(buf, i, dtype, shape):
            n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
            return buf[offs[i]:offs[i] + n].view(dtype).view(*shape)
        views = [dict(q=dview(bf, 0, torch.bfloat16, step.q.shape),
                      k=dview(bf, 1, torch.bfloat16, step.k.shape),
                      v=dview(bf, 2, torch.bfloat16, step.v.shape),
                      bt=dview(bf, 3, torch.int32, step.bt.shape),
                      sl=dview(bf, 4, torch.int32, step.sl.shape),
                      qsl=dview(bf, 5, torch.int32, step.qsl.shape)) for bf in dbufs]
        h2d = total  # bytes each step's H2D copy moves (inputs plus 256-byte alignment padding)
        d2h = houts[0].numel() * houts[0].element_size()

        def e2e_steps(n, t0=None, t1=None):
            ev = lambda: torch.cuda.Event()  # noqa: E731
            up_done = [ev(), ev()]
            comp_done = [ev(), ev()]
            down_done = [ev(), ev()]
            if t0 is not None:
                t0.record(up)
            with torch.cuda.stream(up):
                dbufs[0].copy_(hbuf, non_blocking=True)
                up_done[0].record(up)
            for i in range(n):
                b = i & 1
                if i + 1 < n:  # next step's inputs, once step i-1 has finished with that buffer
                    with torch.cuda.stream(up):
                        if i >= 1:
                            up.wait_event(comp_done[1 - b])
                        dbufs[1 - b].copy_(hbuf, non_blocking=True)
                        up_done[1 - b].record(up)
                stream.wait_event(up_done[b])
                if i >= 2:  # step i-2's output has been read back from this buffer
                    stream.wait_event(down_done[b])
                if flush_l2:
                    flush.zero_()
                step.run(out=douts[b], **views[b])
                comp_done[b].record(stream)
                with torch.cuda.stream(down):
                    down.wait_event(comp_done[b])
                    houts[b].copy_(douts[b], non_blocking=True)
                    down_done[b].record(down)
            stream.wait_event(down_done[(n - 1) & 1])
            if n >= 2:
                stream.wait_event(down_done[n & 1])
            if t1 is not None:
                t1.record(stream)

        e2e_steps(max(args.warmup, 1))
        torch.cuda.synchronize(device)
        barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_steps(args.steps, t0, t1)
        torch.cuda.synchronize(device)
        barrier()
        e2e_ms = max_over_ranks(t0.elapsed_time(t1), world, device) / args.steps
        # the pipelined path returns what the device-resident step computes, bit for bit
        step.run()
        torch.cuda.synchronize(device)
        if not torch.equal(houts[(args.steps - 1) & 1], step.out.cpu()):
            raise RuntimeError("end-to-end output differs from the device-resident step")
        e2e = {"value": round(world * nbytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e2e_ms, 4),
               "pipelining": "step i+1's H2D and step i's D2H overlap step i's compute"}

    # ---- variants of the workload (same metric, same timing), e.g. its FP8 E4M3 cache
    variants = None
    if not args.no_variants and args.workload in VARIANTS:
        variants = {key: measure_variant(name, args, world, local, device, flush, stream)
                    for key, name in VARIANTS[args.workload].items()}

    result = None
    if rank == 0:
        peak, peak_kind = load_peaks()
        value = world * nbytes / (ms_per_step * 1e-3) / 1e9
        roof = None
        if dec_ms:
            roof = decode_roofline(wl, args.workload, dec_ms, args.sliding_window,
                                   args.local_chunk, step.prefix)
            if step.prefix:  # the recorded traffic is of the non-cascade decode kernel
                roof["traffic"] = None
        cascade = None
        if step.prefix:
            pb, pf = prefix_pass_work(wl, step.prefix)
            cascade = {"prefix_tokens": step.prefix, "prefix_splits": step.plan["prefix_splits"],
                       "prefix_pass_ms": round(chunk_ms, 4) if chunk_ms else None,
                       "prefix_pass_flops": pf, "prefix_pass_kv_bytes": pb,
                       "prefix_pass_tflops": round(pf / (chunk_ms * 1e-3) / 1e12, 1)
                       if chunk_ms else None}
        chunk_roof = None
        if chunk_ms and not step.prefix:
            flops = chunk_flops(wl, args.sliding_window, args.local_chunk)
            tflops = flops / (chunk_ms * 1e-3) / 1e12
            tpeak, tkind = load_tensor_peak()
            chunk_roof = {"bound": "tensor", "kernel": "chunk_tc_kernel", "achieved": round(tflops, 1),
                          "peak": tpeak, "unit": "TFLOP/s", "frac": round(tflops / tpeak, 4),
                          "traffic": None, "peak_kind": tkind,
                          "flops_per_launch": flops,
                          "ms_per_launch": round(chunk_ms, 4)}
            y = step.plan.get("chunk_ctas_per_kv_head", 0)
            if y and not step.prefix and step.plan["num_decode_seqs"]:
                # beside the decode kernel the chunk kernel holds y CTAs (SMs) per kv head only
                sms = torch.cuda.get_device_properties(device).multi_processor_count
                held = min(sms, y * wl.num_kv_heads)
                chunk_roof["sms_held"] = held
                chunk_roof["frac_of_held_sms"] = round(tflops / (tpeak * held / sms), 4)
            if roof is None:
                roof = chunk_roof
        result = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": dtype_name(wl),
            "data": "synthetic (seeded; random-init Q/K/V ~ N(0,1) in bf16)",
            "config": {"workload": args.workload, "num_seqs": wl.num_seqs,
                       "tokens_per_step": wl.num_tokens, "num_q_heads": wl.num_q_heads,
                       "num_kv_heads": wl.num_kv_heads, "head_size": wl.head_size,
                       "block_size": 16, "num_blocks": wl.num_blocks,
                       "kv_bytes_per_step": nbytes, "unique_kv_bytes_per_step": unique_kv_bytes(wl),
                       "l2": ("flushed between steps (256 MiB write outside the step events)"
                              if flush_l2 else
                              f"inputs larger than L2: {nbytes / 1e6:.0f} MB of KV per step vs "
                              f"126 MB L2, no flush"),
                       "launch": (f"the timed steps are enqueued behind a ~{queue_ahead_ms(args.steps):.0f} ms "
                                  "device-side wait (device time only, no host gaps)"),
                       "kv_split_tokens": args.kv_split_tokens or "planner",
                       "cascade_prefix_tokens": step.prefix or None,
                       "sliding_window": args.sliding_window or None,
                       "local_chunk": args.local_chunk or None,
                       "parallelism": f"replicas x{world} (one batch per GPU)"},
            "tokens_per_s": round(world * wl.num_tokens / (ms_per_step * 1e-3), 1),
            "pct_hbm_peak": round(100 * value / world / peak, 2),
            "unique": ({"kv_bytes_per_step": ub,
                        "value": round(world * ub / (ms_per_step * 1e-3) / 1e9, 2),
                        "unit": "GB/s",
                        "pct_hbm_peak": round(100 * ub / (ms_per_step * 1e-3) / 1e9 / peak, 2)}
                       if (ub := unique_kv_bytes(wl)) < nbytes else None),
            "cascade": cascade,
            "roofline": roof,
            "kernel_ms": {"decode": dec_ms, "chunk": chunk_ms, "reduce": reduce_ms},
            "ms_per_step_with_kernel_events": round(ms_per_step_events, 4),
            "chunk_roofline": chunk_roof,
            "alloc": alloc,
            "e2e": e2e,
            "gpu_launches": step.launches_per_step() * args.steps,
            "clocks": clk,
            "variants": variants,
        }
    return result, wl


def reference_arm(args, rank, world):
    """The oracle, as it stands, on the host cores (its OpenMP build over (request, kv head)
    units, every core this process may use): each step a bounded sample (the leading requests
    of the same workload), slot mapping + cache write + fp64 attention, sized so that the
    warm-up and timed steps together take about a minute and a half."""
    if rank != 0:
        return None
    import oracle
    from paged_kv_cache_421_b200 import workloads as W
    wl = W.CONFIGS[args.workload]()
    run = oracle_step_timer(wl, args.sliding_window, args.local_chunk)
    per_step_s = max(0.25, 90.0 / max(1, args.steps + max(args.warmup, 0)))
    n, _, _ = _grow_sample(run, wl, per_step_s, 0)
    cores = oracle.threads_in_use(0)
    for _ in range(max(args.warmup, 0)):
        run(n, 0)
    secs, nb = [], 0
    for _ in range(args.steps):
        s, nb = run(n, 0)
        secs.append(s)
    sec = sum(secs) / len(secs)
    value = nb / sec / 1e9
    sample = (f"first {n} of {wl.num_seqs} requests per step (slot mapping, cache write, fp64 "
              f"attention; C oracle built with OpenMP, {cores} threads)")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": args.workload, "num_seqs": wl.num_seqs,
                   "tokens_per_step": wl.num_tokens, "num_q_heads": wl.num_q_heads,
                   "num_kv_heads": wl.num_kv_heads, "head_size": wl.head_size, "block_size": 16},
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.impl == "reference":
        res = reference_arm(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(f"cuda:{local}"))
    result, wl = run_device_bench(args, rank, world, local)
    if rank == 0:
        if not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(wl, args.cpu_budget_s, args.sliding_window,
                                                  args.local_chunk)
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
