#!/usr/bin/env python3
"""Benchmark of the paged decode-attention hot path on B200.

One step = one decode step of the whole model's attention cache traffic:
for each of the 16 layers, append the new token's K/V of every sequence and
run decode attention over the paged cache, through the C ABI -- by default
as one fused call per layer (paged_attention_decode_append), with --unfused
as pkv_append then paged_attention_decode.  Default workload: the
continuous-batching mix (batch 64, lengths log-uniform in [1, 8192],
fragmented block tables, 16 layers).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--kernel auto|simt|mma] [--unfused]
                    [--queries 1..8] [--out-dtype f32|bf16] [--no-early-pages]
                    [--grid CTAS] [--no-pdl] [--no-fill] [--no-cpu-baseline]
                    [--also W1,W2 | --also none] [--cold-l2] [--clock-seconds S]
                    [--e2e-steps N] [--cpu-seconds S] [--reference-seconds S]
    python bench.py --table      # every workload and option row, one run

Prints one JSON line (rank 0).  ``value`` is decode-queries/s over all
ranks, one query being one sequence's 32 query heads at one layer
(``head_queries_per_s`` counts heads, ``tokens_per_s`` sequences' tokens
per whole-model step; ``append``, in --unfused runs, the separate append's
share of a layer).  The ``roofline`` object reports the decode call's
algorithmic HBM bytes per launch divided by its measured average launch
time, against the measured HBM copy bandwidth, with the DRAM traffic of the
committed ncu capture.  ``clocks`` are sampled over the timed steps and a
following window of at least --clock-seconds of the same graph replays
(``clocks.window``: that window's own per-launch time).  ``per_workload``
holds the same measurement for the other workloads (long context, the second
speed target; the Llama-1B batch with a cold-L2 figure; the 35 GB stress
batch).  ``e2e`` is
the same step with its inputs and outputs crossing from and to pinned host
memory every step; ``prefill_fill`` the page-fill bandwidth;
``cpu_baseline`` the FP64 oracle on the host cores.  ``--impl reference``
times the FP64 CPU oracle on the same workload instead (bounded sample per
step, host cores).  ``--table`` measures every workload (hot and cold L2
for the two whose layer fits in L2) and the multi-query, BF16-output and
fill rows, and prints them as JSON lines and a markdown table.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_attention_decode_pkv_b200 import workloads as W  # noqa: E402

METRIC = "paged decode attention: achieved HBM GB/s (% of peak) and decode-queries/sec"
UNIT = "decode-queries/s"
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------ helpers --

def alg_bytes_decode(seq_lens: np.ndarray, queries: int = 1, out_bytes: int = 4) -> int:
    """Algorithmic bytes of one decode launch: per sequence K+V of every
    token (2048 B/token), q (4096 B per query), out (32 x 64 elements of
    out_bytes per query: 8192 B in FP32), block-table entries (4 B per page)
    and the length (4 B)."""
    L = seq_lens.astype(np.int64)
    per_seq = 2048 * L + queries * (4096 + 2048 * out_bytes) + 4 * ((L + 15) // 16) + 4
    return int(per_seq.sum())


def _strip_comments(src: str) -> str:
    """C/C++ source without comments and with whitespace runs collapsed
    (string and character literals kept as they are)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            while i < n and src[i] != "\n":
                i += 1
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_digest() -> str:
    """sha256 of the decode kernel's sources without comments (the ncu
    traffic figure is only valid for the code it was captured on)."""
    import hashlib
    h = hashlib.sha256()
    for fn in ("decode.cu", "pkv_internal.cuh"):
        with open(os.path.join(ROOT, "paged_attention_decode_pkv_b200", "csrc", fn)) as f:
            h.update(_strip_comments(f.read()).encode())
    return h.hexdigest()


def recorded_traffic(workload: str, alg_bytes: float):
    """DRAM bytes per decode launch from the committed ncu summary of this
    workload, scaled to `alg_bytes`; None if there is none or the kernel
    sources changed since it was captured."""
    p = os.path.join(ROOT, "profiles", "decode_traffic_%s.txt" % workload)
    try:
        kv = {}
        with open(p) as f:
            for line in f:
                if ":" in line:
                    k, v = line.split(":", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("kernel_source_sha256") != kernel_source_digest():
            return None
        return float(kv["dram_bytes_per_launch"]) * alg_bytes / float(kv["alg_bytes_of_launch"])
    except (OSError, KeyError, ValueError):
        return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons, taken while the
    timed region runs: sampling starts (and its first line is awaited)
    before the region, every line is stamped with the host clock as it
    arrives, and only lines stamped inside the region are kept."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.stamped = []
        self.lines = []

    def _read(self):
        for line in self.proc.stdout:
            if line.strip():
                self.stamped.append((time.monotonic(), line))

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
            deadline = time.monotonic() + 5.0
            while not self.stamped and time.monotonic() < deadline:
                time.sleep(0.01)
        except Exception:
            self.proc = None
        self.t0 = time.monotonic()
        return self

    def __exit__(self, *exc):
        self.t1 = time.monotonic()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.reader.join(timeout=5)
        self.lines = [l for t, l in self.stamped if self.t0 <= t <= self.t1]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------- multi-rank --
# The path shards by sequence with no exchange: each rank runs its own
# replica of the workload (its own pool, block tables and sequences, seeded
# per rank), so per-GPU work is fixed as ranks are added (weak scaling) and
# the only collectives are the barrier around the timed region and the max
# of the elapsed times.

def workload_for_rank(name: str, rank: int) -> W.Workload:
    """Rank r gets the same workload shape drawn with seed + 1000 r."""
    base = W.make(name)
    return base if rank == 0 else W.make(name, seed=base.seed + 1000 * rank)


def max_over_ranks(value: float, device) -> float:
    """Largest `value` over all ranks (identity without a process group)."""
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as tdist
    if tdist.is_available() and tdist.is_initialized():
        tdist.barrier()


def whole_job_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Units processed by all ranks per second of the slowest rank."""
    return units_per_rank * world / (max_ms / 1e3)


# ---------------------------------------------------------------- our arm --

def launch_flags(pkv, pdl: bool = True, early_pages: bool = True) -> int:
    """Pool launch flags of the benchmarked step.  No kernel of the step
    writes the lengths or the block tables, and the only pages a step writes
    are the sequences' last pages (the appended token), which decode never
    loads early, so with PDL both early flags hold for the fused and the
    separate-append step alike."""
    if not pdl:
        return 0
    flags = pkv.LAUNCH_PDL | pkv.LAUNCH_EARLY_TABLES
    if early_pages:
        flags |= pkv.LAUNCH_EARLY_PAGES
    return flags


class Runner:
    """Device-resident state of one workload on one GPU."""

    def __init__(self, w: W.Workload, device, kernel: int, fused: bool, queries: int = 1,
                 out_dtype=torch.float32, grid: int = 0, min_chunk: int = 0):
        from paged_attention_decode_pkv_b200 import pkv
        self.pkv = pkv
        self.w = w
        self.device = device
        self.kernel = kernel
        self.grid = grid
        self.min_chunk = min_chunk
        self.queries = queries
        self.out_dtype = out_dtype
        # two queries per sequence: decode only (their tokens would be
        # written with pkv_fill, not the one-token fused append)
        self.fused = fused and queries == 1
        # Two queries need a context of at least two tokens: such sequences get
        # length max(L, 2), and the pool holds values (not NaN) in every slot,
        # the second token of a one-token sequence included.
        self.pool_t = W.make_pool(w, device, poison=queries == 1)
        self.pool = pkv.Pool(w.num_pages, storage=self.pool_t)
        self.bt = torch.from_numpy(w.block_tables).to(device)
        nl, B = w.num_layers, w.batch
        self.lens_np = [np.maximum(w.seq_lens(s), queries).astype(np.int32)
                        for s in range(1, w.num_steps + 1)]
        self.seq_lens = [torch.from_numpy(x).to(device) for x in self.lens_np]
        # one set of per-layer inputs, reused every step (values do not change timing)
        ins = [W.step_inputs(w, 1, l, device) for l in range(nl)]
        self.q = torch.stack([x[0] for x in ins])
        if queries > 1:   # more queries per sequence: the first one again, scaled
            self.q = torch.stack([(self.q.float() * (1.0 - 0.1 * i)).to(torch.bfloat16)
                                  for i in range(queries)], dim=2)
        self.k = torch.stack([x[1] for x in ins])
        self.v = torch.stack([x[2] for x in ins])
        oshape = (nl, B, 32, 64) if queries == 1 else (nl, B, queries, 32, 64)
        self.out = torch.empty(oshape, dtype=out_dtype, device=device)
        self.ws = self.pool.workspace(B, kernel, grid, queries)
        self.graphs, self.decode_graphs = [], []
        self.twins = []

    def twin(self, stream):
        """A second set of step inputs and outputs (same pool, tables and
        workspace) with its own step graphs, for double-buffered end-to-end
        runs.  Steps of the two sets run one after another on one stream, so
        sharing the workspace is safe."""
        import copy
        t = copy.copy(self)
        t.seq_lens = [x.clone() for x in self.seq_lens]
        t.q, t.k, t.v = self.q.clone(), self.k.clone(), self.v.clone()
        t.out = torch.empty_like(self.out)
        t.twins = []
        t.capture(stream)
        self.twins.append(t)
        return t

    def launch_step(self, stream, variant, decode_only=False):
        """Launch one decode step (all layers) for lengths variant `variant`:
        per layer the fused append + decode, or append then decode, or (for
        the unfused decode roofline) only the decodes."""
        pkv = self.pkv
        sl = self.seq_lens[variant]
        for l in range(self.w.num_layers):
            if self.queries > 1 or self.out_dtype != torch.float32:
                kv = dict(k_new=self.k[l], v_new=self.v[l]) if self.fused else {}
                if not self.fused and not decode_only and self.queries == 1:
                    pkv.append(self.pool, self.bt, sl, self.k[l], self.v[l], l, stream=stream)
                pkv.decode_general(self.q[l], self.pool, self.bt, sl, l, self.w.scale,
                                   num_queries=self.queries, out_dtype=self.out_dtype,
                                   out=self.out[l], workspace=self.ws, kernel=self.kernel,
                                   grid_ctas=self.grid, min_chunk=self.min_chunk,
                                   stream=stream, **kv)
                continue
            if self.fused:
                pkv.decode_append(self.q[l], self.k[l], self.v[l], self.pool, self.bt, sl, l,
                                  self.w.scale, out=self.out[l], workspace=self.ws,
                                  kernel=self.kernel, grid_ctas=self.grid,
                                  min_chunk=self.min_chunk, stream=stream)
                continue
            if not decode_only:
                pkv.append(self.pool, self.bt, sl, self.k[l], self.v[l], l, stream=stream)
            pkv.decode(self.q[l], self.pool, self.bt, sl, l, self.w.scale, out=self.out[l],
                       workspace=self.ws, kernel=self.kernel, grid_ctas=self.grid,
                       min_chunk=self.min_chunk, stream=stream)

    def capture(self, stream):
        """CUDA graphs, one per lengths variant (the workload's step cycle):
        the full step, and the step's decodes alone (for the decode roofline).
        No timing events inside the graphs: an event node costs a few
        microseconds and would break the launch chaining."""
        self.graphs, self.decode_graphs = [], []
        kinds = ((False, self.graphs),) if self.fused else \
            ((False, self.graphs), (True, self.decode_graphs))
        for v in range(self.w.num_steps):
            for only, dst in kinds:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    self.launch_step(stream, v, decode_only=only)
                dst.append(g)

    def replay(self, i):
        self.graphs[i % len(self.graphs)].replay()

    def replay_decodes(self, i):
        self.decode_graphs[i % len(self.decode_graphs)].replay()

    def decode_bytes(self, i):
        """Algorithmic bytes of one decode launch of lengths variant i (with
        the fused append: plus each sequence's new K/V rows read from the
        inputs and written into the pool)."""
        b = alg_bytes_decode(self.lens_np[i % self.w.num_steps], self.queries,
                             self.out.element_size())
        return b + (4096 * self.w.batch if self.fused else 0)

    def mean_decode_bytes(self, start, n):
        """Mean of decode_bytes(i) over steps start .. start + n - 1."""
        per = [self.decode_bytes(v) for v in range(self.w.num_steps)]
        full, rem = divmod(n, len(per))
        tot = full * sum(per) + sum(per[(start + j) % len(per)] for j in range(rem))
        return tot / n

    def kernels_per_layer(self, decode_only=False):
        """Kernels one layer of a step launches: the decode kernel and the
        split-KV merge, plus the separate append unless fused."""
        return 2 + (0 if self.fused or decode_only or self.queries > 1 else 1)

    def close(self):
        """Release the graphs (they hold this library's kernel nodes), the
        twins' graphs and the pool, device synchronised, before anything
        they reference goes away."""
        torch.cuda.synchronize(self.device)
        for t in self.twins:
            t.graphs, t.decode_graphs = [], []
        self.twins = []
        self.graphs, self.decode_graphs = [], []
        self.pool.close()


def _events():
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def _replays(r: Runner, stream, steps, decode_only=False, start=0):
    """CUDA-event time (ms) of `steps` back-to-back step replays on `stream`."""
    e0, e1 = _events()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(start, start + steps):
            (r.replay_decodes if decode_only else r.replay)(i)
        e1.record(stream)
    return e0, e1


def _replays_each(r: Runner, stream, steps, start=0):
    """`steps` back-to-back step replays with an event after each one (the
    events sit between graph launches, never inside a graph).  Returns the
    first and last events and the per-step durations (ms) after a sync."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    with torch.cuda.stream(stream):
        evs[0].record(stream)
        for i in range(steps):
            r.replay(start + i)
            evs[i + 1].record(stream)
    stream.synchronize()
    return evs[0], evs[-1], [evs[i].elapsed_time(evs[i + 1]) for i in range(steps)]


def _cold_replays(r: Runner, stream, steps, decode_only=False):
    """Per-step CUDA-event times (ms) with L2 flushed before every step: a
    buffer twice the L2 size is written between replays, outside the
    timed events."""
    l2 = torch.cuda.get_device_properties(r.device).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=r.device)
    pairs = []
    with torch.cuda.stream(stream):
        for i in range(steps):
            flush.fill_(i & 0xFF)
            e0, e1 = _events()
            e0.record(stream)
            (r.replay_decodes if decode_only else r.replay)(i)
            e1.record(stream)
            pairs.append((e0, e1))
    stream.synchronize()
    del flush
    return [a.elapsed_time(b) for a, b in pairs]


def measure(args, name, device, rank, world, local_rank, *, full=False, cold=False,
            cpu_seconds=0.0, cpu_rows=None, queries=None, out_dtype=None, kernel=None):
    """Set up one workload and time its step the way the benchmark line
    reports it.  Every rank runs the same collectives in the same order.
    Returns the workload's record (rank 0) or None."""
    from paged_attention_decode_pkv_b200 import pkv
    queries = args.queries if queries is None else queries
    out_dtype = args.out_dtype if out_dtype is None else out_dtype
    kname = args.kernel if kernel is None else kernel
    kern = {"auto": pkv.KERNEL_AUTO, "simt": pkv.KERNEL_SIMT, "mma": pkv.KERNEL_MMA}[kname]
    w = workload_for_rank(name, rank)
    fused = not args.unfused and queries == 1
    tdtype = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    r = Runner(w, device, kern, fused, queries, tdtype, args.grid, args.min_chunk)
    flags = launch_flags(pkv, pdl=not args.no_pdl, early_pages=not args.no_early_pages)
    r.pool.set_launch_flags(flags)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            r.launch_step(stream, i % w.num_steps)
    stream.synchronize()
    if pkv.get_device_error(r.pool, stream) != 0:
        raise RuntimeError("device error in the warm-up steps of %s" % name)
    r.capture(stream)
    for i in range(max(args.warmup, w.num_steps)):
        r.replay(i)
        if not fused:
            r.replay_decodes(i)
    torch.cuda.synchronize()

    # ---- timed region: (A) K full steps; unfused only, then (B) the decodes
    # of K steps alone, back to back, for the decode call's launch duration
    # (fused, a step is nothing but the decode calls, so (A) gives it).  The
    # clock sampler keeps running over a window of at least clock_seconds of
    # the same full-step replays right after, so that its record has samples
    # however short the timed region is.
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t0, t1 = _replays(r, stream, args.steps)
        if not fused:
            d0, d1 = _replays(r, stream, args.steps, decode_only=True)
        stream.synchronize()
        ms = t0.elapsed_time(t1)
        n_win = max(1, int(math.ceil(args.clock_seconds * 1e3 / max(ms / args.steps, 1e-3))))
        n_win = min(n_win, 2_000_000)
        w0, w1, per_step = _replays_each(r, stream, n_win, start=args.steps)
    barrier()
    torch.cuda.synchronize()
    layers = w.num_layers
    dec_launches = args.steps * layers
    dec_ms = ms if fused else d0.elapsed_time(d1)
    win_ms = w0.elapsed_time(w1)
    err = pkv.get_device_error(r.pool, stream)
    if err != 0:
        raise RuntimeError("device error during the timed region: %s" % pkv.status_string(err))
    ms = max_over_ranks(ms, device)
    avg_dec_s = max_over_ranks(dec_ms, device) / dec_launches / 1e3
    units = layers * w.batch * r.queries   # decode-queries per step
    value = whole_job_rate(args.steps * units, world, ms)
    avg_bytes = r.mean_decode_bytes(0, args.steps)
    win_bytes = r.mean_decode_bytes(args.steps, n_win)

    cold_ms = None
    if cold:
        reps = min(args.steps, 50)
        cold_ms = max_over_ranks(sum(_cold_replays(r, stream, reps, decode_only=not fused)), device)
        cold_reps = reps
    append_us = None
    if not fused and r.queries == 1:
        append_us = (t0.elapsed_time(t1) - d0.elapsed_time(d1)) / dec_launches * 1e3

    e2e = run_e2e(r, stream, args.e2e_steps, device, world) if full else None
    fill = run_fill(r, stream, min(args.steps, 50), device) if full and not args.no_fill \
        else None
    cpu = None
    if cpu_seconds > 0 and world == 1 and rank == 0:
        cpu = cpu_baseline(w, r.pool_t, cpu_seconds, rows=cpu_rows)
    r.close()
    if rank != 0:
        return None

    peak, peak_kind = measured_peaks()
    achieved = avg_bytes / avg_dec_s / 1e9
    win_achieved = win_bytes / (win_ms / (n_win * layers) / 1e3) / 1e9
    clocks = clk.summary()
    clocks["window"] = {
        "what": "sampler running over the %d timed steps and %d more replays of the same "
                "step graphs right after them" % (args.steps, n_win),
        "seconds": (ms + win_ms) / 1e3, "replays": n_win,
        "us_per_launch": win_ms / (n_win * layers) * 1e3,
        "median_us_per_launch": statistics.median(per_step) / layers * 1e3,
        "achieved_gbs": win_achieved, "frac": win_achieved / peak}
    rec = {
        "workload": w.name, "description": w.description, "batch": w.batch, "layers": layers,
        "pool_pages": w.num_pages, "kv_bytes_per_layer": w.kv_bytes(1),
        "queries_per_sequence": r.queries, "out_dtype": out_dtype, "kernel": kname,
        "grid": args.grid, "min_chunk": args.min_chunk,
        "fused": fused, "flags": flags, "steps": args.steps, "ms_per_step": ms / args.steps,
        "value": value, "unit": UNIT,
        "decode_queries_per_s": w.batch * r.queries / avg_dec_s,
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": recorded_traffic(w.name, avg_bytes)
            if r.queries == 1 and out_dtype == "f32" else None,
            "peak_kind": peak_kind,
            "kernel": "decode_kernel%s (+ split-KV merge_kernel)" %
                      (" with fused append" if fused else ""),
            "alg_bytes_per_launch": avg_bytes, "avg_launch_us": avg_dec_s * 1e6,
            "launches": dec_launches},
        "gpu_launches": args.steps * layers * r.kernels_per_layer() +
                        (0 if fused else dec_launches * r.kernels_per_layer(decode_only=True)),
        "decode_timing": ("CUDA events around the %d full-step replays (fused append + decode "
                          "+ merge per layer, %d launches)" % (args.steps, dec_launches)
                          if fused else
                          "CUDA events around %d back-to-back replays of the step's decode "
                          "calls alone (decode + merge per layer, %d launches)" %
                          (args.steps, dec_launches)),
        "clocks": clocks,
        "kernel_source_sha256": kernel_source_digest(),
    }
    if cold_ms is not None:
        cold_us = cold_ms / (cold_reps * layers) * 1e3
        cold_ach = avg_bytes / (cold_us / 1e6) / 1e9
        rec["cold_l2"] = {
            "us_per_launch": cold_us, "achieved": cold_ach, "frac": cold_ach / peak,
            "how": "%d steps, each replayed alone after writing 2 x L2 bytes, CUDA events "
                   "around each replay; per launch = total / (steps x layers)" % cold_reps}
    if append_us is not None:
        rec["append"] = {
            "kernel": "append_kernel", "us_per_launch": append_us,
            "bytes_per_launch": w.batch * (2 * 2048 + 8),
            "how": "unfused step time minus decode + merge time, per layer (PDL-chained)"}
    if e2e is not None:
        rec["e2e"] = e2e
    if fill is not None:
        rec["prefill_fill"] = fill
    if cpu is not None:
        rec["cpu_baseline"] = cpu
    return rec


def run_ours(args, rank, world, local_rank):
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    main = measure(args, args.workload, device, rank, world, local_rank, full=True,
                   cold=args.cold_l2,
                   cpu_seconds=0.0 if args.no_cpu_baseline else args.cpu_seconds)
    others = []
    for name in args.also:
        rec = measure(args, name, device, rank, world, local_rank,
                      cold=name in COLD_WORKLOADS or args.cold_l2,
                      cpu_seconds=0.0 if args.no_cpu_baseline else min(args.cpu_seconds, 3.0),
                      cpu_rows=STRESS_CPU_ROWS if name == "stress_b256" else None)
        others.append(rec)
    if rank != 0:
        return None
    m = main
    line = {
        "metric": METRIC, "value": m["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": m["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": m["workload"], "description": m["description"], "batch": m["batch"],
            "layers": m["layers"], "pool_pages": m["pool_pages"],
            "kv_bytes_per_layer": m["kv_bytes_per_layer"], "accumulate": "f32",
            "kernel": m["kernel"], "parallelism": "dp%d (independent replicas)" % world,
            "queries_per_sequence": m["queries_per_sequence"], "out_dtype": m["out_dtype"],
            "launch": "one CUDA graph per step (16 x %s + split merge)%s" %
                      ("fused append+decode" if m["fused"] else
                       "%d-query decode" % m["queries_per_sequence"]
                       if m["queries_per_sequence"] > 1 else "append + decode",
                       "" if args.no_pdl else ", programmatic dependent launch, tables %sread "
                                              "before the preceding kernels end" %
                       ("and first pages " if m["flags"] & 4 else "")),
            "l2": "inputs larger than L2: one step reads %.0f MB of K/V" %
                  (m["kv_bytes_per_layer"] * m["layers"] / 1e6),
        },
        "roofline": m["roofline"],
        "decode_queries_per_s": m["decode_queries_per_s"],
        "head_queries_per_s": m["value"] * 32,
        "tokens_per_s": m["value"] / m["layers"],
        "e2e": m.get("e2e"),
        "prefill_fill": m.get("prefill_fill"),
        "gpu_launches": m["gpu_launches"],
        "decode_timing": m["decode_timing"],
        "clocks": m["clocks"],
        "kernel_source_sha256": m["kernel_source_sha256"],
    }
    for k in ("append", "cold_l2", "cpu_baseline"):
        if k in m:
            line[k] = m[k]
    if others:
        line["per_workload"] = {
            o["workload"]: {k: o[k] for k in ("value", "unit", "ms_per_step", "roofline",
                                              "decode_queries_per_s", "clocks", "cold_l2",
                                              "cpu_baseline", "batch", "layers", "steps",
                                              "description") if k in o}
            for o in others}
    return line


def run_e2e(r: Runner, stream, steps, device, world):
    """Same step through the public API, with every step's inputs (q, k_new,
    v_new of all layers, seq_lens) copied from pinned host memory before the
    step's graph runs and all outputs copied back to pinned host memory.
    Double-buffered as a serving loop would be: step i's inputs go up on one
    copy stream and step i-1's outputs come back on another while step i-1
    (then i) computes, each buffer set reused only after its previous step's
    copies are done.  The same loop runs untimed first (warm copy streams,
    pinned buffers and graphs), then `steps` steps are timed."""
    w = r.w
    sets = [r, r.twin(stream)]
    hq = r.q.cpu().pin_memory()
    hk = r.k.cpu().pin_memory()
    hv = r.v.cpu().pin_memory()
    hsl = [x.cpu().pin_memory() for x in r.seq_lens]
    hout = [torch.empty(r.out.shape, dtype=r.out.dtype).pin_memory() for _ in sets]
    h2d = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2 + hsl[0].numel() * 4
    d2h = hout[0].numel() * hout[0].element_size()
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in sets]     # inputs of the set's step are up
    ev_done = [torch.cuda.Event() for _ in sets]   # the set's step has computed
    ev_out = [torch.cuda.Event() for _ in sets]    # the set's outputs are down

    def loop(n, t0=None, t1=None):
        if t0 is not None:
            t0.record(stream)
        up.wait_stream(stream)
        down.wait_stream(stream)
        for i in range(n):
            k = i % 2
            R = sets[k]
            v = i % w.num_steps
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(ev_done[k])      # step i-2 has read this set's inputs
                R.q.copy_(hq, non_blocking=True)
                R.k.copy_(hk, non_blocking=True)
                R.v.copy_(hv, non_blocking=True)
                R.seq_lens[v].copy_(hsl[v], non_blocking=True)
                ev_in[k].record(up)
            stream.wait_event(ev_in[k])
            if i >= 2:
                stream.wait_event(ev_out[k])       # step i-2's outputs have left this set
            with torch.cuda.stream(stream):
                R.replay(i)
                ev_done[k].record(stream)
            down.wait_event(ev_done[k])
            with torch.cuda.stream(down):
                hout[k].copy_(R.out, non_blocking=True)
                ev_out[k].record(down)
        for k in range(min(n, len(sets))):
            stream.wait_event(ev_out[k])
        if t1 is not None:
            t1.record(stream)
        stream.synchronize()

    loop(max(4, min(steps, 20)))   # warm: streams, pinned buffers, the twin's graphs
    t0, t1 = _events()
    barrier()
    torch.cuda.synchronize()
    loop(steps, t0, t1)
    barrier()
    ms = max_over_ranks(t0.elapsed_time(t1), device)
    return {"value": whole_job_rate(steps * w.num_layers * w.batch * r.queries, world, ms),
            "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": ms / steps,
            "overlap": "double-buffered: host-to-device copies, step graphs and device-to-host "
                       "copies on three streams; the loop runs untimed first, then %d timed "
                       "steps" % steps}


def run_fill(r: Runner, stream, steps, device):
    """Prefill page fill (pkv_fill) of every sequence's prompt, all layers:
    one CUDA graph of num_layers fill launches, each from its own source
    buffer into that layer's pages, so a step moves far more than L2 holds.
    Algorithmic bytes per launch: each prompt token's K and V read once and
    written once (2 x 2048 B)."""
    pkv = r.pkv
    w = r.w
    counts = w.prefill_lens.astype(np.int64)
    T = int(counts.sum())
    if T == 0:
        return None
    cu = torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)).to(device)
    start = torch.zeros(w.batch, dtype=torch.int32, device=device)
    per_layer = 2 * T * 2048
    nbuf = max(1, min(w.num_layers, (8 << 30) // per_layer))
    gen = torch.Generator(device=device)
    gen.manual_seed(1234)
    src = [(torch.randn((T, 8, 64), generator=gen, device=device).to(torch.bfloat16),
            torch.randn((T, 8, 64), generator=gen, device=device).to(torch.bfloat16))
           for _ in range(nbuf)]

    def launch():
        for l in range(w.num_layers):
            k, v = src[l % nbuf]
            pkv.fill(r.pool, r.bt, cu, start, k, v, l, stream=stream)

    with torch.cuda.stream(stream):
        launch()
    stream.synchronize()
    if pkv.get_device_error(r.pool, stream) != 0:
        raise RuntimeError("device error in pkv_fill")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        launch()
    for _ in range(3):
        g.replay()
    t0, t1 = _events()
    barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(steps):
            g.replay()
        t1.record(stream)
    stream.synchronize()
    barrier()
    ms = max_over_ranks(t0.elapsed_time(t1), device)
    if pkv.get_device_error(r.pool, stream) != 0:
        raise RuntimeError("device error in pkv_fill")
    del g
    launches = steps * w.num_layers
    avg_s = ms / launches / 1e3
    peak, peak_kind = measured_peaks()
    achieved = per_layer / avg_s / 1e9
    return {"kernel": "fill_kernel", "tokens_per_launch": T, "alg_bytes_per_launch": per_layer,
            "avg_launch_us": avg_s * 1e6, "launches": launches, "achieved": achieved,
            "peak": peak, "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind,
            "source_buffers": nbuf,
            "timing": "CUDA events around %d replays of one graph of %d fill launches" %
                      (steps, w.num_layers)}


# ------------------------------------------------------------ oracle arms --

def oracle_sample(w: W.Workload, pool_t, max_seconds: float, layers=None, max_layers=None,
                  threads=None, rows=None):
    """Time the FP64 oracle on whole-layer append + decode of step 1 (the
    sequences `rows`, all by default), cycling over `layers`, until
    `max_seconds` of oracle time have passed (at least one layer; at most
    `max_layers`).  Each layer's pages are copied to the host once; repeats
    append the same token again, which rewrites the same bits.  Returns
    (queries, seconds, threads, layer-decodes done)."""
    import oracle
    layers = list(range(w.num_layers)) if layers is None else list(layers)
    rows = list(range(w.batch)) if rows is None else list(rows)
    threads = threads or os.cpu_count() or 1
    sl = w.seq_lens(1)
    cache = {}
    done, secs = 0, 0.0
    while True:
        l = layers[done % len(layers)]
        if l not in cache:
            pool_h, bt_h = W.compact_pages(w, pool_t, rows, [l])
            q, k, v = W.step_inputs(w, 1, l, pool_t.device)
            # sequences outside `rows` have no pages in the compact pool: give
            # them length 0 (skipped by append and decode)
            sl_rows = np.zeros_like(sl)
            sl_rows[rows] = sl[rows]
            cache[l] = (pool_h, bt_h, W.bits(q), W.bits(k), W.bits(v), sl_rows)
        pool_h, bt_h, qb, kb, vb, sl_rows = cache[l]
        t = time.perf_counter()
        oracle.append(pool_h, bt_h[:, rows], sl_rows[rows], kb[rows], vb[rows], l)
        oracle.decode(qb, pool_h, bt_h, sl_rows, l, w.scale, rows=rows, nthreads=threads)
        secs += time.perf_counter() - t
        done += 1
        if secs >= max_seconds or (max_layers is not None and done >= max_layers):
            break
    return done * len(rows), secs, threads, done


def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w, pool_t, max_seconds, rows=None):
    """The FP64 oracle on the host cores (all threads, then one) on whole
    layers of step 1 (`rows`: a sample of the batch, reported as such)."""
    q, s, thr, layers = oracle_sample(w, pool_t, max_seconds, max_layers=4096, rows=rows)
    q1, s1, _, layers1 = oracle_sample(w, pool_t, max_seconds / 4, max_layers=4096, threads=1,
                                       rows=rows)
    nrows = w.batch if rows is None else len(rows)
    what = "whole-layer" if rows is None else \
        "%d-of-%d-sequence (extrapolated: the rate per sequence is the same)" % (nrows, w.batch)
    return {"value": q / s, "unit": UNIT, "cores": thr, "kind": "oracle",
            "sample": "%d %s append+decode(s) of step 1, cycling over the %d layers "
                      "(%d sequences each), %.1f s of FP64 oracle work" %
                      (layers, what, w.num_layers, nrows, s),
            "cpu_model": cpu_model(),
            "single_core_value": q1 / s1,
            "single_core_sample": "%d %s append+decode(s) on 1 thread, %.1f s" %
                                  (layers1, what, s1)}


def run_reference(args, rank, world, local_rank):
    """The oracle as the reference arm: each step is a bounded sample of the
    same workload -- append of the layer's new tokens and decode of as many
    of its sequences (cycling through the batch) as fit the step's share of
    --reference-seconds -- so that the whole run takes about that long
    whatever the workload and step count."""
    import oracle
    if rank != 0:
        return None
    w = W.make(args.workload)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    if W.Workload.pool_bytes(w) > 8e9 and dev == "cpu":
        raise SystemExit("pool too large to generate on the host")
    pool_t = W.make_pool(w, dev)
    nl, B = w.num_layers, w.batch
    threads = os.cpu_count() or 1
    sl = w.seq_lens(1)
    cache = {}

    def layer_inputs(l):
        if l not in cache:
            pool_h, bt_h = W.compact_pages(w, pool_t, range(B), [l])
            q, k, v = W.step_inputs(w, 1, l, pool_t.device)
            cache[l] = (pool_h, bt_h, W.bits(q), W.bits(k), W.bits(v))
        return cache[l]

    def step(l, rows):
        # appending the same token again rewrites the same bits, so the
        # layer's pages need no fresh copy between steps
        pool_h, bt_h, qb, kb, vb = layer_inputs(l)
        t = time.perf_counter()
        oracle.append(pool_h, bt_h, sl, kb, vb, l)
        oracle.decode(qb, pool_h, bt_h, sl, l, w.scale, rows=rows, nthreads=threads)
        return time.perf_counter() - t

    # calibrate: seconds per sequence of one layer
    per_row = step(0, list(range(B))) / B
    budget = args.reference_seconds / max(1, args.steps + args.warmup)
    n = int(max(1, min(B, budget / max(per_row, 1e-9))))
    rows_of = lambda i: [(i * n + j) % B for j in range(n)]
    for i in range(args.warmup):
        step(i % nl, rows_of(i))
    q_tot, s_tot = 0, 0.0
    for i in range(args.steps):
        s_tot += step(i % nl, rows_of(i))
        q_tot += n
    v = q_tot / s_tot
    sample = ("%d steps x (append of one layer's %d new tokens + decode of %d of its %d "
              "sequences, cycling over layers and sequences)" % (args.steps, B, n, B))
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": s_tot / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "description": w.description, "batch": B,
                   "layers": nl, "sample": sample},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample, "cpu_model": cpu_model()},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------ table --

# Workloads whose layer fits in L2 (26.9 MB and 0.1 MB of K/V): reported hot
# and cold.
COLD_WORKLOADS = ("tiny", "llama1b_b16")
# Sampled CPU baseline for the 35 GB workload (8 of its 256 sequences).
STRESS_CPU_ROWS = [0, 37, 64, 101, 128, 199, 230, 255]


def run_table(args, rank, world, local_rank):
    """Every workload and option row of the measured-results table in one
    run, on the current kernel sources: JSON line per row, then markdown."""
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    rows = []

    def add(label, name, **kw):
        rec = measure(args, name, device, rank, world, local_rank, **kw)
        if rec is not None:
            rec["row"] = label
            print(json.dumps(rec), flush=True)
            rows.append(rec)

    for name in ("tiny", "llama1b_b16", "continuous_batching_b64", "long_context_b4",
                 "stress_b256"):
        add(name, name, full=name != "stress_b256", cold=name in COLD_WORKLOADS,
            cpu_seconds=0.0 if args.no_cpu_baseline else 3.0,
            cpu_rows=STRESS_CPU_ROWS if name == "stress_b256" else None)
    for name, qs in (("continuous_batching_b64", (2, 4, 8)), ("long_context_b4", (2, 8))):
        for q in qs:
            add("%s, %d queries" % (name, q), name, queries=q)
    add("continuous_batching_b64, BF16 output", "continuous_batching_b64", out_dtype="bf16")
    if rank != 0:
        return
    print("| row | us per launch | alg. GB/s | of peak | cold L2: us, of peak | "
          "decode-queries/s (step) | e2e | fill GB/s (of peak) | CPU oracle (cores) | "
          "SM MHz (samples, reasons) |")
    print("|---|---|---|---|---|---|---|---|---|---|")
    for r in rows:
        rf, c = r["roofline"], r["clocks"]
        cold = r.get("cold_l2")
        e2e = r.get("e2e")
        fill = r.get("prefill_fill")
        cpu = r.get("cpu_baseline")
        print("| %s | %.2f | %.0f | %.1f %% | %s | %.4g | %s | %s | %s | %s (%d, %s) |" % (
            r["row"], rf["avg_launch_us"], rf["achieved"], 100 * rf["frac"],
            "%.2f, %.1f %%" % (cold["us_per_launch"], 100 * cold["frac"]) if cold else "-",
            r["value"], "%.4g" % e2e["value"] if e2e else "-",
            "%.0f (%.1f %%)" % (fill["achieved"], 100 * fill["frac"]) if fill else "-",
            "%.4g (%d)" % (cpu["value"], cpu["cores"]) if cpu else "-",
            c.get("sm_mhz"), c.get("samples", 0), ",".join(c.get("reasons", [])) or "none"))


# --------------------------------------------------------------------- main --

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="continuous_batching_b64", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "mma"])
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--clock-seconds", type=float, default=1.0,
                    help="replay the step graphs at least this long with the clock sampler on")
    ap.add_argument("--also", default=None,
                    help="comma-separated workloads measured beside the main one (default: "
                         "long_context_b4,llama1b_b16,stress_b256 for the default workload; "
                         "'none')")
    ap.add_argument("--cold-l2", action="store_true",
                    help="also time the main workload with L2 flushed before every step")
    ap.add_argument("--table", action="store_true",
                    help="measure every workload and option row; print JSON lines and a table")
    ap.add_argument("--reference-seconds", type=float, default=60.0,
                    help="oracle time the --impl reference run spends in its timed steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fill", action="store_true", help="skip the prefill fill timing")
    ap.add_argument("--no-early-pages", action="store_true",
                    help="wait for the preceding kernels before the first page loads")
    ap.add_argument("--queries", type=int, default=1, choices=range(1, 9),
                    help="queries per sequence (> 1: causal among them, decode only)")
    ap.add_argument("--out-dtype", default="f32", choices=["f32", "bf16"])
    ap.add_argument("--grid", type=int, default=0,
                    help="decode CTAs (0: one persistent wave over the device)")
    ap.add_argument("--min-chunk", type=int, default=0,
                    help="minimum pages per decode CTA range (0: automatic)")
    ap.add_argument("--unfused", action="store_true",
                    help="separate append and decode launches instead of the fused call")
    ap.add_argument("--no-pdl", action="store_true",
                    help="launch without programmatic dependent launch")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.also is None:
        args.also = ["long_context_b4", "llama1b_b16", "stress_b256"] \
            if args.workload == "continuous_batching_b64" else []
    else:
        args.also = [] if args.also in ("", "none") else args.also.split(",")
    for name in args.also:
        if name not in W.WORKLOADS:
            ap.error("unknown workload %s" % name)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world, local_rank)
        elif args.table:
            run_table(args, rank, world, local_rank)
            line = None
        else:
            line = run_ours(args, rank, world, local_rank)
        if line is not None and rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as tdist
            tdist.destroy_process_group()


if __name__ == "__main__":
    main()
