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
                    [--e2e-steps N] [--cpu-seconds S] [--reference-seconds S]

Prints one JSON line (rank 0).  ``value`` is decode-queries/s over all
ranks, one query being one sequence's 32 query heads at one layer
(``head_queries_per_s`` counts heads, ``tokens_per_s`` sequences' tokens
per whole-model step; ``append``, in --unfused runs, the separate append's
share of a layer).  The
``roofline`` object reports the decode kernel's algorithmic HBM bytes per
launch divided by its measured average launch time, against the measured
HBM copy bandwidth, with the DRAM traffic of the committed ncu capture.
``e2e`` is the same step with its inputs and outputs crossing from and to
pinned host memory every step; ``prefill_fill`` the page-fill bandwidth;
``cpu_baseline`` the FP64 oracle on the host cores.  ``--impl reference``
times the FP64 CPU oracle on the same workload instead (bounded sample per
step, host cores).
"""
from __future__ import annotations

import argparse
import json
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
                 "--format=csv,noheader,nounits", "-lms", "100"],
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

class Runner:
    """Device-resident state of one workload on one GPU."""

    def __init__(self, w: W.Workload, device, kernel: int, fused: bool, queries: int = 1,
                 out_dtype=torch.float32, grid: int = 0):
        from paged_attention_decode_pkv_b200 import pkv
        self.pkv = pkv
        self.w = w
        self.device = device
        self.kernel = kernel
        self.grid = grid
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
        t.capture(stream)
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
                                   grid_ctas=self.grid,
                                   stream=stream, **kv)
                continue
            if self.fused:
                pkv.decode_append(self.q[l], self.k[l], self.v[l], self.pool, self.bt, sl, l,
                                  self.w.scale, out=self.out[l], workspace=self.ws,
                                  kernel=self.kernel, grid_ctas=self.grid, stream=stream)
                continue
            if not decode_only:
                pkv.append(self.pool, self.bt, sl, self.k[l], self.v[l], l, stream=stream)
            pkv.decode(self.q[l], self.pool, self.bt, sl, l, self.w.scale, out=self.out[l],
                       workspace=self.ws, kernel=self.kernel, grid_ctas=self.grid,
                       stream=stream)

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


def run_ours(args, rank, world, local_rank):
    from paged_attention_decode_pkv_b200 import pkv
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    kernel = {"auto": pkv.KERNEL_AUTO, "simt": pkv.KERNEL_SIMT, "mma": pkv.KERNEL_MMA}[args.kernel]
    w = workload_for_rank(args.workload, rank)
    fused = not args.unfused and args.queries == 1
    out_dtype = torch.bfloat16 if args.out_dtype == "bf16" else torch.float32
    r = Runner(w, device, kernel, fused, args.queries, out_dtype, args.grid)
    flags = 0
    if not args.no_pdl:
        # No kernel of the step writes the lengths or the block tables.  With
        # no separate append, the kernel before each decode (the previous
        # layer's decode or merge) writes no page that decode reads, so its
        # first page loads start early too (--no-early-pages turns that off).
        flags = pkv.LAUNCH_PDL | pkv.LAUNCH_EARLY_TABLES
        if (fused or args.queries > 1) and not args.no_early_pages:
            flags |= pkv.LAUNCH_EARLY_PAGES
        r.pool.set_launch_flags(flags)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            r.launch_step(stream, i % w.num_steps)
    stream.synchronize()
    assert pkv.get_device_error(r.pool, stream) == 0
    r.capture(stream)
    for i in range(max(args.warmup, w.num_steps)):
        r.replay(i)
    torch.cuda.synchronize()

    # ---- timed region: (A) K full steps; unfused only, then (B) the decodes
    # of K steps alone, back to back, for the decode kernel's launch duration
    # (fused, a step is nothing but the decode launches, so (A) gives it)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if not fused:
        for i in range(max(args.warmup, w.num_steps)):
            r.replay_decodes(i)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        with torch.cuda.stream(stream):
            t0.record(stream)
            for i in range(args.steps):
                r.replay(i)
            t1.record(stream)
            if not fused:
                d0.record(stream)
                for i in range(args.steps):
                    r.replay_decodes(i)
                d1.record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
    barrier()
    ms = t0.elapsed_time(t1)
    dec_launches = args.steps * w.num_layers
    dec_ms = t0.elapsed_time(t1) if fused else d0.elapsed_time(d1)
    avg_dec_s = max_over_ranks(dec_ms, device) / dec_launches / 1e3
    avg_bytes = sum(r.decode_bytes(i) for i in range(args.steps)) / args.steps
    err = pkv.get_device_error(r.pool, stream)
    if err != 0:
        raise RuntimeError("device error during timed region: %s" % pkv.status_string(err))
    ms = max_over_ranks(ms, device)
    value = whole_job_rate(args.steps * w.num_layers * w.batch * r.queries, world, ms)

    # ---- end to end through the public API from pinned host buffers
    e2e = run_e2e(r, stream, min(args.steps, args.e2e_steps), device, world)

    # ---- prefill page fill bandwidth (rewrites the prompt tokens' values)
    fill = None if args.no_fill else run_fill(r, stream, min(args.steps, 50), device)

    if rank != 0:
        return None
    peak, peak_kind = measured_peaks()
    achieved = avg_bytes / avg_dec_s / 1e9
    traffic = recorded_traffic(w.name, avg_bytes)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": w.name, "description": w.description, "batch": w.batch,
            "layers": w.num_layers, "pool_pages": w.num_pages,
            "kv_bytes_per_layer": w.kv_bytes(1), "accumulate": "f32",
            "kernel": args.kernel, "parallelism": "dp%d (independent replicas)" % world,
            "queries_per_sequence": r.queries, "out_dtype": args.out_dtype,
            "launch": "one CUDA graph per step (16 x %s + split merge)%s" %
                      ("fused append+decode" if fused else
                       "%d-query decode" % r.queries if r.queries > 1 else "append + decode",
                       "" if args.no_pdl else ", programmatic dependent launch, tables %sread "
                                              "before the preceding kernel ends" %
                       ("and first pages " if flags & pkv.LAUNCH_EARLY_PAGES else "")),
            "l2": "inputs larger than L2: one step reads %.0f MB of K/V" %
                  (w.kv_bytes(1) * w.num_layers / 1e6),
        },
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": traffic, "peak_kind": peak_kind,
            "kernel": "decode_kernel%s (+ split-KV merge_kernel)" %
                      (" with fused append" if fused else ""),
            "alg_bytes_per_launch": avg_bytes, "avg_launch_us": avg_dec_s * 1e6,
            "launches": dec_launches,
        },
        "decode_queries_per_s": w.batch * r.queries / avg_dec_s,
        "head_queries_per_s": value * 32,
        "tokens_per_s": value / w.num_layers,
        "e2e": e2e,
        "prefill_fill": fill,
        "gpu_launches": (args.steps * w.num_layers * (2 if fused or r.queries > 1 else 3) +
                         (0 if fused else dec_launches * 2)),
        "decode_timing": ("CUDA events around the %d full-step replays (fused append + decode "
                          "+ merge per layer, %d launches)" % (args.steps, dec_launches)
                          if fused else
                          "CUDA events around %d back-to-back replays of the step's decode "
                          "launches alone (decode + merge per layer, %d launches)" %
                          (args.steps, dec_launches)),
        "clocks": clk.summary(),
    }
    if not fused and r.queries == 1:
        # the separate append's share of a layer: full step replays minus the
        # replays of the same decode + merge launches alone
        line["append"] = {
            "kernel": "append_kernel", "us_per_launch":
                (t0.elapsed_time(t1) - d0.elapsed_time(d1)) / dec_launches * 1e3,
            "bytes_per_launch": w.batch * (2 * 2048 + 8),
            "how": "unfused step time minus decode + merge time, per layer (PDL-chained)"}
    if not args.no_cpu_baseline and world == 1:   # the host baseline is taken at N = 1 only
        line["cpu_baseline"] = cpu_baseline(w, r.pool_t, args.cpu_seconds)
    return line


def run_e2e(r: Runner, stream, steps, device, world):
    """Same step through the public API, with every step's inputs (q, k_new,
    v_new of all layers, seq_lens) copied from pinned host memory before the
    step's graph runs and all outputs copied back to pinned host memory.
    Double-buffered as a serving loop would be: step i's inputs go up on one
    copy stream and step i-1's outputs come back on another while step i-1
    (then i) computes, each buffer set reused only after its previous step's
    copies are done."""
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
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    up.wait_event(t0)
    down.wait_event(t0)
    for i in range(steps):
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
    for k in range(len(sets)):
        stream.wait_event(ev_out[k])
    t1.record(stream)
    stream.synchronize()
    barrier()
    ms = max_over_ranks(t0.elapsed_time(t1), device)
    return {"value": whole_job_rate(steps * w.num_layers * w.batch * r.queries, world, ms),
            "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": ms / steps,
            "overlap": "double-buffered: host-to-device copies, step graphs and device-to-host "
                       "copies on three streams"}


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
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
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
                  threads=None):
    """Time the FP64 oracle on whole-layer append + decode of step 1 (all
    sequences of the batch), cycling over `layers`, until `max_seconds` of
    oracle time have passed (at least one layer; at most `max_layers`).
    Each layer's pages are copied to the host once; repeats append the same
    token again, which rewrites the same bits.  Returns (queries, seconds,
    threads, layer-decodes done)."""
    import oracle
    layers = list(range(w.num_layers)) if layers is None else list(layers)
    threads = threads or os.cpu_count() or 1
    sl = w.seq_lens(1)
    cache = {}
    done, secs = 0, 0.0
    while True:
        l = layers[done % len(layers)]
        if l not in cache:
            pool_h, bt_h = W.compact_pages(w, pool_t, range(w.batch), [l])
            q, k, v = W.step_inputs(w, 1, l, pool_t.device)
            cache[l] = (pool_h, bt_h, W.bits(q), W.bits(k), W.bits(v))
        pool_h, bt_h, qb, kb, vb = cache[l]
        t = time.perf_counter()
        oracle.append(pool_h, bt_h, sl, kb, vb, l)
        oracle.decode(qb, pool_h, bt_h, sl, l, w.scale, nthreads=threads)
        secs += time.perf_counter() - t
        done += 1
        if secs >= max_seconds or (max_layers is not None and done >= max_layers):
            break
    return done * w.batch, secs, threads, done


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


def cpu_baseline(w, pool_t, max_seconds):
    q, s, thr, layers = oracle_sample(w, pool_t, max_seconds, max_layers=4096)
    q1, s1, _, layers1 = oracle_sample(w, pool_t, max_seconds / 4, max_layers=4096, threads=1)
    return {"value": q / s, "unit": UNIT, "cores": thr, "kind": "oracle",
            "sample": "%d whole-layer append+decode(s) of step 1, cycling over the %d layers "
                      "(%d sequences each), %.1f s of FP64 oracle work" %
                      (layers, w.num_layers, w.batch, s),
            "cpu_model": cpu_model(),
            "single_core_value": q1 / s1,
            "single_core_sample": "%d whole-layer append+decode(s) on 1 thread, %.1f s" %
                                  (layers1, s1)}


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


# --------------------------------------------------------------------- main --

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="continuous_batching_b64", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "mma"])
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-seconds", type=float, default=60.0,
                    help="oracle time the --impl reference run spends in its timed steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fill", action="store_true", help="skip the prefill fill timing")
    ap.add_argument("--no-early-pages", action="store_true",
                    help="wait for the preceding kernel before the first page loads")
    ap.add_argument("--queries", type=int, default=1, choices=range(1, 9),
                    help="queries per sequence (> 1: causal among them, decode only)")
    ap.add_argument("--out-dtype", default="f32", choices=["f32", "bf16"])
    ap.add_argument("--grid", type=int, default=0,
                    help="decode CTAs (0: one persistent wave over the device)")
    ap.add_argument("--unfused", action="store_true",
                    help="separate append and decode launches instead of the fused call")
    ap.add_argument("--no-pdl", action="store_true",
                    help="launch without programmatic dependent launch")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

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
