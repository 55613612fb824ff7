"""Seeded synthetic workloads for paged decode attention.

This module only makes inputs: sequence lengths, page allocation (block
tables), and the random BF16 contents of the pool, the queries and the new
keys/values.  It holds none of the attention arithmetic, so both the CUDA
path and the CPU oracle can be fed from it.

The five workloads follow the shapes the pages give for the Llama-3.2-1B
engine: 16-token BF16 pages in one shared pool with a block table per
sequence and layer ("Curso gratuito recorre la inferencia de LLM...",
section on the KV cache), 32 query heads over 8 kv heads of dimension 64 and
16 layers ("Construye tu propio motor de inferencia LLM...", section "La
arquitectura del modelo: Llama 3.2 1B"), and continuous batching that hands
pages out from a pool and frees them when sequences end (same two pages,
batching sections).  Values are N(0, 1) rounded to BF16 (round to nearest
even), as the workloads prescribe.

Randomness: lengths, page permutations and the allocation trace come from a
CPU ``torch.Generator`` seeded per workload, so they are identical on every
machine.  Tensor contents come from a generator on the requested device;
CPU and CUDA streams differ, so a parity check always hands the *same
realised bits* to both sides (the oracle reads back what was generated,
before any kernel touched it).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch

PAGE_TOKENS = 16
NUM_KV_HEADS = 8
NUM_Q_HEADS = 32
HEAD_DIM = 64
NUM_LAYERS_LLAMA_1B = 16
PAGE_ELEMS = 2 * NUM_KV_HEADS * PAGE_TOKENS * HEAD_DIM  # 16384 BF16 = 32 KiB
BF16_NAN_BITS = 0x7FC0


@dataclasses.dataclass
class Workload:
    """One synthetic decode workload.

    ``prefill_lens[b]`` tokens are already in the cache before step 1; step s
    (1-based) appends one token per sequence, so the length after step s is
    ``prefill_lens + s``.  ``block_tables`` already hold every page the
    sequences need through ``num_steps`` (-1 marks unused entries).
    """

    name: str
    seed: int
    batch: int
    num_layers: int
    num_pages: int
    block_tables: np.ndarray  # int32 [num_layers, batch, max_blocks]
    prefill_lens: np.ndarray  # int32 [batch]
    num_steps: int
    scale: float = 0.125
    key_outlier_prob: float = 0.0  # Bernoulli probability of a x4 key row
    key_outlier_scale: float = 4.0
    description: str = ""

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[2])

    def seq_lens(self, step: int) -> np.ndarray:
        """Lengths after the append of step ``step`` (1-based)."""
        if not 1 <= step <= self.num_steps:
            raise ValueError("step %d outside 1..%d" % (step, self.num_steps))
        return (self.prefill_lens + step).astype(np.int32)

    def pool_bytes(self) -> int:
        return self.num_pages * PAGE_ELEMS * 2

    def kv_bytes(self, step: int) -> int:
        """K+V bytes one layer's decode reads at ``step`` (2048 B per token)."""
        return int(self.seq_lens(step).astype(np.int64).sum()) * 2 * NUM_KV_HEADS * HEAD_DIM * 2


# ----------------------------------------------------------------- helpers --

def _cpu_gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _pages_for(length: int) -> int:
    return (int(length) + PAGE_TOKENS - 1) // PAGE_TOKENS


def _deal_pages(perm: np.ndarray, need: np.ndarray) -> np.ndarray:
    """Deal pages of ``perm`` in (layer, seq, page) order; need is [L, B]."""
    num_layers, batch = need.shape
    max_blocks = max(1, int(need.max()))
    bt = np.full((num_layers, batch, max_blocks), -1, np.int32)
    cur = 0
    for layer in range(num_layers):
        for b in range(batch):
            n = int(need[layer, b])
            bt[layer, b, :n] = perm[cur:cur + n]
            cur += n
    return bt


def _log_uniform_lengths(gen: torch.Generator, n: int, hi: int) -> np.ndarray:
    """clamp(floor(exp(U * ln hi)), 1, hi), U ~ U[0, 1)."""
    u = torch.rand(n, generator=gen, dtype=torch.float64).numpy()
    return np.clip(np.floor(np.exp(u * math.log(hi))), 1, hi).astype(np.int64)


# -------------------------------------------------------------- workloads --

def tiny(seed: int = 1) -> Workload:
    """2 sequences with 17 and 40 tokens after the append, one layer,
    16-page pool with shuffled physical pages, scale 1/8."""
    gen = _cpu_gen(seed)
    perm = torch.randperm(16, generator=gen).numpy().astype(np.int32)
    final = np.array([17, 40], np.int64)
    need = np.array([[_pages_for(x) for x in final]])
    bt = _deal_pages(perm, need)
    return Workload("tiny", seed, 2, 1, 16, bt, (final - 1).astype(np.int32), 1, 0.125,
                    description="B=2, L=(17,40), 1 layer, 16-page shuffled pool")


def llama1b(seed: int = 2) -> Workload:
    """Batch 16, lengths uniform in [1, 2048] after the append, 16 layers;
    pages from one shared pool of max(4096, needed) pages, randomly assigned."""
    gen = _cpu_gen(seed)
    final = torch.randint(1, 2049, (16,), generator=gen).numpy().astype(np.int64)
    need = np.tile(np.array([_pages_for(x) for x in final]), (16, 1))
    n_pool = max(4096, int(need.sum()))
    perm = torch.randperm(n_pool, generator=gen).numpy().astype(np.int32)
    bt = _deal_pages(perm, need)
    return Workload("llama1b_b16", seed, 16, 16, n_pool, bt, (final - 1).astype(np.int32), 1,
                    description="B=16, L~U[1,2048], 16 layers, random pages, pool max(4096, need)")


def continuous_batching(seed: int = 3, batch: int = 64, steps: int = 16,
                        churn_rounds: int = 4, phantoms: int = 256) -> Workload:
    """Batch 64, final-step lengths log-uniform in [1, 8192], 16 layers,
    ``steps`` decode steps, and block tables fragmented by an alloc/free trace.

    Trace (the pages do not give one; this is the plainest reading of "pages
    are handed out from a shared pool and freed when a sequence ends"):
    the free list starts as a random permutation of the pool and is used as a
    LIFO stack.  In each of ``churn_rounds`` rounds, ``phantoms`` short-lived
    sequences with log-uniform lengths take pages one at a time, round-robin
    over (sequence, layer), as long as more pages than the live batch needs
    remain free; then a random half of all phantom sequences held so far end,
    in random order, pushing their pages back.  After the last round every
    remaining phantom ends (random order) and the live batch takes its pages
    round-robin over (page index, sequence, layer).
    """
    gen = _cpu_gen(seed)
    nl = NUM_LAYERS_LLAMA_1B
    d = _log_uniform_lengths(gen, batch, 8192)          # length at step 1
    prefill = d - 1
    final = prefill + steps
    need_seq = np.array([_pages_for(x) for x in final], np.int64)
    need = int(need_seq.sum()) * nl
    n_pool = int(math.ceil(1.5 * need))
    free: List[int] = torch.randperm(n_pool, generator=gen).numpy().astype(np.int64).tolist()
    held = {}
    next_id = 0
    for _ in range(churn_rounds):
        plen = _log_uniform_lengths(gen, phantoms, 8192)
        ppages = np.array([_pages_for(x) for x in plen], np.int64)
        # round-robin order: (page index j, phantom p, layer) for j < ppages[p]
        jmax = int(ppages.max())
        jj, pp, ll = np.meshgrid(np.arange(jmax), np.arange(phantoms), np.arange(nl), indexing="ij")
        jj, pp, ll = jj.ravel(), pp.ravel(), ll.ravel()
        keep = jj < ppages[pp]
        pp = pp[keep]
        budget = max(0, len(free) - need)
        pp = pp[:budget]
        taken = free[len(free) - len(pp):][::-1] if len(pp) else []
        if len(pp):
            del free[len(free) - len(pp):]
        ids = np.arange(next_id, next_id + phantoms)
        for p, page in zip(pp.tolist(), taken):
            held.setdefault(int(ids[p]), []).append(page)
        next_id += phantoms
        keys = sorted(held)
        order = torch.randperm(len(keys), generator=gen).numpy()
        for k in order[: len(keys) // 2]:
            free.extend(held.pop(keys[int(k)]))
    keys = sorted(held)
    order = torch.randperm(len(keys), generator=gen).numpy()
    for k in order:
        free.extend(held.pop(keys[int(k)]))
    max_blocks = int(need_seq.max())
    bt = np.full((nl, batch, max_blocks), -1, np.int32)
    for j in range(max_blocks):
        for b in range(batch):
            if j < need_seq[b]:
                for layer in range(nl):
                    bt[layer, b, j] = free.pop()
    return Workload("continuous_batching_b64", seed, batch, nl, n_pool, bt,
                    prefill.astype(np.int32), steps,
                    description="B=64, L log-uniform [1,8192], 16 layers x %d steps, "
                                "fragmented block tables from a seeded alloc/free trace" % steps)


def long_context(seed: int = 4) -> Workload:
    """Batch 4 with 32768/65536/98304/131072 tokens after the append, one
    layer, pages placed by a random permutation of a pool with 8 spare pages;
    5% of key rows scaled by 4 before rounding to BF16."""
    gen = _cpu_gen(seed)
    final = np.array([32768, 65536, 98304, 131072], np.int64)
    need = np.array([[_pages_for(x) for x in final]])
    n_pool = int(need.sum()) + 8
    perm = torch.randperm(n_pool, generator=gen).numpy().astype(np.int32)
    bt = _deal_pages(perm, need)
    return Workload("long_context_b4", seed, 4, 1, n_pool, bt, (final - 1).astype(np.int32), 1,
                    key_outlier_prob=0.05,
                    description="B=4, L=32k/64k/96k/128k, 1 layer, 5% keys x4")


def stress(seed: int = 5, steps: int = 50, batch: int = 256, prefill: int = 4095) -> Workload:
    """Batch 256 with 4095 cached tokens, 16 layers, ``steps`` decode steps
    (4096 .. 4095+steps tokens), pages placed by a random permutation."""
    gen = _cpu_gen(seed)
    nl = NUM_LAYERS_LLAMA_1B
    final = prefill + steps
    per = _pages_for(final)
    need = np.full((nl, batch), per, np.int64)
    n_pool = int(need.sum())
    perm = torch.randperm(n_pool, generator=gen).numpy().astype(np.int32)
    bt = _deal_pages(perm, need)
    return Workload("stress_b256", seed, batch, nl, n_pool, bt,
                    np.full(batch, prefill, np.int32), steps,
                    description="B=256, L=4096..%d, 16 layers, random pages" % final)


WORKLOADS = {
    "tiny": tiny,
    "llama1b_b16": llama1b,
    "continuous_batching_b64": continuous_batching,
    "long_context_b4": long_context,
    "stress_b256": stress,
}


def make(name: str, **kw) -> Workload:
    return WORKLOADS[name](**kw)


# --------------------------------------------------------- tensor contents --

def _dev_gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def written_slots(w: Workload) -> np.ndarray:
    """bool [num_pages, 16]: slots holding a prefilled token of some
    (layer, sequence).  Everything else in the pool is never valid input."""
    mask = np.zeros((w.num_pages, PAGE_TOKENS), bool)
    for layer in range(w.num_layers):
        for b in range(w.batch):
            n = int(w.prefill_lens[b])
            if n == 0:
                continue
            full, rem = divmod(n, PAGE_TOKENS)
            pages = w.block_tables[layer, b]
            if full:
                mask[pages[:full]] = True
            if rem:
                mask[pages[full], :rem] = True
    return mask


def make_pool(w: Workload, device="cpu", chunk_pages: int = 4096,
              poison: bool = True) -> torch.Tensor:
    """Pool contents before step 1: bfloat16 [num_pages, 2, 8, 16, 64].

    Prefilled slots hold N(0,1) values rounded to BF16 (key rows scaled by
    ``key_outlier_scale`` with probability ``key_outlier_prob`` before the
    rounding).  With ``poison``, every slot that holds no prefilled token
    (tails of last pages, pages reserved for later steps, unused pages) is
    set to the BF16 quiet NaN 0x7FC0, so any read of it shows up.
    """
    device = torch.device(device)
    gen = _dev_gen(device, w.seed * 7919 + 17)
    pool = torch.empty((w.num_pages, 2, NUM_KV_HEADS, PAGE_TOKENS, HEAD_DIM),
                       dtype=torch.bfloat16, device=device)
    for p0 in range(0, w.num_pages, chunk_pages):
        p1 = min(w.num_pages, p0 + chunk_pages)
        x = torch.randn((p1 - p0, 2, NUM_KV_HEADS, PAGE_TOKENS, HEAD_DIM), generator=gen,
                        device=device, dtype=torch.float32)
        if w.key_outlier_prob > 0:
            sel = torch.rand((p1 - p0, NUM_KV_HEADS, PAGE_TOKENS), generator=gen,
                             device=device) < w.key_outlier_prob
            x[:, 0] = torch.where(sel[..., None], x[:, 0] * w.key_outlier_scale, x[:, 0])
        pool[p0:p1] = x.to(torch.bfloat16)
        del x
    if poison:
        keep = torch.from_numpy(written_slots(w)).to(device)
        bits = pool.view(torch.int16)
        bits.masked_fill_(~keep[:, None, None, :, None], BF16_NAN_BITS)
    return pool


def step_inputs(w: Workload, step: int, layer: int, device="cpu"):
    """(q [B,32,64], k_new [B,8,64], v_new [B,8,64]) bfloat16 for one
    (step, layer).  Each (step, layer) has its own seed, so any subset can be
    regenerated without the others."""
    device = torch.device(device)
    gen = _dev_gen(device, (w.seed * 1_000_003 + step * 1009 + layer) & 0x7FFFFFFFFFFF)
    q = torch.randn((w.batch, NUM_Q_HEADS, HEAD_DIM), generator=gen, device=device)
    k = torch.randn((w.batch, NUM_KV_HEADS, HEAD_DIM), generator=gen, device=device)
    v = torch.randn((w.batch, NUM_KV_HEADS, HEAD_DIM), generator=gen, device=device)
    if w.key_outlier_prob > 0:
        sel = torch.rand((w.batch, NUM_KV_HEADS), generator=gen, device=device) < w.key_outlier_prob
        k = torch.where(sel[..., None], k * w.key_outlier_scale, k)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    """BF16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def compact_pages(w: Workload, pool: torch.Tensor, rows, layers):
    """Host copy of only the pages that sequences ``rows`` use at ``layers``,
    with block tables renumbered into that small pool.

    Returns (pool_u16 [n, 2, 8, 16, 64], block_tables int32 [num_layers,
    batch, max_blocks]); entries of other sequences/layers are -1.  Used to
    check sampled sequences of pools too large to copy whole.
    """
    rows = list(rows)
    layers = list(layers)
    sel = np.unique(np.concatenate([w.block_tables[l, b][w.block_tables[l, b] >= 0]
                                    for l in layers for b in rows]))
    remap = np.full(w.num_pages, -1, np.int64)
    remap[sel] = np.arange(sel.size)
    bt = np.full_like(w.block_tables, -1)
    for l in layers:
        for b in rows:
            src = w.block_tables[l, b]
            bt[l, b] = np.where(src >= 0, remap[np.maximum(src, 0)], -1)
    idx = torch.from_numpy(sel.astype(np.int64)).to(pool.device)
    small = pool.index_select(0, idx)
    return bits(small), bt.astype(np.int32)
