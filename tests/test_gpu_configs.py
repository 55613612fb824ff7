"""GPU parity on the full-size workloads, through the C ABI, against the FP64
oracle on the same input bits.

Each test runs the workload's decode steps the way the benchmark does
(append and decode, layer by layer, step by step; as two calls or as the
fused call the benchmark times) and checks, against the oracle:
  - attention output: max abs error <= 2e-3 at the sampled (step, layer)
    points, for every sequence (or a sample of sequences for the 35 GB
    pool);
  - append and page indexing: the GPU pool's pages of the sampled
    sequences and layers are bit-identical to the oracle's pool model after
    all the appends (every appended slot and every untouched slot of those
    pages).
The 35 GB stress pool is also checked on the GPU for all sequences: every
appended slot holds exactly the new token's bits and a per-slot checksum of
every other slot of the pool is unchanged.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_attention_decode_pkv_b200 import pkv
from paged_attention_decode_pkv_b200 import workloads as W
from tests.harness import ATOL, KERNELS, bits, max_err, to_dev

pytestmark = pytest.mark.gpu


def _append_rows(host_pool, host_bt, sl_np, kb, vb, layer, rows):
    """Oracle append restricted to `rows` (the other sequences have no pages
    in the compact host model)."""
    oracle.append(host_pool, host_bt[:, rows, :], sl_np[rows], kb[rows], vb[rows], layer)


def _run(w, kernel, sample_layers, sample_steps, rows=None, flags=0, on_pool=None, fused=False):
    """Run every step x layer of `w` on the GPU.  Returns (GPU outputs and
    oracle outputs at the sampled points for `rows`, GPU and oracle copies
    of the pages those rows use at the sampled layers)."""
    dev = "cuda"
    rows = np.arange(w.batch) if rows is None else np.asarray(rows)
    pool_t = W.make_pool(w, dev)
    if on_pool is not None:
        on_pool(pool_t)
    host_pool, host_bt = W.compact_pages(w, pool_t, rows, sample_layers)
    host_pool = host_pool.reshape(-1, 2, 8, 16, 64).copy()
    pool = pkv.Pool(w.num_pages, storage=pool_t)
    pool.set_launch_flags(flags)
    bt = to_dev(w.block_tables)
    got, want = {}, {}
    for step in range(1, w.num_steps + 1):
        sl_np = w.seq_lens(step)
        sl = to_dev(sl_np)
        for layer in range(w.num_layers):
            q, k, v = W.step_inputs(w, step, layer, dev)
            if fused:   # the benchmark's call: append and decode in one launch
                out = pkv.decode_append(q, k, v, pool, bt, sl, layer, w.scale, kernel=kernel)
            else:
                pkv.append(pool, bt, sl, k, v, layer)
                out = pkv.decode(q, pool, bt, sl, layer, w.scale, kernel=kernel)
            if layer in sample_layers:
                _append_rows(host_pool, host_bt, sl_np, bits(k), bits(v), layer, rows)
                if step in sample_steps:
                    got[(step, layer)] = out[rows].cpu().numpy().astype(np.float64)
                    want[(step, layer)] = oracle.decode(bits(q), host_pool, host_bt, sl_np, layer,
                                                        w.scale, rows=rows)[rows]
    torch.cuda.synchronize()
    assert pkv.get_device_error(pool) == 0
    gpu_pages, _ = W.compact_pages(w, pool_t, rows, sample_layers)
    return got, want, gpu_pages.reshape(host_pool.shape), host_pool, pool_t


def _check(got, want, gpu_pages, host_pages):
    assert got and got.keys() == want.keys()
    for key in got:
        assert np.isfinite(got[key]).all(), key
        err = max_err(got[key], want[key])
        assert err <= ATOL, (key, err)
    assert np.array_equal(gpu_pages, host_pages)


@pytest.mark.parametrize("kernel", KERNELS)
def test_llama1b_batch16_all_layers(kernel):
    w = W.llama1b()
    got, want, gp, hp, _ = _run(w, kernel, sample_layers=list(range(16)), sample_steps=[1])
    _check(got, want, gp, hp)


def _bench_flags():
    import bench
    return bench.launch_flags(pkv)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("fused", [False, True])
def test_continuous_batching_batch64(kernel, fused):
    w = W.continuous_batching()
    got, want, gp, hp, _ = _run(w, kernel, sample_layers=[0, 15],
                                sample_steps=[1, w.num_steps], flags=_bench_flags(), fused=fused)
    _check(got, want, gp, hp)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("fused", [False, True])
def test_long_context_batch4(kernel, fused):
    w = W.long_context()
    flags = _bench_flags() if fused else 0
    got, want, gp, hp, _ = _run(w, kernel, sample_layers=[0], sample_steps=[1], flags=flags,
                                fused=fused)
    _check(got, want, gp, hp)


def _slot_checksums(pool_t, chunk=65536):
    """Position-weighted checksum of every (page, slot): int64 [pages, 16]."""
    P = pool_t.shape[0]
    wts = torch.arange(1, 2 * 8 * 64 + 1, device=pool_t.device, dtype=torch.int32)
    wts = wts.view(1, 2, 8, 1, 64)
    out = torch.empty((P, 16), dtype=torch.int64, device=pool_t.device)
    bits16 = pool_t.view(torch.int16)
    for p0 in range(0, P, chunk):
        p1 = min(P, p0 + chunk)
        v = bits16[p0:p1].to(torch.int32)
        out[p0:p1] = (v * wts).sum(dim=(1, 2, 4), dtype=torch.int64)
    return out


def test_stress_batch256_sampled():
    w = W.stress()
    rows = [0, 37, 64, 101, 128, 199, 230, 255]
    before = {}
    got, want, gp, hp, pool_t = _run(
        w, pkv.KERNEL_AUTO, sample_layers=[0, 15], sample_steps=[1, w.num_steps], rows=rows,
        on_pool=lambda p: before.setdefault("cs", _slot_checksums(p)))
    _check(got, want, gp, hp)
    # every appended slot of every sequence holds exactly the new token's bits
    dev = pool_t.device
    pos = np.arange(int(w.prefill_lens[0]), int(w.prefill_lens[0]) + w.num_steps)
    touched = torch.zeros((w.num_pages, 16), dtype=torch.bool, device=dev)
    view = pool_t.view(torch.int16).view(w.num_pages, 2, 8, 16, 64)
    for layer in range(w.num_layers):
        pages = to_dev(w.block_tables[layer][:, pos // 16].astype(np.int64))      # [B, steps]
        slots = to_dev(np.ascontiguousarray(np.broadcast_to(pos % 16, (w.batch, pos.size)))
                       .astype(np.int64))
        touched[pages, slots] = True
        for si, step in enumerate(range(1, w.num_steps + 1)):
            _, k, v = W.step_inputs(w, step, layer, dev)
            kv = view[pages[:, si], :, :, slots[:, si], :]                      # [B, 2, 8, 64]
            assert torch.equal(kv[:, 0], k.view(torch.int16))
            assert torch.equal(kv[:, 1], v.view(torch.int16))
    # nothing else in the pool changed
    after = _slot_checksums(pool_t)
    assert torch.equal(before["cs"][~touched], after[~touched])


# ---------------------------------------------------------------------------
# The benchmarked launch itself: bench.py's Runner (one CUDA graph per step of
# 16 fused append + decode calls plus their merges), with bench.py's launch
# flags (programmatic dependent launch, tables and first pages read before
# the preceding kernels end), replayed step after step as the benchmark
# replays it.  The only difference from the benchmark: before each step's
# replay the step's own inputs are copied into the graphs' input buffers
# (the benchmark reuses one set), so every step appends and attends to fresh
# tokens that the oracle also sees.

def _run_as_benchmarked(w, sample_layers, sample_steps, rows=None):
    import bench
    dev = torch.device("cuda", 0)
    rows = np.arange(w.batch) if rows is None else np.asarray(rows)
    r = bench.Runner(w, dev, pkv.KERNEL_AUTO, fused=True)
    flags = bench.launch_flags(pkv)
    assert flags == pkv.LAUNCH_PDL | pkv.LAUNCH_EARLY_TABLES | pkv.LAUNCH_EARLY_PAGES
    r.pool.set_launch_flags(flags)
    host_pool, host_bt = W.compact_pages(w, r.pool_t, rows, sample_layers)
    host_pool = host_pool.reshape(-1, 2, 8, 16, 64).copy()
    stream = torch.cuda.Stream(dev)
    r.capture(stream)
    got, want = {}, {}
    for step in range(1, w.num_steps + 1):
        sl_np = r.lens_np[step - 1]
        assert np.array_equal(sl_np, w.seq_lens(step))
        ins = [W.step_inputs(w, step, l, dev) for l in range(w.num_layers)]
        for l, (q, k, v) in enumerate(ins):
            r.q[l].copy_(q)
            r.k[l].copy_(k)
            r.v[l].copy_(v)
        r.replay(step - 1)
        for layer in sample_layers:
            q, k, v = ins[layer]
            _append_rows(host_pool, host_bt, sl_np, bits(k), bits(v), layer, rows)
            if step in sample_steps:
                got[(step, layer)] = r.out[layer][rows].cpu().numpy().astype(np.float64)
                want[(step, layer)] = oracle.decode(bits(q), host_pool, host_bt, sl_np, layer,
                                                    w.scale, rows=rows)[rows]
    torch.cuda.synchronize()
    assert pkv.get_device_error(r.pool) == 0
    gpu_pages, _ = W.compact_pages(w, r.pool_t, rows, sample_layers)
    pages = gpu_pages.reshape(host_pool.shape)
    r.close()
    return got, want, pages, host_pool


def test_continuous_batching_batch64_as_benchmarked():
    w = W.continuous_batching()
    got, want, gp, hp = _run_as_benchmarked(w, sample_layers=[0, 7, 15],
                                            sample_steps=[1, 2, 8, 15, 16])
    _check(got, want, gp, hp)


def test_llama1b_batch16_as_benchmarked():
    w = W.llama1b()
    got, want, gp, hp = _run_as_benchmarked(w, sample_layers=list(range(16)), sample_steps=[1])
    _check(got, want, gp, hp)


def test_long_context_batch4_as_benchmarked():
    w = W.long_context()
    got, want, gp, hp = _run_as_benchmarked(w, sample_layers=[0], sample_steps=[1])
    _check(got, want, gp, hp)


def test_stress_batch256_as_benchmarked_sampled():
    w = W.stress()
    rows = [0, 37, 64, 101, 128, 199, 230, 255]
    got, want, gp, hp = _run_as_benchmarked(w, sample_layers=[0, 15],
                                            sample_steps=[1, 2, 25, w.num_steps], rows=rows)
    _check(got, want, gp, hp)
