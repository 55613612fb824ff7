"""GPU parity on small cases: CUDA path (through the C ABI) vs the FP64
oracle, on the same BF16 input bits.  Covers ragged lengths around page
boundaries, empty sequences, forced split-KV patterns, NaN in every slot
outside the context, bit-exact append and gather, device-side error reports
and launch-to-launch determinism."""
import numpy as np
import pytest
import torch

import oracle
from paged_attention_decode_pkv_b200 import pkv
from paged_attention_decode_pkv_b200 import workloads as W
from tests.cases import NAN, bf16_bits, make_case, shared_prefix_case
from tests.harness import ATOL, KERNELS, GpuCase, bits, max_err, to_dev, u16_to_bf16

pytestmark = pytest.mark.gpu

EDGE_LENS = [[1], [15], [16], [17], [31], [32], [33], [0, 5], [1, 15, 16, 17, 31, 32, 33, 0, 64],
             [200, 3, 77, 1000, 16]]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("lens", EDGE_LENS)
def test_decode_edge_lengths(kernel, lens):
    g = GpuCase(make_case(lens, seed=len(lens) * 100 + sum(lens), spare_pages=5))
    got = g.decode(kernel=kernel)
    want = g.oracle()
    assert np.isfinite(got).all()
    assert max_err(got, want) <= ATOL
    for b, L in enumerate(lens):
        if L == 0:
            assert not got[b].any()


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("grid,min_chunk", [(1, 0), (2, 0), (7, 0), (3, 1), (0, 1), (0, 3),
                                            (0, 64), (50, 2), (100, 1), (77, 0), (400, 1),
                                            (600, 0)])
def test_decode_split_patterns(kernel, grid, min_chunk):
    # Different grids / chunk sizes cut the sequences' page runs at
    # different places, exercising the split-KV merge; the result must stay
    # within tolerance of the oracle for every cut, including grids (400,
    # 600 CTAs) larger than the device holds at once.
    g = GpuCase(make_case([300, 1, 47, 129, 16, 517], seed=77, spare_pages=9))
    want = g.oracle(scale=0.09)
    got = g.decode(scale=0.09, kernel=kernel, grid_ctas=grid, min_chunk=min_chunk)
    assert max_err(got, want) <= ATOL


@pytest.mark.parametrize("kernel", KERNELS)
def test_tiny_workload_append_and_decode(kernel):
    w = W.tiny()
    dev = "cuda"
    pool_t = W.make_pool(w, dev)
    host_pool = bits(pool_t).reshape(w.num_pages, 2, 8, 16, 64).copy()
    pool = pkv.Pool(w.num_pages, storage=pool_t)
    bt = to_dev(w.block_tables)
    sl_np = w.seq_lens(1)
    sl = to_dev(sl_np)
    q, k, v = W.step_inputs(w, 1, 0, dev)
    pkv.append(pool, bt, sl, k, v, 0)
    out = pkv.decode(q, pool, bt, sl, 0, w.scale, kernel=kernel)
    torch.cuda.synchronize()
    assert pkv.get_device_error(pool) == 0
    oracle.append(host_pool, w.block_tables, sl_np, bits(k), bits(v), 0)
    assert np.array_equal(bits(pool_t).reshape(host_pool.shape), host_pool)   # whole pool
    want = oracle.decode(bits(q), host_pool, w.block_tables, sl_np, 0, w.scale)
    assert max_err(out.cpu().numpy().astype(np.float64), want) <= ATOL


def test_append_bit_exact_and_touches_nothing_else():
    c = make_case([17, 40, 1, 16, 33], seed=5, spare_pages=7, num_layers=2)
    g = GpuCase(c)
    rng = np.random.default_rng(0)
    k = bf16_bits(rng.standard_normal((5, 8, 64)))
    v = bf16_bits(rng.standard_normal((5, 8, 64)))
    host = c["pool"].copy()
    for layer in (1, 0):
        pkv.append(g.pool, g.bt, g.sl, u16_to_bf16(k), u16_to_bf16(v), layer)
        oracle.append(host, c["bt"], c["seq_lens"], k, v, layer)
    torch.cuda.synchronize()
    assert pkv.get_device_error(g.pool) == 0
    assert np.array_equal(bits(g.pool_t).reshape(host.shape), host)


def test_gather_bit_exact_and_leaves_tail():
    c = make_case([17, 40, 0, 33, 1], seed=9, spare_pages=4, num_layers=3)
    g = GpuCase(c)
    for layer in range(3):
        k0 = np.full((5, 8, 48, 64), 0x1234, np.uint16)
        v0 = np.full((5, 8, 48, 64), 0x4321, np.uint16)
        kd, vd = u16_to_bf16(k0), u16_to_bf16(v0)
        pkv.gather(g.pool, g.bt, g.sl, layer, 48, kd, vd)
        ko, vo = oracle.gather(c["pool"], c["bt"], c["seq_lens"], layer, 48, k0.copy(), v0.copy())
        assert np.array_equal(bits(kd).reshape(ko.shape), ko)
        assert np.array_equal(bits(vd).reshape(vo.shape), vo)
    assert pkv.get_device_error(g.pool) == 0


@pytest.mark.parametrize("kernel", KERNELS)
def test_nan_outside_context_never_reaches_output(kernel):
    c = make_case([1, 15, 17, 31, 49], seed=11, spare_pages=8)
    assert (c["pool"] == NAN).sum() > 0
    g = GpuCase(c)
    got = g.decode(kernel=kernel)
    assert np.isfinite(got).all()
    assert max_err(got, g.oracle()) <= ATOL


@pytest.mark.parametrize("kernel", KERNELS)
def test_repeated_launches_are_bitwise_identical(kernel):
    g = GpuCase(make_case([700, 33, 1, 260, 95, 16, 17], seed=13, spare_pages=3))
    ref = g.decode(kernel=kernel, grid_ctas=5)
    for _ in range(100):
        assert np.array_equal(g.decode(kernel=kernel, grid_ctas=5), ref)


@pytest.mark.parametrize("kernel", KERNELS)
def test_bad_page_is_reported_not_faulted(kernel):
    c = make_case([40, 20], seed=17, spare_pages=2)
    bad = c["bt"].copy()
    bad[0, 0, 1] = 1 << 20          # far outside the pool
    g = GpuCase(dict(c, bt=bad))
    got = g.decode(kernel=kernel)
    assert pkv.get_device_error(g.pool) == pkv.ERR_BAD_PAGE
    # the other sequence is unaffected
    want = oracle.decode(c["q"], c["pool"], c["bt"], c["seq_lens"], 0, 0.125)
    assert max_err(got[1], want[1]) <= ATOL
    pkv.append(g.pool, g.bt, g.sl, u16_to_bf16(c["k_new"]), u16_to_bf16(c["v_new"]), 0)
    assert pkv.get_device_error(g.pool) in (pkv.ERR_BAD_PAGE, 0)
    assert pkv.get_device_error(g.pool) == 0       # cleared by the previous read


@pytest.mark.parametrize("kernel", KERNELS)
def test_bad_seq_len_is_reported_and_row_zeroed(kernel):
    c = make_case([40, 20], seed=19, spare_pages=2)
    g = GpuCase(c)
    g.sl = to_dev(np.array([40, 10_000], np.int32))
    got = g.decode(kernel=kernel)
    assert pkv.get_device_error(g.pool) == pkv.ERR_BAD_SEQ_LEN
    assert not got[1].any()
    assert max_err(got[0], g.oracle()[0]) <= ATOL
    g.sl = to_dev(np.array([0, 20], np.int32))
    pkv.append(g.pool, g.bt, g.sl, u16_to_bf16(c["k_new"]), u16_to_bf16(c["v_new"]), 0)
    assert pkv.get_device_error(g.pool) == pkv.ERR_BAD_SEQ_LEN


def test_workspace_too_small_is_rejected():
    g = GpuCase(make_case([40, 20], seed=23))
    need = g.pool.workspace_bytes(2)
    ws = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(pkv.PkvError) as e:
        pkv.decode(g.q, g.pool, g.bt, g.sl, 0, 0.125, workspace=ws)
    assert e.value.status == pkv.ERR_WORKSPACE


def test_scale_and_layer_arguments():
    c = make_case([33, 70], seed=29, num_layers=3, spare_pages=2)
    g = GpuCase(c)
    for layer in range(3):
        for scale in (0.0, 0.125, 0.5):
            got = g.decode(layer=layer, scale=scale)
            assert max_err(got, g.oracle(layer=layer, scale=scale)) <= ATOL


@pytest.mark.parametrize("kernel", KERNELS)
def test_programmatic_dependent_launch_keeps_results(kernel):
    # With PDL each kernel waits for its predecessor before touching memory,
    # so an append followed by decodes must give the same answer.
    c = make_case([40, 1, 77, 16], seed=31, spare_pages=3)
    g = GpuCase(c)
    g.pool.set_launch_flags(pkv.LAUNCH_PDL)
    pkv.append(g.pool, g.bt, g.sl, u16_to_bf16(c["k_new"]), u16_to_bf16(c["v_new"]), 0)
    first = g.decode(kernel=kernel)
    for _ in range(5):
        pkv.append(g.pool, g.bt, g.sl, u16_to_bf16(c["k_new"]), u16_to_bf16(c["v_new"]), 0)
        assert np.array_equal(g.decode(kernel=kernel), first)
    assert max_err(first, g.oracle()) <= ATOL
    assert pkv.get_device_error(g.pool) == 0
    with pytest.raises(pkv.PkvError):
        g.pool.set_launch_flags(pkv.LAUNCH_EARLY_TABLES)   # needs PDL
    with pytest.raises(pkv.PkvError):
        g.pool.set_launch_flags(pkv.LAUNCH_PDL | pkv.LAUNCH_EARLY_PAGES)   # needs early tables
    with pytest.raises(pkv.PkvError):
        g.pool.set_launch_flags(16)   # no such flag
    g.pool.set_launch_flags(pkv.LAUNCH_PDL | pkv.LAUNCH_EARLY_TABLES)
    for _ in range(3):
        pkv.append(g.pool, g.bt, g.sl, u16_to_bf16(c["k_new"]), u16_to_bf16(c["v_new"]), 0)
        assert np.array_equal(g.decode(kernel=kernel), first)


@pytest.mark.parametrize("kernel", KERNELS)
def test_bounded_wait_reports_timeout_and_context_survives(kernel):
    # A stage that nothing fills: every wait on it gives up after ~1 s, the
    # kernel reports PKV_ERR_DEVICE_TIMEOUT, and the next launch works.
    c = make_case([40, 300, 17], seed=37, spare_pages=2)
    g = GpuCase(c)
    g.pool.set_launch_flags(pkv.LAUNCH_TEST_STALL)
    g.decode(kernel=kernel)
    assert pkv.get_device_error(g.pool) == pkv.ERR_DEVICE_TIMEOUT
    g.pool.set_launch_flags(0)
    got = g.decode(kernel=kernel)
    assert pkv.get_device_error(g.pool) == 0
    assert max_err(got, g.oracle()) <= ATOL


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("grid,min_chunk", [(0, 0), (7, 0), (0, 3), (400, 0), (600, 1)])
def test_stale_workspace_contents_do_not_matter(kernel, grid, min_chunk):
    # The merge may only read partial records that this launch wrote: a
    # workspace full of earlier records (here: NaN bytes, and then the
    # records of a different batch) must give the same result.
    c = make_case([300, 1, 47, 129, 16, 517, 2], seed=41, spare_pages=5)
    g = GpuCase(c)
    want = g.oracle(scale=0.11)
    ws = g.pool.workspace(7, kernel, grid)
    ws.fill_(0xFF)                       # every float of it is NaN
    got = g.decode(scale=0.11, kernel=kernel, grid_ctas=grid, min_chunk=min_chunk, workspace=ws)
    assert np.isfinite(got).all()
    assert max_err(got, want) <= ATOL
    other = GpuCase(make_case([900, 33, 400, 5, 260, 1, 1200], seed=42, spare_pages=2))
    other.decode(kernel=kernel, grid_ctas=grid, min_chunk=min_chunk, workspace=ws)
    again = g.decode(scale=0.11, kernel=kernel, grid_ctas=grid, min_chunk=min_chunk, workspace=ws)
    assert np.array_equal(again, got)


@pytest.mark.parametrize("batch", [3000, 5000])
def test_large_batches(batch):
    # 5,000 sequences no longer fit two tensor-core CTAs per SM (8 bytes of
    # shared memory per sequence per CTA): the grid shrinks to one per SM
    rng = np.random.default_rng(batch)
    lens = [int(x) for x in rng.integers(0, 40, batch)]
    c = make_case(lens, seed=batch, spare_pages=3)
    g = GpuCase(c)
    for kernel in (pkv.KERNEL_MMA, pkv.KERNEL_SIMT):
        got = g.decode(kernel=kernel)
        assert pkv.get_device_error(g.pool) == 0
        assert max_err(got, g.oracle()) <= ATOL


def test_batch_beyond_shared_memory_is_unsupported():
    g = GpuCase(make_case([16, 16], seed=3))
    with pytest.raises(pkv.PkvError) as e:
        g.pool.workspace_bytes(20000)
    assert e.value.status == pkv.ERR_UNSUPPORTED


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("fused", [False, True])
def test_shared_prefix_pages_are_read_in_place(kernel, fused):
    # several sequences read the same physical pages (a reused prefix,
    # read-only): the result equals the oracle and, bit for bit, the same
    # batch with the prefix in private pages; the fused call appends into
    # each sequence's own last page only
    shared, private = shared_prefix_case()
    outs = []
    for c in (shared, private):
        g = GpuCase(c)
        if fused:
            got = pkv.decode_append(g.q, u16_to_bf16(c["k_new"]), u16_to_bf16(c["v_new"]), g.pool,
                                    g.bt, g.sl, 0, 0.125, kernel=kernel)
            torch.cuda.synchronize()
            got = got.cpu().numpy().astype(np.float64)
        else:
            got = g.decode(kernel=kernel)
        assert pkv.get_device_error(g.pool) == 0
        assert max_err(got, g.oracle()) <= ATOL
        if fused:   # only the appended slots were written, with the bits they held
            assert np.array_equal(bits(g.pool_t).reshape(c["pool"].shape), c["pool"])
        outs.append(got)
    assert np.array_equal(outs[0], outs[1])
