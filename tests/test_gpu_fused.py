"""GPU parity of the fused append + decode (paged_attention_decode_append).

Decode adds the new token to the cache and attends to it (comrad404 article
on samir-vllm, section on the KV cache and batched decode).  The fused call
must equal pkv_append followed by paged_attention_decode: the pool bit for
bit against oracle.append (the new token lands in slot (L-1) % 16 of the
last page, nothing else changes), the output within 2e-3 of oracle.decode
on the appended pool, and -- since it is the same arithmetic on the same
bits -- bitwise equal to the two separate calls.  The appended slot starts
out as NaN, so a missed or misplaced append shows up in the output too.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_attention_decode_pkv_b200 import pkv
from tests.cases import NAN, make_case
from tests.harness import ATOL, KERNELS, GpuCase, bits, max_err, to_dev, u16_to_bf16

pytestmark = pytest.mark.gpu


def _blank_new_slots(c):
    """The case with the new token's slot NaN in the pool (every layer)."""
    pool = c["pool"].copy()
    for layer in range(c["bt"].shape[0]):
        for b, L in enumerate(c["seq_lens"]):
            if L > 0:
                t = int(L) - 1
                pool[c["bt"][layer, b, t // 16], :, :, t % 16, :] = NAN
    return dict(c, pool=pool)


def _host_after_append(c, layer):
    host = c["pool"].copy()
    rows = np.nonzero(c["seq_lens"] > 0)[0]
    oracle.append(host, c["bt"][:, rows, :], c["seq_lens"][rows], c["k_new"][rows],
                  c["v_new"][rows], layer)
    return host


def _fused(g, layer=0, scale=0.125, **kw):
    c = g.case
    out = pkv.decode_append(g.q, u16_to_bf16(c["k_new"]), u16_to_bf16(c["v_new"]), g.pool, g.bt,
                            g.sl, layer, scale, **kw)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("lens", [[1], [15], [16], [17], [32], [33], [1, 15, 16, 17, 31, 0, 64],
                                  [200, 3, 77, 1000, 16]])
def test_fused_equals_oracle_append_then_decode(kernel, lens):
    c = _blank_new_slots(make_case(lens, seed=sum(lens) + 7, spare_pages=4))
    g = GpuCase(c)
    got = _fused(g, kernel=kernel)
    assert pkv.get_device_error(g.pool) == 0
    host = _host_after_append(c, 0)
    assert np.array_equal(bits(g.pool_t).reshape(host.shape), host)   # whole pool
    want = oracle.decode(c["q"], host, c["bt"], c["seq_lens"], 0, 0.125)
    assert np.isfinite(got).all()
    assert max_err(got, want) <= ATOL
    for b, L in enumerate(lens):
        if L == 0:
            assert not got[b].any()


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("grid,min_chunk", [(1, 0), (3, 1), (7, 0), (0, 1), (50, 2), (400, 1)])
def test_fused_split_patterns_bitwise_equal_to_two_calls(kernel, grid, min_chunk):
    # the appending CTA holds the last piece of a split sequence
    base = _blank_new_slots(make_case([300, 1, 47, 129, 16, 517], seed=77, spare_pages=9,
                                      num_layers=2))
    for layer in (1, 0):
        fused = GpuCase(base)
        got = _fused(fused, layer=layer, scale=0.09, kernel=kernel, grid_ctas=grid,
                     min_chunk=min_chunk)
        two = GpuCase(base)
        pkv.append(two.pool, two.bt, two.sl, u16_to_bf16(base["k_new"]),
                   u16_to_bf16(base["v_new"]), layer)
        ref = two.decode(layer=layer, scale=0.09, kernel=kernel, grid_ctas=grid,
                         min_chunk=min_chunk)
        assert np.array_equal(got, ref)
        assert torch.equal(fused.pool_t.view(torch.int16), two.pool_t.view(torch.int16))
        host = _host_after_append(base, layer)
        want = oracle.decode(base["q"], host, base["bt"], base["seq_lens"], layer, 0.09)
        assert max_err(got, want) <= ATOL
        assert pkv.get_device_error(fused.pool) == 0


EARLY_ALL = pkv.LAUNCH_PDL | pkv.LAUNCH_EARLY_TABLES | pkv.LAUNCH_EARLY_PAGES


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("flags", [pkv.LAUNCH_PDL | pkv.LAUNCH_EARLY_TABLES, EARLY_ALL])
@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("lens0,grid", [([40, 1, 77, 15, 300], 0),
                                        ([40, 1, 77, 15, 300], 3),
                                        (list(range(1, 33)) + [200, 31, 17], 0)])
def test_repeated_steps_on_one_layer_with_pdl(kernel, flags, fused, lens0, grid):
    # Steps of a one-layer model: lengths grow by one, each step appends the
    # new token (fused, or pkv_append then decode) and attends to it.  With
    # programmatic launch a step's decode may start while the previous
    # step's kernels still run -- and with early pages load pages before
    # they end -- so the pages the previous steps append into must not be
    # loaded early.  Every step is checked against the oracle, and the pool
    # bit for bit at the end.  Lengths cross page boundaries during the 20
    # steps, and the many short sequences put CTA ranges' first pages on
    # sequences' last pages.
    lens0 = np.array(lens0, np.int32)
    steps = 20
    B = lens0.size
    c = make_case(list(lens0 + steps), seed=31 + B, spare_pages=3)
    g = GpuCase(c)
    g.pool.set_launch_flags(flags)
    host = c["pool"].copy()
    rng = np.random.default_rng(5)
    from tests.cases import bf16_bits
    outs, wants = [], []
    for s in range(1, steps + 1):
        sl = lens0 + s
        k = bf16_bits(rng.standard_normal((B, 8, 64)))
        v = bf16_bits(rng.standard_normal((B, 8, 64)))
        sl_d = to_dev(sl)
        if fused:
            out = pkv.decode_append(g.q, u16_to_bf16(k), u16_to_bf16(v), g.pool, g.bt, sl_d, 0,
                                    0.125, kernel=kernel, grid_ctas=grid)
        else:
            pkv.append(g.pool, g.bt, sl_d, u16_to_bf16(k), u16_to_bf16(v), 0)
            out = pkv.decode(g.q, g.pool, g.bt, sl_d, 0, 0.125, kernel=kernel, grid_ctas=grid)
        oracle.append(host, c["bt"], sl, k, v, 0)
        outs.append(out)
        wants.append(oracle.decode(c["q"], host, c["bt"], sl, 0, 0.125))
    torch.cuda.synchronize()
    assert pkv.get_device_error(g.pool) == 0
    assert np.array_equal(bits(g.pool_t).reshape(host.shape), host)
    for s, (out, want) in enumerate(zip(outs, wants), 1):
        assert max_err(out.cpu().numpy().astype(np.float64), want) <= ATOL, s


def test_fused_bad_last_page_is_reported_and_not_written():
    c = _blank_new_slots(make_case([40, 20], seed=17, spare_pages=2))
    bad = c["bt"].copy()
    bad[0, 0, 2] = 1 << 20          # sequence 0's last page: outside the pool
    g = GpuCase(dict(c, bt=bad))
    got = _fused(g)
    assert pkv.get_device_error(g.pool) == pkv.ERR_BAD_PAGE
    host = c["pool"].copy()
    oracle.append(host, c["bt"][:, 1:], c["seq_lens"][1:], c["k_new"][1:], c["v_new"][1:], 0)
    assert np.array_equal(bits(g.pool_t).reshape(host.shape), host)   # only sequence 1 appended
    want = oracle.decode(c["q"], host, c["bt"], c["seq_lens"], 0, 0.125)
    assert max_err(got[1], want[1]) <= ATOL


@pytest.mark.parametrize("kernel", KERNELS)
def test_fused_timeout_reports_and_context_survives(kernel):
    c = _blank_new_slots(make_case([40, 300, 17], seed=37, spare_pages=2))
    g = GpuCase(c)
    g.pool.set_launch_flags(pkv.LAUNCH_TEST_STALL)
    _fused(g, kernel=kernel)
    assert pkv.get_device_error(g.pool) == pkv.ERR_DEVICE_TIMEOUT
    g.pool.set_launch_flags(0)
    got = _fused(g, kernel=kernel)
    assert pkv.get_device_error(g.pool) == 0
    host = _host_after_append(c, 0)
    assert max_err(got, oracle.decode(c["q"], host, c["bt"], c["seq_lens"], 0, 0.125)) <= ATOL


def test_fused_rejects_missing_new_rows():
    g = GpuCase(make_case([40, 20], seed=3))
    ws = g.pool.workspace(2)
    P = torch.zeros(1, dtype=torch.int8, device="cuda")
    st = pkv.lib.paged_attention_decode_append(
        g.q.data_ptr(), None, None, g.pool.handle, g.bt.data_ptr(), g.sl.data_ptr(), 0, 0.125,
        P.data_ptr(), 1, 2, g.bt.shape[2], ws.data_ptr(), ws.numel(), None)
    assert st == pkv.ERR_INVALID_ARG


def test_large_batch_fused_chain_with_early_pages():
    # Above 512 sequences decode writes the merge's split table right after
    # its dependency wait, while the previous step's merge (which reads the
    # table) may still be running beside the early part of this decode: a
    # chain of fused steps with programmatic launch and early pages, every
    # step checked against the oracle.
    rng = np.random.default_rng(640)
    lens0 = rng.integers(1, 300, 640).astype(np.int32)
    lens0[[3, 333, 639]] = [2500, 1800, 3000]
    steps = 4
    c = make_case(list(lens0 + steps), seed=641, spare_pages=2)
    g = GpuCase(c)
    g.pool.set_launch_flags(EARLY_ALL)
    host = c["pool"].copy()
    from tests.cases import bf16_bits
    outs, wants = [], []
    for s in range(1, steps + 1):
        sl = lens0 + s
        k = bf16_bits(rng.standard_normal((640, 8, 64)))
        v = bf16_bits(rng.standard_normal((640, 8, 64)))
        outs.append(pkv.decode_append(g.q, u16_to_bf16(k), u16_to_bf16(v), g.pool, g.bt,
                                      to_dev(sl), 0, 0.125))
        oracle.append(host, c["bt"], sl, k, v, 0)
        wants.append(oracle.decode(c["q"], host, c["bt"], sl, 0, 0.125))
    torch.cuda.synchronize()
    assert pkv.get_device_error(g.pool) == 0
    assert np.array_equal(bits(g.pool_t).reshape(host.shape), host)
    for s, (out, want) in enumerate(zip(outs, wants), 1):
        assert max_err(out.cpu().numpy().astype(np.float64), want) <= ATOL, s
