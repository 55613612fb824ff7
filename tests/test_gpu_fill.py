"""GPU parity of the prefill page fill (pkv_fill) against the oracle.

Prefill writes a request's prompt tokens into its pages (comrad404 article on
samir-vllm, section on the KV cache and batched decode).  pkv_fill does that
for a ragged batch; every check here is bit for bit against oracle.fill on
the whole pool (so slots the fill must not touch are checked too), plus
fill-then-decode attention parity and the device-side error reports.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_attention_decode_pkv_b200 import pkv
from tests.cases import NAN, bf16_bits, make_case
from tests.harness import ATOL, KERNELS, GpuCase, bits, max_err, to_dev, u16_to_bf16

pytestmark = pytest.mark.gpu


def _tokens(rng, n):
    return (bf16_bits(rng.standard_normal((n, 8, 64))),
            bf16_bits(rng.standard_normal((n, 8, 64))))


def _cu(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def _fill_both(g, host, counts, starts, layer, rng):
    cu = _cu(counts)
    k, v = _tokens(rng, int(cu[-1]))
    st = np.asarray(starts, np.int32)
    pkv.fill(g.pool, g.bt, to_dev(cu), to_dev(st), u16_to_bf16(k), u16_to_bf16(v), layer)
    oracle.fill(host, g.case["bt"], cu, st, k, v, layer)


@pytest.mark.parametrize("counts,starts", [
    ([1], [0]), ([16], [0]), ([17], [0]), ([31], [1]), ([33], [15]),
    ([0, 5, 16, 1, 40], [0, 3, 16, 47, 8]),
    ([100, 0, 7, 64, 33, 2], [0, 0, 9, 0, 31, 200]),
])
def test_fill_bit_exact_whole_pool(counts, starts):
    ends = [s + n for s, n in zip(starts, counts)]
    c = make_case([max(e, 1) for e in ends], seed=sum(ends) + len(ends), spare_pages=6,
                  num_layers=2)
    g = GpuCase(c)
    host = c["pool"].copy()
    rng = np.random.default_rng(len(counts))
    for layer in (1, 0):
        _fill_both(g, host, counts, starts, layer, rng)
    torch.cuda.synchronize()
    assert pkv.get_device_error(g.pool) == 0
    assert np.array_equal(bits(g.pool_t).reshape(host.shape), host)


@pytest.mark.parametrize("batch", [510, 511, 512, 1300])
def test_fill_batches_around_the_shared_memory_index(batch):
    """Up to 511 sequences the CTA searches cu in shared memory, from 512 on
    in global memory: both bit-exact, with empty, short and page-crossing
    prompts and starts inside a page."""
    rng = np.random.default_rng(batch)
    counts = [int(x) for x in rng.choice([0, 1, 3, 16, 17, 40], batch)]
    starts = [int(x) for x in rng.integers(0, 20, batch)]
    c = make_case([s + n for s, n in zip(starts, counts)], seed=batch, spare_pages=2)
    g = GpuCase(c)
    host = c["pool"].copy()
    _fill_both(g, host, counts, starts, 0, rng)
    torch.cuda.synchronize()
    assert pkv.get_device_error(g.pool) == 0
    assert np.array_equal(bits(g.pool_t).reshape(host.shape), host)


def test_long_ragged_fill_spans_many_ctas():
    # ~8600 rows = 536 CTAs of 16 rows and a ragged last CTA; prompts cross
    # many page boundaries, and start mid page
    counts = [6000, 1, 2047, 0, 513]
    starts = [5, 0, 16, 0, 100]
    c = make_case([s + n for s, n in zip(starts, counts)], seed=3, spare_pages=3)
    g = GpuCase(c)
    host = c["pool"].copy()
    _fill_both(g, host, counts, starts, 0, np.random.default_rng(4))
    torch.cuda.synchronize()
    assert pkv.get_device_error(g.pool) == 0
    assert np.array_equal(bits(g.pool_t).reshape(host.shape), host)


def test_chunked_fill_equals_one_fill():
    counts = [300, 45, 129]
    c = make_case(counts, seed=5, spare_pages=2)
    rng = np.random.default_rng(6)
    cu = _cu(counts)
    k, v = _tokens(rng, int(cu[-1]))
    whole = GpuCase(c)
    pkv.fill(whole.pool, whole.bt, to_dev(cu), to_dev(np.zeros(3, np.int32)), u16_to_bf16(k),
             u16_to_bf16(v), 0)
    chunked = GpuCase(c)
    done = np.zeros(3, np.int32)
    for chunk in (64, 100, 1000):   # chunked prefill: each chunk continues where the last ended
        take = np.minimum(np.asarray(counts) - done, chunk).astype(np.int32)
        rows = np.concatenate([np.arange(cu[b] + done[b], cu[b] + done[b] + take[b])
                               for b in range(3)]).astype(np.int64)
        pkv.fill(chunked.pool, chunked.bt, to_dev(_cu(take)), to_dev(done),
                 u16_to_bf16(k[rows]), u16_to_bf16(v[rows]), 0)
        done += take
    torch.cuda.synchronize()
    assert pkv.get_device_error(chunked.pool) == 0
    assert torch.equal(whole.pool_t.view(torch.int16), chunked.pool_t.view(torch.int16))


@pytest.mark.parametrize("kernel", KERNELS)
def test_fill_then_decode_matches_oracle(kernel):
    # prompts filled into NaN pages, then decode over exactly those tokens
    lens = [700, 1, 16, 17, 260]
    c = make_case(lens, seed=8, spare_pages=4)
    c = dict(c, pool=np.full_like(c["pool"], NAN))
    g = GpuCase(c)
    host = c["pool"].copy()
    _fill_both(g, host, lens, [0] * len(lens), 0, np.random.default_rng(9))
    torch.cuda.synchronize()
    assert pkv.get_device_error(g.pool) == 0
    got = g.decode(kernel=kernel)
    want = oracle.decode(c["q"], host, c["bt"], c["seq_lens"], 0, 0.125)
    assert np.isfinite(got).all()
    assert max_err(got, want) <= ATOL


def test_fill_errors_are_reported_and_other_sequences_written():
    counts = [20, 20, 20]
    c = make_case(counts, seed=10, spare_pages=2)
    rng = np.random.default_rng(11)
    cu = _cu(counts)
    k, v = _tokens(rng, int(cu[-1]))
    host = c["pool"].copy()
    oracle.fill(host, c["bt"][:, 1:2], cu[1:3] - cu[1], np.zeros(1, np.int32),
                k[cu[1]:cu[2]], v[cu[1]:cu[2]], 0)

    # sequence 0: start beyond its table; sequence 2: a page outside the pool
    bt = c["bt"].copy()
    bt[0, 2, 1] = 1 << 20
    g = GpuCase(dict(c, bt=bt))
    pkv.fill(g.pool, g.bt, to_dev(cu), to_dev(np.array([40, 0, 0], np.int32)), u16_to_bf16(k),
             u16_to_bf16(v), 0)
    err = pkv.get_device_error(g.pool)
    assert err in (pkv.ERR_BAD_SEQ_LEN, pkv.ERR_BAD_PAGE)
    out = bits(g.pool_t).reshape(host.shape)
    # sequence 1 written exactly; sequence 0 untouched; sequence 2's first page written
    p1 = c["bt"][0, 1, :2]
    assert np.array_equal(out[p1], host[p1])
    p0 = c["bt"][0, 0, :2]
    assert np.array_equal(out[p0], c["pool"][p0])
    first2 = c["bt"][0, 2, 0]
    assert np.array_equal(out[first2, 0, :, :16], k[cu[2]:cu[2] + 16].transpose(1, 0, 2))

    # cu_tokens not starting at 0, or not ending at the row count: nothing
    # written; a decreasing cu: reported
    g = GpuCase(c)
    for bad in (cu + 1, np.array([0, 20, 40, 59], np.int32)):
        pkv.fill(g.pool, g.bt, to_dev(bad), to_dev(np.zeros(3, np.int32)), u16_to_bf16(k),
                 u16_to_bf16(v), 0)
        assert pkv.get_device_error(g.pool) == pkv.ERR_BAD_SEQ_LEN
        assert np.array_equal(bits(g.pool_t).reshape(host.shape), c["pool"])
    bad_cu = np.array([0, 30, 10, 40], np.int32)
    pkv.fill(g.pool, g.bt, to_dev(bad_cu), to_dev(np.zeros(3, np.int32)), u16_to_bf16(k[:40]),
             u16_to_bf16(v[:40]), 0)
    assert pkv.get_device_error(g.pool) == pkv.ERR_BAD_SEQ_LEN
    assert pkv.get_device_error(g.pool) == 0


def test_empty_fill_launches_nothing():
    c = make_case([5, 0], seed=12, spare_pages=1)
    g = GpuCase(c)
    empty = torch.empty((0, 8, 64), dtype=torch.bfloat16, device="cuda")
    pkv.fill(g.pool, g.bt, to_dev(np.zeros(3, np.int32)), to_dev(np.zeros(2, np.int32)), empty,
             empty, 0)
    assert pkv.get_device_error(g.pool) == 0
    assert np.array_equal(bits(g.pool_t).reshape(c["pool"].shape), c["pool"])
