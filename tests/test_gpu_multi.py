"""GPU parity of the general decode call (pkv_decode): several queries per
sequence (causal among them) and BF16 output, against the FP64 oracle.

Query i of T attends to the tokens t < L - T + 1 + i: query T-1 sees the
whole context, each earlier query one token fewer (the plainest multi-token
decode, as when T drafted tokens are checked at once).  The BF16 output must
be the FP32 result rounded to nearest even, bit for bit, so it is checked
against the FP32 output of the same launch configuration as well as against
the oracle (within 2e-3 plus half a BF16 step).
"""
import numpy as np
import pytest
import torch

import oracle
from paged_attention_decode_pkv_b200 import pkv
from tests.cases import bf16_bits, make_case
from tests.harness import ATOL, KERNELS, GpuCase, bits, max_err, to_dev, u16_to_bf16

pytestmark = pytest.mark.gpu


def _q2(case, seed, nq=2):
    rng = np.random.default_rng(seed)
    return bf16_bits(rng.standard_normal((len(case["seq_lens"]), nq, 32, 64)))


def _run(g, q, nq, **kw):
    out = pkv.decode_general(u16_to_bf16(q), g.pool, g.bt, g.sl, kw.pop("layer", 0),
                             kw.pop("scale", 0.125), num_queries=nq, **kw)
    torch.cuda.synchronize()
    return out


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("lens", [[2], [16], [17], [18], [32], [33], [2, 17, 0, 33, 16, 1000],
                                  [300, 47, 129, 2, 517]])
def test_two_queries_match_oracle(lens):
    c = make_case(lens, seed=sum(lens) + 5, spare_pages=3)
    g = GpuCase(c)
    q = _q2(c, 1)
    got = _f64(_run(g, q, 2))
    assert pkv.get_device_error(g.pool) == 0
    want = oracle.decode_multi(q, c["pool"], c["bt"], c["seq_lens"], 0, 0.125)
    assert np.isfinite(got).all()
    assert max_err(got, want) <= ATOL
    for b, L in enumerate(lens):
        if L == 0:
            assert not got[b].any()


@pytest.mark.parametrize("grid,min_chunk", [(1, 0), (3, 1), (7, 0), (0, 1), (50, 2), (400, 1)])
def test_two_queries_split_patterns(grid, min_chunk):
    # a piece may hold only the last page, where query 0 can have no token
    c = make_case([300, 2, 47, 129, 17, 517, 33], seed=77, spare_pages=9)
    g = GpuCase(c)
    q = _q2(c, 2)
    want = oracle.decode_multi(q, c["pool"], c["bt"], c["seq_lens"], 0, 0.09)
    got = _f64(_run(g, q, 2, scale=0.09, grid_ctas=grid, min_chunk=min_chunk))
    assert max_err(got, want) <= ATOL
    assert pkv.get_device_error(g.pool) == 0


def test_two_queries_repeat_bitwise():
    c = make_case([700, 33, 2, 260, 95, 16, 17], seed=13, spare_pages=3)
    g = GpuCase(c)
    q = _q2(c, 3)
    ref = _run(g, q, 2, grid_ctas=5).cpu()
    for _ in range(20):
        assert torch.equal(_run(g, q, 2, grid_ctas=5).cpu(), ref)


def test_one_query_general_call_equals_decode():
    c = make_case([300, 1, 47, 129, 16, 517], seed=8, spare_pages=2)
    for kernel in KERNELS:
        g = GpuCase(c)
        ref = pkv.decode(g.q, g.pool, g.bt, g.sl, 0, 0.125, kernel=kernel)
        got = _run(g, c["q"], 1, kernel=kernel)
        assert torch.equal(got, ref)


@pytest.mark.parametrize("nq,kernel", [(1, pkv.KERNEL_SIMT), (1, pkv.KERNEL_MMA),
                                       (2, pkv.KERNEL_MMA)])
@pytest.mark.parametrize("grid", [0, 7])
def test_bf16_output_is_the_rounded_fp32_output(nq, kernel, grid):
    lens = [300, 2, 47, 129, 16, 517, 0]
    c = make_case(lens, seed=9, spare_pages=4)
    g = GpuCase(c)
    q = c["q"] if nq == 1 else _q2(c, 4)
    f32 = _run(g, q, nq, kernel=kernel, grid_ctas=grid)
    b16 = _run(g, q, nq, kernel=kernel, grid_ctas=grid, out_dtype=torch.bfloat16)
    assert b16.dtype == torch.bfloat16
    assert np.array_equal(bits(b16), bf16_bits(f32.cpu().numpy()))
    want = (oracle.decode(c["q"], c["pool"], c["bt"], c["seq_lens"], 0, 0.125) if nq == 1 else
            oracle.decode_multi(q, c["pool"], c["bt"], c["seq_lens"], 0, 0.125))
    got = _f64(b16)
    assert (np.abs(got - want) <= ATOL + np.abs(want) * 2.0 ** -8).all()
    assert not got[-1].any()
    assert pkv.get_device_error(g.pool) == 0


def test_fused_append_with_bf16_output():
    c = make_case([40, 1, 17, 300], seed=10, spare_pages=2)
    base = GpuCase(c)
    ref = pkv.decode_append(base.q, u16_to_bf16(c["k_new"]), u16_to_bf16(c["v_new"]), base.pool,
                            base.bt, base.sl, 0, 0.125)
    g = GpuCase(c)
    b16 = pkv.decode_general(g.q, g.pool, g.bt, g.sl, 0, 0.125, out_dtype=torch.bfloat16,
                             k_new=u16_to_bf16(c["k_new"]), v_new=u16_to_bf16(c["v_new"]))
    torch.cuda.synchronize()
    assert np.array_equal(bits(b16), bf16_bits(ref.cpu().numpy()))
    assert torch.equal(base.pool_t.view(torch.int16), g.pool_t.view(torch.int16))


def test_two_queries_reject_length_one_and_unsupported_forms():
    c = make_case([1, 20], seed=11, spare_pages=1)
    g = GpuCase(c)
    q = _q2(c, 5)
    got = _f64(_run(g, q, 2))
    assert pkv.get_device_error(g.pool) == pkv.ERR_BAD_SEQ_LEN
    assert not got[0].any()
    want = oracle.decode_multi(q[1:], c["pool"], c["bt"][:, 1:], c["seq_lens"][1:], 0, 0.125)
    assert max_err(got[1:], want) <= ATOL
    with pytest.raises(pkv.PkvError) as e:
        _run(g, q, 2, kernel=pkv.KERNEL_SIMT)
    assert e.value.status == pkv.ERR_UNSUPPORTED
    with pytest.raises(pkv.PkvError) as e:
        pkv.decode_general(u16_to_bf16(q), g.pool, g.bt, g.sl, 0, 0.125, num_queries=2,
                           k_new=u16_to_bf16(c["k_new"]), v_new=u16_to_bf16(c["v_new"]))
    assert e.value.status == pkv.ERR_UNSUPPORTED
    with pytest.raises(pkv.PkvError) as e:
        _run(g, np.zeros((2, 9, 32, 64), np.uint16), 9)
    assert e.value.status == pkv.ERR_UNSUPPORTED


@pytest.mark.parametrize("nq", [3, 4, 5, 8])
@pytest.mark.parametrize("grid", [0, 7, 300])
def test_up_to_eight_queries_match_oracle(nq, grid):
    # lengths at and around page boundaries for every query: the first query's
    # context can end one or more pages before the last one's
    lens = [nq, 16, 16 + nq - 1, 17, 33, 0, 100, 517, 2 * 16 + nq]
    c = make_case(lens, seed=nq * 10 + 1, spare_pages=4)
    g = GpuCase(c)
    q = _q2(c, nq, nq)
    got = _f64(_run(g, q, nq, grid_ctas=grid))
    assert pkv.get_device_error(g.pool) == 0
    want = oracle.decode_multi(q, c["pool"], c["bt"], c["seq_lens"], 0, 0.125)
    assert np.isfinite(got).all()
    assert max_err(got, want) <= ATOL
    assert not got[5].any()
    b16 = _run(g, q, nq, grid_ctas=grid, out_dtype=torch.bfloat16)
    assert np.array_equal(bits(b16), bf16_bits(got.astype(np.float32)))


def test_more_queries_than_context_is_reported():
    c = make_case([3, 40], seed=12, spare_pages=1)
    g = GpuCase(c)
    q = _q2(c, 6, 4)
    got = _f64(_run(g, q, 4))
    assert pkv.get_device_error(g.pool) == pkv.ERR_BAD_SEQ_LEN
    assert not got[0].any()
    want = oracle.decode_multi(q[1:], c["pool"], c["bt"][:, 1:], c["seq_lens"][1:], 0, 0.125)
    assert max_err(got[1:], want) <= ATOL


@pytest.mark.parametrize("grid,nq,bf16", [(0, 1, False), (0, 2, True), (7, 1, False),
                                          (400, 3, False), (50, 1, True)])
def test_large_batch_split_table(grid, nq, bf16):
    # Above 512 sequences the merge kernel takes each split from a table the
    # decode CTAs write (one entry per CTA) instead of rescanning the
    # lengths: long and short sequences mixed so that many are split, some
    # over many CTAs, for one and several queries and both output types.
    rng = np.random.default_rng(600 + grid + nq)
    lens = [int(x) for x in rng.integers(nq, 400, 600)]
    lens[5], lens[300], lens[599] = 3000, 0, 2500
    c = make_case(lens, seed=601, spare_pages=2)
    g = GpuCase(c)
    q = _q2(c, 3, nq)
    dt = torch.bfloat16 if bf16 else torch.float32
    kw = dict(grid_ctas=grid, out_dtype=dt)
    if nq == 1:
        got = pkv.decode_general(u16_to_bf16(q[:, 0]), g.pool, g.bt, g.sl, 0, 0.125, **kw)
        torch.cuda.synchronize()
        got = _f64(got)[:, None]
    else:
        got = _f64(_run(g, q, nq, **kw))
    assert pkv.get_device_error(g.pool) == 0
    want = oracle.decode_multi(q, c["pool"], c["bt"], c["seq_lens"], 0, 0.125)
    tol = ATOL + (2.0 ** -8 * np.abs(want).max() if bf16 else 0.0)
    assert np.isfinite(got).all()
    assert max_err(got, want) <= tol
    assert not got[300].any()


@pytest.mark.parametrize("nq", [1, 2])
def test_merge_in_many_rounds_when_decode_leaves_little_shared_memory(nq):
    # About 3,400 sequences: every decode CTA keeps the batch's lengths and
    # page-count prefix in shared memory, so the shared memory an SM has left
    # beside two decode CTAs (what the merge kernel stages its records in)
    # holds only a few records, and the two long sequences, split over ~40
    # CTAs each, are merged in many rounds with the running max rescaled
    # between them.  Checked against the oracle on every sequence.
    rng = np.random.default_rng(900 + nq)
    lens = [int(x) for x in rng.integers(nq, 40, 3400)]
    lens[7], lens[2000], lens[3399] = 30000, 24000, 0
    c = make_case(lens, seed=901, spare_pages=2)
    g = GpuCase(c)
    q = _q2(c, 5, nq)
    if nq == 1:
        got = pkv.decode_general(u16_to_bf16(q[:, 0]), g.pool, g.bt, g.sl, 0, 0.125)
        torch.cuda.synchronize()
        got = _f64(got)[:, None]
    else:
        got = _f64(_run(g, q, nq))
    assert pkv.get_device_error(g.pool) == 0
    want = oracle.decode_multi(q, c["pool"], c["bt"], c["seq_lens"], 0, 0.125)
    assert np.isfinite(got).all()
    assert max_err(got, want) <= ATOL
    assert not got[3399].any()
