"""GPU parity of the opt-in race check (PKV_LAUNCH_CHECK_APPENDS).

Two sequences appending to one slot race, and the fused append + decode
also races when a sequence appends into a slot that a context of the same
call reads.  With the flag set, pkv_append and the fused call must report
PKV_ERR_APPEND_CONFLICT exactly when oracle.append_conflict finds such a
race -- on the hand-worked cases and on seeded random tables drawn from a
few pages, so that races are common -- and otherwise only the append's own
errors (bad length, page outside the pool).  On full-size workloads, whose
appends never race, the flag must change nothing: no error, and the output
and the pool bitwise equal to a run without it.  A racing call writes
nothing outside the pool and waits on nothing, so these cases only give
undefined values, which the tests do not read.  pkv_fill's check (two
tokens written to one slot) is held to oracle.fill_conflict the same way.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_attention_decode_pkv_b200 import pkv
from paged_attention_decode_pkv_b200 import workloads as W
from tests.cases import APPEND_CASE_PAGES, APPEND_CONFLICT_CASES, FILL_CONFLICT_CASES
from tests.harness import to_dev

pytestmark = pytest.mark.gpu


def _status(bt, lens, num_pages, fused, seed):
    gen = torch.Generator(device="cuda").manual_seed(seed)
    B = bt.shape[1]

    def randn(*shape):
        return torch.randn(shape, generator=gen, device="cuda").to(torch.bfloat16)

    pool_t = randn(num_pages, 2, 8, 16, 64)
    pool = pkv.Pool(num_pages, storage=pool_t)
    pool.set_launch_flags(pkv.LAUNCH_CHECK_APPENDS)
    k, v = randn(B, 8, 64), randn(B, 8, 64)
    bt_d, sl_d = to_dev(bt), to_dev(lens)
    if fused:
        pkv.decode_append(randn(B, 32, 64), k, v, pool, bt_d, sl_d, 0, 0.125)
    else:
        pkv.append(pool, bt_d, sl_d, k, v, 0)
    torch.cuda.synchronize()
    status = pkv.get_device_error(pool)
    pool.close()
    return status


def _allowed(bt, lens, num_pages, fused):
    """Statuses a call may report: the race, else its own errors (any of them)."""
    if oracle.append_conflict(bt, lens, 0, num_pages, fused):
        return {pkv.ERR_APPEND_CONFLICT}
    rows, mb = bt[0], bt.shape[2]
    errs = set()
    for b, L in enumerate(int(x) for x in lens):
        if L < (0 if fused else 1) or L > 16 * mb:
            errs.add(pkv.ERR_BAD_SEQ_LEN)
            continue
        used = range((L + 15) // 16) if fused else ([(L - 1) // 16] if L > 0 else [])
        if any(not 0 <= rows[b, j] < num_pages for j in used):
            errs.add(pkv.ERR_BAD_PAGE)
    return errs or {0}


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("case", APPEND_CONFLICT_CASES, ids=[c[0] for c in APPEND_CONFLICT_CASES])
def test_hand_worked_cases(case, fused):
    _, rows, lens, plain_race, fused_race = case
    bt = np.array([rows], np.int32)
    sl = np.array(lens, np.int32)
    got = _status(bt, sl, APPEND_CASE_PAGES, fused, seed=len(rows))
    assert (got == pkv.ERR_APPEND_CONFLICT) == (fused_race if fused else plain_race)
    assert got in _allowed(bt, sl, APPEND_CASE_PAGES, fused)


@pytest.mark.parametrize("fused", [False, True])
def test_random_tables_match_oracle(fused):
    rng = np.random.default_rng(77 + fused)
    races = 0
    for i in range(150):
        batch = int(rng.integers(1, 9))
        mb = int(rng.integers(1, 5))
        pages = int(rng.integers(1, 7))
        bt = rng.integers(-1, pages + 1, size=(1, batch, mb)).astype(np.int32)
        lens = rng.integers(0, 16 * mb + 1, size=batch).astype(np.int32)
        if rng.random() < 0.5:
            lens = np.minimum(lens, rng.integers(0, 20, size=batch)).astype(np.int32)
        if not fused:   # plain appends race only on a shared slot: favour short contexts
            lens = np.maximum(lens if rng.random() < 0.3 else lens % 3, 1).astype(np.int32)
        want = _allowed(bt, lens, pages, fused)
        got = _status(bt, lens, pages, fused, seed=i)
        assert got in want, (i, bt, lens, pages, got, want)
        races += want == {pkv.ERR_APPEND_CONFLICT}
    assert 20 < races < 130


def test_large_batch_spans_several_staging_chunks():
    """Batch 5000 with the only race between sequences 1 and 4999 (the check
    stages appended slots 2048 at a time)."""
    B = 5000
    bt = np.arange(B, dtype=np.int32).reshape(1, B, 1)
    bt[0, 4999, 0] = 1
    lens = np.full(B, 3, np.int32)
    for fused in (False, True):
        assert oracle.append_conflict(bt, lens, 0, B, fused)
        assert _status(bt, lens, B, fused, seed=5) == pkv.ERR_APPEND_CONFLICT
        lens2 = lens.copy()
        lens2[4999] = 4   # (1, 3) and (1, 2): only the fused call reads the other's slot
        assert oracle.append_conflict(bt, lens2, 0, B, fused) == fused
        assert _status(bt, lens2, B, fused, seed=6) == (pkv.ERR_APPEND_CONFLICT if fused else 0)


@pytest.mark.parametrize("make", [W.llama1b, W.continuous_batching], ids=["llama1b_b16",
                                                                          "continuous_batching_b64"])
def test_flag_changes_nothing_on_workloads(make):
    w = make()
    dev = torch.device("cuda")
    bt = torch.from_numpy(w.block_tables).to(dev)
    sl_np = w.seq_lens(1)
    sl = torch.from_numpy(sl_np).to(dev)
    outs, pools = [], []
    for flags in (pkv.LAUNCH_PDL, pkv.LAUNCH_PDL | pkv.LAUNCH_CHECK_APPENDS):
        pool_t = W.make_pool(w, dev)
        pool = pkv.Pool(w.num_pages, storage=pool_t)
        pool.set_launch_flags(flags)
        for layer in (0, w.block_tables.shape[0] - 1):
            assert not oracle.append_conflict(w.block_tables, sl_np, layer, w.num_pages, True)
            q, k, v = W.step_inputs(w, 1, layer, dev)
            outs.append(pkv.decode_append(q, k, v, pool, bt, sl, layer, w.scale).clone())
            pkv.append(pool, bt, sl, k, v, layer)   # the same token again: no race either
        torch.cuda.synchronize()
        assert pkv.get_device_error(pool) == 0
        pools.append(pool_t)
        pool.close()
    half = len(outs) // 2
    for a, b in zip(outs[:half], outs[half:]):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    assert torch.equal(pools[0].view(torch.int16), pools[1].view(torch.int16))


def _cu(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def _fill_status(bt, counts, starts, num_pages, seed):
    gen = torch.Generator(device="cuda").manual_seed(seed)
    cu = _cu(counts)
    T = int(cu[-1])
    pool_t = torch.randn((num_pages, 2, 8, 16, 64), generator=gen,
                         device="cuda").to(torch.bfloat16)
    pool = pkv.Pool(num_pages, storage=pool_t)
    pool.set_launch_flags(pkv.LAUNCH_CHECK_APPENDS)
    k = torch.randn((T, 8, 64), generator=gen, device="cuda").to(torch.bfloat16)
    v = torch.randn((T, 8, 64), generator=gen, device="cuda").to(torch.bfloat16)
    pkv.fill(pool, to_dev(bt), to_dev(cu), to_dev(np.asarray(starts, np.int32)), k, v, 0)
    torch.cuda.synchronize()
    status = pkv.get_device_error(pool)
    pool.close()
    return status


def _fill_allowed(bt, counts, starts, num_pages):
    if oracle.fill_conflict(bt, _cu(counts), np.asarray(starts, np.int32), 0, num_pages):
        return {pkv.ERR_APPEND_CONFLICT}
    rows, mb = bt[0], bt.shape[2]
    errs = set()
    for b, (n, s0) in enumerate(zip(counts, starts)):
        if n == 0:
            continue
        if s0 < 0 or s0 + n > 16 * mb:
            errs.add(pkv.ERR_BAD_SEQ_LEN)
        elif any(not 0 <= rows[b, p // 16] < num_pages for p in range(s0, s0 + n)):
            errs.add(pkv.ERR_BAD_PAGE)
    return errs or {0}


@pytest.mark.parametrize("case", FILL_CONFLICT_CASES, ids=[c[0] for c in FILL_CONFLICT_CASES])
def test_fill_hand_worked_cases(case):
    _, rows, counts, starts, race = case
    bt = np.array([rows], np.int32)
    got = _fill_status(bt, counts, starts, APPEND_CASE_PAGES, seed=len(rows))
    assert (got == pkv.ERR_APPEND_CONFLICT) == race
    assert got in _fill_allowed(bt, counts, starts, APPEND_CASE_PAGES)


def test_fill_random_tables_match_oracle():
    rng = np.random.default_rng(123)
    races = 0
    for i in range(150):
        batch = int(rng.integers(1, 6))
        mb = int(rng.integers(1, 4))
        pages = int(rng.integers(1, 7))
        bt = rng.integers(-1, pages + 1, size=(1, batch, mb)).astype(np.int32)
        counts = [int(x) for x in rng.integers(0, 10, size=batch)]
        starts = [int(x) for x in rng.integers(-2, 16 * mb, size=batch)]
        want = _fill_allowed(bt, counts, starts, pages)
        got = _fill_status(bt, counts, starts, pages, seed=i)
        assert got in want, (i, bt, counts, starts, pages, got, want)
        races += want == {pkv.ERR_APPEND_CONFLICT}
    assert 10 < races < 140


def test_fill_flag_changes_nothing_on_a_workload():
    """Every prompt token of the batch-64 mix, with and without the check:
    no error, and the same pool bit for bit."""
    w = W.continuous_batching()
    dev = torch.device("cuda")
    counts = w.prefill_lens.astype(np.int64)
    cu = _cu(counts)
    assert not oracle.fill_conflict(w.block_tables, cu, np.zeros(w.batch, np.int32), 3,
                                    w.num_pages)
    gen = torch.Generator(device=dev).manual_seed(7)
    T = int(cu[-1])
    k = torch.randn((T, 8, 64), generator=gen, device=dev).to(torch.bfloat16)
    v = torch.randn((T, 8, 64), generator=gen, device=dev).to(torch.bfloat16)
    bt = torch.from_numpy(w.block_tables).to(dev)
    pools = []
    for flags in (0, pkv.LAUNCH_CHECK_APPENDS):
        pool_t = W.make_pool(w, dev)
        pool = pkv.Pool(w.num_pages, storage=pool_t)
        pool.set_launch_flags(flags)
        pkv.fill(pool, bt, to_dev(cu), torch.zeros(w.batch, dtype=torch.int32, device=dev), k, v,
                 3)
        torch.cuda.synchronize()
        assert pkv.get_device_error(pool) == 0
        pools.append(pool_t)
        pool.close()
    assert torch.equal(pools[0].view(torch.int16), pools[1].view(torch.int16))
