"""Pins of oracle.fill_conflict, the definition of racing fill writes.

Checked against hand-worked cases (tests/cases.py); against a different
formulation -- apply the call's token writes forwards and backwards and see
whether the pool differs; and against oracle.append_conflict, since a fill
of one token per sequence at position L - 1 is an append.  Planted mistakes
in the oracle's source must fail these pins.
"""
import inspect

import numpy as np
import pytest

import oracle
import oracle.oracle as oo
from tests.cases import APPEND_CASE_PAGES, FILL_CONFLICT_CASES


def _cu(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def _race_by_simulation(bt, counts, starts, num_pages):
    batch, mb = bt.shape

    def pool_after(order):
        pool = -1 - np.arange(num_pages * 16).reshape(num_pages, 16)
        for b, i in order:
            pos = starts[b] + i
            if starts[b] < 0 or starts[b] + counts[b] > 16 * mb:
                continue
            p = bt[b, pos // 16]
            if 0 <= p < num_pages:
                pool[p, pos % 16] = 1000 * b + i
        return pool

    writes = [(b, i) for b in range(batch) for i in range(counts[b])]
    return not np.array_equal(pool_after(writes), pool_after(writes[::-1]))


def _random_case(rng):
    batch = int(rng.integers(1, 6))
    mb = int(rng.integers(1, 4))
    pages = int(rng.integers(1, 7))
    bt = rng.integers(-1, pages + 1, size=(1, batch, mb)).astype(np.int32)
    counts = rng.integers(0, 10, size=batch).astype(np.int32)
    starts = rng.integers(-2, 16 * mb, size=batch).astype(np.int32)
    return bt, counts, starts, pages


@pytest.mark.parametrize("case", FILL_CONFLICT_CASES, ids=[c[0] for c in FILL_CONFLICT_CASES])
def test_hand_worked_cases(case):
    _, rows, counts, starts, race = case
    bt = np.array([rows], np.int32)
    assert oracle.fill_conflict(bt, _cu(counts), np.array(starts, np.int32), 0,
                                APPEND_CASE_PAGES) == race
    assert _race_by_simulation(bt[0], counts, starts, APPEND_CASE_PAGES) == race


def test_matches_order_dependence_on_random_cases():
    rng = np.random.default_rng(99)
    seen = [0, 0]
    for _ in range(3000):
        bt, counts, starts, pages = _random_case(rng)
        want = _race_by_simulation(bt[0], counts, starts, pages)
        assert oracle.fill_conflict(bt, _cu(counts), starts, 0, pages) == want, (bt, counts,
                                                                                  starts, pages)
        seen[want] += 1
    assert min(seen) > 300, seen


def test_one_token_fill_is_an_append():
    rng = np.random.default_rng(5)
    for _ in range(2000):
        batch = int(rng.integers(1, 7))
        mb = int(rng.integers(1, 4))
        pages = int(rng.integers(1, 6))
        bt = rng.integers(-1, pages + 1, size=(1, batch, mb)).astype(np.int32)
        lens = rng.integers(1, 16 * mb + 1, size=batch).astype(np.int32)
        got = oracle.fill_conflict(bt, _cu(np.ones(batch, np.int32)), lens - 1, 0, pages)
        assert got == oracle.append_conflict(bt, lens, 0, pages, False)


def test_cu_not_from_zero_writes_nothing_and_decreasing_cu_is_refused():
    bt = np.array([[[5, 0], [5, 1]]], np.int32)
    assert not oracle.fill_conflict(bt, np.array([1, 3, 5], np.int32),
                                    np.zeros(2, np.int32), 0, 8)
    with pytest.raises(ValueError):
        oracle.fill_conflict(bt, np.array([0, 3, 2], np.int32), np.zeros(2, np.int32), 0, 8)


MUTANTS = {
    "slot_from_token_index": ("(page, pos % 16) in seen", "(page, (pos - s0) % 16) in seen"),
    "range_check_dropped": ("if s0 < 0 or s0 + n > 16 * max_blocks:", "if False:"),
    "outside_pool_written": ("if not 0 <= page < num_pages:", "if False:"),
    "own_duplicates_ignored": ("        for pos in range(s0, s0 + n):",
                               "        seen_b = set(seen)\n        for pos in range(s0, s0 + n):"),
    "pages_compared": ("if (page, pos % 16) in seen:", "if (page, 0) in seen:"),
}


def _mutant(old, new):
    src = inspect.getsource(oo.fill_conflict)
    assert src.count(old) == 1, old
    src = src.replace(old, new)
    if "seen_b" in src:   # compare within the other sequences' slots only
        src = src.replace("            if (page, pos % 16) in seen:",
                          "            if (page, pos % 16) in seen_b:")
    ns = {"np": np}
    exec(compile(src, "<mutant>", "exec"), ns)
    return ns["fill_conflict"]


def _pins_pass():
    try:
        for case in FILL_CONFLICT_CASES:
            test_hand_worked_cases(case)
        test_matches_order_dependence_on_random_cases()
        test_one_token_fill_is_an_append()
    except (AssertionError, IndexError):
        return False
    return True


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_mutant_fails_a_pin(name, monkeypatch):
    monkeypatch.setattr(oracle, "fill_conflict", _mutant(*MUTANTS[name]))
    assert not _pins_pass()


def test_unmutated_source_passes(monkeypatch):
    monkeypatch.setattr(oracle, "fill_conflict", _mutant("if s0 < 0", "if s0 < 0"))
    assert _pins_pass()
