"""Pins of oracle.append_conflict, the definition of racing appends.

The oracle states the race as index conditions (two writes to one slot; for
the fused call, a written slot inside a context the call reads).  Here it is
checked against hand-worked cases (tests/cases.py) and against a different
formulation: run the call's accesses in different orders and see whether
anything observable changes -- the final pool when the writes are applied
forwards and backwards, and, for the fused call, what each context reads
before and after the writes.  Planted mistakes in the oracle's source must
fail these pins.
"""
import inspect

import numpy as np
import pytest

import oracle
import oracle.oracle as oo
from tests.cases import APPEND_CASE_PAGES, APPEND_CONFLICT_CASES


def _race_by_simulation(bt, lens, num_pages, fused):
    batch, mb = bt.shape

    def pool_after(order):
        pool = -1 - np.arange(num_pages * 16).reshape(num_pages, 16)   # distinct old values
        for b in order:
            L = int(lens[b])
            if 1 <= L <= 16 * mb and 0 <= bt[b, (L - 1) // 16] < num_pages:
                pool[bt[b, (L - 1) // 16], (L - 1) % 16] = b
        return pool

    before = pool_after([])
    fwd = pool_after(range(batch))
    if not np.array_equal(fwd, pool_after(reversed(range(batch)))):
        return True
    if not fused:
        return False
    for c in range(batch):
        L = int(lens[c])
        if not 1 <= L <= 16 * mb:
            continue
        for t in range(L - 1):   # position L-1 is c's own new token, defined as the new value
            p = bt[c, t // 16]
            if 0 <= p < num_pages and before[p, t % 16] != fwd[p, t % 16]:
                return True
    return False


def _random_case(rng):
    batch = int(rng.integers(1, 7))
    mb = int(rng.integers(1, 5))
    pages = int(rng.integers(1, 7))
    bt = rng.integers(-1, pages + 1, size=(1, batch, mb)).astype(np.int32)
    lens = rng.integers(0, 16 * mb + 1, size=batch).astype(np.int32)
    if rng.random() < 0.2:
        lens[rng.integers(batch)] = rng.choice([-1, 16 * mb + 1])
    if rng.random() < 0.5:   # short contexts on few pages make more races
        lens = np.minimum(lens, rng.integers(0, 20, size=batch)).astype(np.int32)
    return bt, lens, pages


@pytest.mark.parametrize("case", APPEND_CONFLICT_CASES, ids=[c[0] for c in APPEND_CONFLICT_CASES])
def test_hand_worked_cases(case):
    _, rows, lens, plain, fused = case
    bt = np.array([rows], np.int32)
    sl = np.array(lens, np.int32)
    assert oracle.append_conflict(bt, sl, 0, APPEND_CASE_PAGES, False) == plain
    assert oracle.append_conflict(bt, sl, 0, APPEND_CASE_PAGES, True) == fused


def test_hand_worked_cases_agree_with_simulation():
    for _, rows, lens, plain, fused in APPEND_CONFLICT_CASES:
        bt = np.array(rows, np.int32)
        assert _race_by_simulation(bt, lens, APPEND_CASE_PAGES, False) == plain
        assert _race_by_simulation(bt, lens, APPEND_CASE_PAGES, True) == fused


def test_matches_order_dependence_on_random_cases():
    rng = np.random.default_rng(2024)
    seen = {}
    for _ in range(3000):
        bt, lens, pages = _random_case(rng)
        for fused in (False, True):
            want = _race_by_simulation(bt[0], lens, pages, fused)
            assert oracle.append_conflict(bt, lens, 0, pages, fused) == want, (bt, lens, pages,
                                                                               fused)
            seen[(fused, want)] = seen.get((fused, want), 0) + 1
    assert min(seen.get(k, 0) for k in [(False, False), (False, True), (True, False),
                                        (True, True)]) > 50, seen


def test_layer_selects_the_slab():
    rows = [[5, 0], [5, 1]]
    bt = np.array([[[0, 1], [2, 3]], rows], np.int32)
    sl = np.array([3, 3], np.int32)
    assert not oracle.append_conflict(bt, sl, 0, APPEND_CASE_PAGES, False)
    assert oracle.append_conflict(bt, sl, 1, APPEND_CASE_PAGES, False)


MUTANTS = {
    "new_positions_not_read": ("if t < L and", "if t < L - 1 and"),
    "own_table_ignored": ("not (b == c and t == L - 1)", "b != c"),
    "own_position_counted": ("not (b == c and t == L - 1)", "True"),
    "slot_off_by_one": ("((L - 1) % 16, b)", "(L % 16, b)"),
    "page_index_off_by_one": ("bt[b, (L - 1) // 16]", "bt[b, L // 16 % max_blocks]"),
    "plain_compares_pages": ("slots = [s for s, _ in lst]", "slots = [0 for s, _ in lst]"),
    "outside_pool_written": ("if 0 <= page < num_pages:", "if True:"),
    "idle_sequences_read": ("        if not 1 <= L <= 16 * max_blocks:\n            continue\n"
                            "        for j", "        for j"),
}


def _mutant(old, new):
    src = inspect.getsource(oo.append_conflict)
    assert src.count(old) == 1, old
    ns = {"np": np}
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    return ns["append_conflict"]


def _pins_pass():
    try:
        for case in APPEND_CONFLICT_CASES:
            test_hand_worked_cases(case)
        test_matches_order_dependence_on_random_cases()
    except (AssertionError, IndexError):
        return False
    return True


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_mutant_fails_a_pin(name, monkeypatch):
    monkeypatch.setattr(oracle, "append_conflict", _mutant(*MUTANTS[name]))
    assert not _pins_pass()


def test_unmutated_source_passes(monkeypatch):
    monkeypatch.setattr(oracle, "append_conflict", _mutant("if t < L and", "if t < L and"))
    assert _pins_pass()
