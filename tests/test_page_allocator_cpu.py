"""Host page allocator of the C ABI (pkv_allocator_*), on the CPU.

Pages of the shared pool belong to one sequence at a time and are freed when
it ends (comrad404 article on samir-vllm, section on the KV cache and batched
decode); continuous batching admits a queued request only when its page
budget fits, queues the rest first in first out, and rejects a request larger
than the whole pool ("Curso gratuito recorre la inferencia de LLM...",
section on KV-cache memory).  The checks: allocation is all or nothing, the
two refusals are distinct, no page is ever held twice, freeing validates
before it frees, and a FIFO admission loop built on it runs every request to
completion without exceeding the pool.
"""
import collections

import numpy as np
import pytest

from paged_attention_decode_pkv_b200 import pkv


def test_fresh_allocator_hands_out_every_page_once():
    a = pkv.PageAllocator(40)
    assert a.free_count == 40
    got = a.alloc(16) + a.alloc(24)
    assert sorted(got) == list(range(40))
    assert got[:3] == [0, 1, 2]       # LIFO stack, page 0 on top of a fresh one
    assert a.free_count == 0
    with pytest.raises(pkv.PkvError) as e:
        a.alloc(1)
    assert e.value.status == pkv.ERR_OUT_OF_PAGES
    assert a.alloc(0) == []


def test_too_large_differs_from_out_of_pages_and_takes_nothing():
    a = pkv.PageAllocator(10)
    held = a.alloc(7)
    with pytest.raises(pkv.PkvError) as e:
        a.alloc(4)                    # fits the pool, not the free pages
    assert e.value.status == pkv.ERR_OUT_OF_PAGES
    with pytest.raises(pkv.PkvError) as e:
        a.alloc(11)                   # can never fit
    assert e.value.status == pkv.ERR_TOO_LARGE
    assert a.free_count == 3          # nothing taken by the failed calls
    a.free(held)
    assert a.free_count == 10
    assert sorted(a.alloc(10)) == list(range(10))


def test_free_rejects_bad_lists_without_freeing_any():
    a = pkv.PageAllocator(8)
    held = a.alloc(5)
    for bad in ([held[0], 99], [held[0], -1], [held[0], held[0]], [held[1], 7]):
        with pytest.raises(pkv.PkvError) as e:
            a.free(bad)               # 7 is still free, 99/-1 out of range, dup listed twice
        assert e.value.status == pkv.ERR_INVALID_ARG
        assert a.free_count == 3
    a.free(held[:2])
    with pytest.raises(pkv.PkvError):
        a.free(held[:1])              # double free
    assert a.free_count == 5


def test_create_and_alloc_reject_bad_arguments():
    for n in (0, -3):
        with pytest.raises(pkv.PkvError) as e:
            pkv.PageAllocator(n)
        assert e.value.status == pkv.ERR_INVALID_ARG
    a = pkv.PageAllocator(4)
    with pytest.raises(pkv.PkvError) as e:
        a.alloc(-1)
    assert e.value.status == pkv.ERR_INVALID_ARG
    assert pkv.lib.pkv_allocator_free_count(None) == -1
    assert pkv.lib.pkv_allocator_destroy(None) == pkv.OK


def test_fifo_admission_loop_runs_every_request_within_the_pool():
    # Requests need ceil((prompt + max_new) / 16) pages; each decode step ends
    # some running sequences, whose pages go back; the queue head is admitted
    # whenever its budget fits (first in first out), a request larger than the
    # pool is rejected.  Invariant: held pages are disjoint and never exceed
    # the pool; every admissible request finishes.
    rng = np.random.default_rng(7)
    P = 300
    a = pkv.PageAllocator(P)
    need = [int(-(-(rng.integers(1, 2000) + rng.integers(1, 400)) // 16)) for _ in range(400)]
    need[17] = P + 1                  # never fits
    queue = collections.deque(range(len(need)))
    running, done, rejected, order = {}, set(), set(), []
    while queue or running:
        while queue:
            r = queue[0]
            try:
                running[r] = a.alloc(need[r])
            except pkv.PkvError as e:
                if e.status == pkv.ERR_TOO_LARGE:
                    rejected.add(queue.popleft())
                    continue
                assert e.status == pkv.ERR_OUT_OF_PAGES
                break                 # the head waits; nothing behind it jumps the queue
            order.append(queue.popleft())
        held = [p for pages in running.values() for p in pages]
        assert len(held) == len(set(held)) <= P
        assert a.free_count == P - len(held)
        for r in list(running):
            if rng.random() < 0.3:
                a.free(running.pop(r))
                done.add(r)
    assert rejected == {17}
    assert done == set(range(len(need))) - {17}
    assert order == sorted(order)     # admitted in arrival order
    assert a.free_count == P


def test_random_operations_match_a_free_stack_model():
    # Thousands of random allocs and frees (good and bad) against a plain
    # Python model of the documented policy: a LIFO stack of free pages
    # (page 0 on top when fresh), all-or-nothing allocation, TOO_LARGE above
    # the pool size, OUT_OF_PAGES above the free count, and frees validated
    # as a whole (in range, held, listed once) before any page goes back.
    import random
    from paged_attention_decode_pkv_b200 import pkv
    rng = random.Random(2024)
    for n in (1, 7, 64, 300):
        a = pkv.PageAllocator(n)
        stack = list(range(n - 1, -1, -1))   # top = end
        held = set()
        for _ in range(3000):
            if rng.random() < 0.55:
                count = rng.choice([0, 1, 2, rng.randint(0, n), n, n + 1])
                if count > n:
                    want = pkv.ERR_TOO_LARGE
                elif count > len(stack):
                    want = pkv.ERR_OUT_OF_PAGES
                else:
                    want = pkv.OK
                if want == pkv.OK:
                    got = a.alloc(count)
                    exp = [stack.pop() for _ in range(count)]
                    assert got == exp
                    held.update(exp)
                else:
                    with pytest.raises(pkv.PkvError) as e:
                        a.alloc(count)
                    assert e.value.status == want
            else:
                pages = rng.sample(sorted(held), rng.randint(0, len(held))) if held else []
                bad = rng.random() < 0.3
                if bad:
                    kind = rng.choice(["range", "free", "twice"])
                    if kind == "range":
                        pages = pages + [rng.choice([-1, n, n + 5])]
                    elif kind == "free" and len(held) < n:
                        pages = pages + [rng.choice(sorted(set(range(n)) - held))]
                    elif kind == "twice" and pages:
                        pages = pages + [pages[0]]
                    else:
                        bad = False
                if bad:
                    with pytest.raises(pkv.PkvError) as e:
                        a.free(pages)
                    assert e.value.status == pkv.ERR_INVALID_ARG
                else:
                    a.free(pages)
                    stack.extend(pages)
                    held.difference_update(pages)
            assert a.free_count == len(stack)
            assert len(stack) + len(held) == n
        a.close()
