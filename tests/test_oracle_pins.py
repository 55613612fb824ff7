"""Pins of the FP64 CPU oracle against things other than itself.

The pages print no worked numeric example, so each part of the oracle is
pinned by mathematics: a brute-force contiguous computation written
separately (numpy fancy indexing + np.repeat for GQA), a library routine
(torch scaled_dot_product_attention in float64), closed forms (one token,
two tokens, equal keys), and invariants (physical-page permutation, kv-head
isolation, key shift).  Each test is chosen so that a plausible slip in the
oracle (a wrong GQA map, a wrong page/slot index, a dropped max, a missing
normalisation, a transposed operand) fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.cases import D, G, H, NAN, T, bf16_bits, bf16_to_f64, contiguous_kv, make_case


def _decode(c, scale=0.125, layer=0, **kw):
    return oracle.decode(c["q"], c["pool"], c["bt"], c["seq_lens"], layer, scale, **kw)


def _brute(c, scale=0.125, layer=0):
    """Contiguous attention, written independently of the oracle."""
    out = np.zeros((len(c["seq_lens"]), H, D))
    for b, (K, V) in enumerate(contiguous_kv(c, layer)):
        if K.shape[1] == 0:
            continue
        Kh = np.repeat(K, H // G, axis=0)          # [H, L, D]; q head h uses kv head h // 4
        Vh = np.repeat(V, H // G, axis=0)
        q = bf16_to_f64(c["q"][b])                 # [H, D]
        s = scale * np.einsum("hd,hld->hl", q, Kh)
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[b] = np.einsum("hl,hld->hd", p, Vh)
    return out


LEN_SETS = [[1], [15], [16], [17], [31, 32, 33], [1, 40, 17, 64, 5], [0, 3]]


@pytest.mark.parametrize("lens", LEN_SETS)
def test_decode_matches_bruteforce(lens):
    c = make_case(lens, seed=sum(lens) + len(lens))
    got = _decode(c)
    want = _brute(c)
    assert np.max(np.abs(got - want)) <= 1e-12


@pytest.mark.parametrize("lens", [[1, 17, 40], [33, 64]])
def test_decode_matches_torch_sdpa_fp64(lens):
    c = make_case(lens, seed=7)
    got = _decode(c, scale=0.3)
    for b, (K, V) in enumerate(contiguous_kv(c)):
        q = torch.from_numpy(bf16_to_f64(c["q"][b]))[:, None, :]          # [H, 1, D]
        k = torch.from_numpy(K).repeat_interleave(H // G, dim=0)          # [H, L, D]
        v = torch.from_numpy(V).repeat_interleave(H // G, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=0.3)[:, 0, :]
        assert np.max(np.abs(got[b] - ref.numpy())) <= 1e-12


def test_physical_page_permutation_is_bitwise_invariant():
    c = make_case([17, 40, 1, 33], seed=3, spare_pages=5)
    base = _decode(c)
    rng = np.random.default_rng(11)
    pi = rng.permutation(c["pool"].shape[0])        # page p moves to pi[p]
    pool2 = np.empty_like(c["pool"])
    pool2[pi] = c["pool"]
    bt2 = np.where(c["bt"] >= 0, pi[np.maximum(c["bt"], 0)], -1).astype(np.int32)
    c2 = dict(c, pool=pool2, bt=bt2)
    assert np.array_equal(_decode(c2), base)        # same sums in the same order


def test_single_token_returns_v_exactly():
    c = make_case([1, 1, 1], seed=5)
    got = _decode(c, scale=0.77)
    for b in range(3):
        v = bf16_to_f64(c["v_new"][b])               # [G, D]
        assert np.array_equal(got[b], np.repeat(v, H // G, axis=0))


@pytest.mark.parametrize("how", ["equal_keys", "zero_q", "zero_scale"])
def test_uniform_weights_give_mean_of_v(how):
    c = make_case([37, 16, 5], seed=9)
    scale = 0.125
    if how == "equal_keys":
        for b, L in enumerate(c["seq_lens"]):
            key = bf16_bits(np.random.default_rng(b).standard_normal((G, D)))
            for t in range(int(L)):
                c["pool"][c["bt"][0, b, t // T], 0, :, t % T, :] = key
    elif how == "zero_q":
        c["q"][:] = 0
    else:
        scale = 0.0
    got = _decode(c, scale=scale)
    for b, (K, V) in enumerate(contiguous_kv(c)):
        want = np.repeat(V.mean(axis=1), H // G, axis=0)
        assert np.max(np.abs(got[b] - want)) <= 1e-12


def test_two_token_closed_form():
    c = make_case([2], seed=13)
    scale = 0.21
    got = _decode(c, scale=scale)[0]
    K, V = contiguous_kv(c)[0]
    q = bf16_to_f64(c["q"][0])
    for h in range(H):
        g = h // 4
        s0 = scale * float(q[h] @ K[g, 0])
        s1 = scale * float(q[h] @ K[g, 1])
        w0 = 1.0 / (1.0 + math.exp(s1 - s0))        # sigma(s0 - s1)
        w1 = 1.0 / (1.0 + math.exp(s0 - s1))
        assert np.max(np.abs(got[h] - (w0 * V[g, 0] + w1 * V[g, 1]))) <= 1e-12


def test_gqa_isolation():
    c = make_case([29, 50], seed=17)
    base = _decode(c)
    g_pert = 5
    pool2 = c["pool"].copy()
    for b, L in enumerate(c["seq_lens"]):
        for t in range(int(L)):
            p = c["bt"][0, b, t // T]
            pool2[p, :, g_pert, t % T, :] = bf16_bits(np.random.default_rng(t).standard_normal((2, D)))
    out = _decode(dict(c, pool=pool2))
    changed = np.any(out != base, axis=(0, 2))
    assert changed.tolist() == [h // 4 == g_pert for h in range(H)]


def test_key_shift_invariance():
    # Adding one vector c to every key of (b, g) adds scale*q.c to all of its
    # scores, which the softmax removes.  Keys and c are small integers so
    # the shifted keys stay exact in BF16.
    c = make_case([23], seed=19)
    rng = np.random.default_rng(1)
    K_int = rng.integers(-4, 5, size=(T * 2, G, D)).astype(np.float32)
    shift = rng.integers(-4, 5, size=(G, D)).astype(np.float32)
    pool_a = c["pool"].copy()
    pool_b = c["pool"].copy()
    for t in range(23):
        p = c["bt"][0, 0, t // T]
        pool_a[p, 0, :, t % T, :] = bf16_bits(K_int[t])
        pool_b[p, 0, :, t % T, :] = bf16_bits(K_int[t] + shift)
    c["q"][:] = bf16_bits(rng.integers(-2, 3, size=(1, H, D)).astype(np.float32) / 8)
    a = _decode(dict(c, pool=pool_a), scale=0.125)
    b = _decode(dict(c, pool=pool_b), scale=0.125)
    assert np.max(np.abs(a - b)) <= 1e-12


def test_nan_outside_context_never_read():
    # make_case fills every slot outside the context with NaN; finite output
    # shows the oracle reads only slots t < L of the listed pages.
    c = make_case([1, 15, 16, 17, 47], seed=23, spare_pages=6)
    assert np.isfinite(_decode(c)).all()


def test_zero_length_gives_zero_row():
    c = make_case([0, 5], seed=29)
    out = _decode(c)
    assert np.array_equal(out[0], np.zeros((H, D)))
    assert np.isfinite(out[1]).all()


def test_rows_and_threads_do_not_change_results():
    c = make_case([40, 1, 17, 33, 5], seed=31)
    full = _decode(c, nthreads=1)
    thr = _decode(c, nthreads=3)
    assert np.array_equal(full, thr)
    part = _decode(c, rows=[3, 1], nthreads=2)
    assert np.array_equal(part[[1, 3]], full[[1, 3]])
    assert not part[[0, 2, 4]].any()


def test_multi_layer_uses_the_layer_slab():
    c = make_case([20, 9], seed=37, num_layers=3)
    for layer in range(3):
        got = _decode(c, layer=layer)
        assert np.max(np.abs(got - _brute(c, layer=layer))) <= 1e-12


# ------------------------------------------------------------------ append --

def test_append_writes_exactly_one_slot_per_kv_head():
    c = make_case([17, 40, 1, 16], seed=41, spare_pages=4)
    pool = c["pool"].copy()
    rng = np.random.default_rng(2)
    k_new = bf16_bits(rng.standard_normal((4, G, D)))
    v_new = bf16_bits(rng.standard_normal((4, G, D)))
    oracle.append(pool, c["bt"], c["seq_lens"], k_new, v_new, 0)
    diff = pool != c["pool"]
    expect = np.zeros_like(diff)
    for b, L in enumerate(c["seq_lens"]):
        p, s = c["bt"][0, b, (L - 1) // T], (L - 1) % T
        expect[p, :, :, s, :] = (np.stack([k_new[b], v_new[b]]) != c["pool"][p, :, :, s, :])
        assert np.array_equal(pool[p, 0, :, s, :], k_new[b])
        assert np.array_equal(pool[p, 1, :, s, :], v_new[b])
    assert np.array_equal(diff, expect)


def test_append_then_single_token_decode_returns_v_new():
    # Cross-check of the append index against the decode index: a sequence
    # whose only token was just appended must decode to v_new.
    c = make_case([1, 1], seed=43, spare_pages=2)
    pool = np.full_like(c["pool"], NAN)
    rng = np.random.default_rng(3)
    k_new = bf16_bits(rng.standard_normal((2, G, D)))
    v_new = bf16_bits(rng.standard_normal((2, G, D)))
    oracle.append(pool, c["bt"], c["seq_lens"], k_new, v_new, 0)
    out = oracle.decode(c["q"], pool, c["bt"], c["seq_lens"], 0, 0.125)
    for b in range(2):
        assert np.array_equal(out[b], np.repeat(bf16_to_f64(v_new[b]), 4, axis=0))


def test_append_rejects_bad_inputs():
    c = make_case([17, 5], seed=47)
    pool = c["pool"].copy()
    with pytest.raises(oracle.OracleError):
        oracle.append(pool, c["bt"], np.array([0, 5], np.int32), c["k_new"], c["v_new"], 0)
    bad = c["bt"].copy()
    bad[0, 1, 0] = pool.shape[0]
    with pytest.raises(oracle.OracleError):
        oracle.append(pool, bad, c["seq_lens"], c["k_new"], c["v_new"], 0)
    assert np.array_equal(pool, c["pool"])          # nothing written on error


# ------------------------------------------------------------------ gather --

def test_gather_matches_fancy_indexing_and_leaves_tail():
    c = make_case([17, 40, 0, 33], seed=53, num_layers=2)
    for layer in range(2):
        k0 = np.full((4, G, 48, D), 0x1234, np.uint16)
        v0 = np.full((4, G, 48, D), 0x4321, np.uint16)
        k, v = oracle.gather(c["pool"], c["bt"], c["seq_lens"], layer, 48, k0.copy(), v0.copy())
        for b, L in enumerate(c["seq_lens"]):
            t = np.arange(int(L))
            pages = c["bt"][layer, b, t // T]
            assert np.array_equal(k[b, :, :L], c["pool"][pages, 0, :, t % T, :].transpose(1, 0, 2))
            assert np.array_equal(v[b, :, :L], c["pool"][pages, 1, :, t % T, :].transpose(1, 0, 2))
            assert (k[b, :, L:] == 0x1234).all() and (v[b, :, L:] == 0x4321).all()


def test_decode_rejects_bad_page_and_length():
    c = make_case([17, 5], seed=59)
    bad = c["bt"].copy()
    bad[0, 0, 1] = -1
    with pytest.raises(oracle.OracleError):
        oracle.decode(c["q"], c["pool"], bad, c["seq_lens"], 0, 0.125)
    with pytest.raises(oracle.OracleError):
        oracle.decode(c["q"], c["pool"], c["bt"], np.array([17, 10_000], np.int32), 0, 0.125)


# -------------------------------------------------------------------- fill --

def _ragged(rng, lens_before, counts):
    cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    k = bf16_bits(rng.standard_normal((int(cu[-1]), G, D)))
    v = bf16_bits(rng.standard_normal((int(cu[-1]), G, D)))
    return cu, np.asarray(lens_before, np.int32), k, v


def test_fill_equals_successive_appends():
    # A prefill of T tokens is T appends in a row (the append index is
    # pinned above), so both must leave the same pool bits.
    lens_after = [37, 16, 5, 50]
    c = make_case(lens_after, seed=61, spare_pages=4)
    rng = np.random.default_rng(4)
    start = [3, 0, 5, 20]
    counts = [34, 16, 0, 30]
    cu, st, k, v = _ragged(rng, start, counts)
    filled = c["pool"].copy()
    oracle.fill(filled, c["bt"], cu, st, k, v, 0)
    appended = c["pool"].copy()
    for i in range(max(counts)):
        rows = [b for b in range(4) if i < counts[b]]
        if not rows:
            continue
        sl = np.array([st[b] + i + 1 for b in rows], np.int32)
        bt = c["bt"][:, rows, :]
        oracle.append(appended, bt, sl, k[[cu[b] + i for b in rows]], v[[cu[b] + i for b in rows]], 0)
    assert np.array_equal(filled, appended)


def test_fill_then_gather_returns_the_tokens():
    c = make_case([40, 17], seed=67, spare_pages=2)
    rng = np.random.default_rng(5)
    cu, st, k, v = _ragged(rng, [0, 0], [40, 17])
    pool = np.full_like(c["pool"], NAN)
    oracle.fill(pool, c["bt"], cu, st, k, v, 0)
    ko, vo = oracle.gather(pool, c["bt"], c["seq_lens"], 0, 40)
    for b, n in enumerate([40, 17]):
        assert np.array_equal(ko[b, :, :n].transpose(1, 0, 2), k[cu[b]:cu[b + 1]])
        assert np.array_equal(vo[b, :, :n].transpose(1, 0, 2), v[cu[b]:cu[b + 1]])


def test_fill_rejects_out_of_range_without_writing():
    c = make_case([20, 5], seed=71)
    rng = np.random.default_rng(6)
    cu, st, k, v = _ragged(rng, [10, 0], [40, 5])    # 10 + 40 > max_blocks * 16 = 32
    pool = c["pool"].copy()
    with pytest.raises(oracle.OracleError):
        oracle.fill(pool, c["bt"], cu, st, k, v, 0)
    assert np.array_equal(pool, c["pool"])


# ---- several queries per sequence, causal among them (oracle.decode_multi)

def _brute_multi(c, q2, scale=0.125):
    """Causal two-query attention written out with an explicit mask: query i
    of a length-L sequence scores every token and masks t > L - 2 + i."""
    B, Tq = q2.shape[0], q2.shape[1]
    out = np.zeros((B, Tq, H, D))
    for b, (K, V) in enumerate(contiguous_kv(c)):
        L = K.shape[1]
        if L == 0:
            continue
        Kh = np.repeat(K, H // G, axis=0)
        Vh = np.repeat(V, H // G, axis=0)
        for i in range(Tq):
            q = bf16_to_f64(q2[b, i])
            s = scale * np.einsum("hd,hld->hl", q, Kh)
            s[:, np.arange(L) > L - Tq + i] = -np.inf
            s -= s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            out[b, i] = np.einsum("hl,hld->hd", p, Vh)
    return out


@pytest.mark.parametrize("lens,nq", [([2], 2), ([16], 2), ([17], 2), ([18], 2),
                                     ([33, 2, 0, 40], 2), ([3, 17, 19], 3), ([8, 16, 23, 40], 8)])
def test_decode_multi_matches_causal_bruteforce(lens, nq):
    c = make_case(lens, seed=sum(lens) + 3)
    rng = np.random.default_rng(len(lens))
    q2 = bf16_bits(rng.standard_normal((len(lens), nq, H, D)))
    got = oracle.decode_multi(q2, c["pool"], c["bt"], c["seq_lens"], 0, 0.125)
    assert np.max(np.abs(got - _brute_multi(c, q2))) <= 1e-12


def test_decode_multi_one_query_is_decode_and_last_query_sees_all():
    c = make_case([40, 2, 17], seed=21)
    got1 = oracle.decode_multi(c["q"][:, None], c["pool"], c["bt"], c["seq_lens"], 0, 0.2)
    assert np.array_equal(got1[:, 0], _decode(c, scale=0.2))
    rng = np.random.default_rng(4)
    q2 = bf16_bits(rng.standard_normal((3, 2, H, D)))
    q2[:, 1] = c["q"]
    got2 = oracle.decode_multi(q2, c["pool"], c["bt"], c["seq_lens"], 0, 0.2)
    assert np.array_equal(got2[:, 1], _decode(c, scale=0.2))   # the last query: plain decode


def test_decode_multi_rejects_a_query_without_tokens():
    c = make_case([1, 5], seed=2)
    with pytest.raises(oracle.OracleError):
        oracle.decode_multi(np.zeros((2, 2, H, D), np.uint16), c["pool"], c["bt"],
                            c["seq_lens"], 0, 0.125)


def test_shared_pages_read_in_place_equal_private_copies():
    # Pages that several sequences' tables name (a reused prompt prefix) are
    # read in place ("Curso gratuito recorre la inferencia de LLM...",
    # section on the KV cache: decode reads the pages where they are): the
    # output is bitwise that of the same batch with the prefix copied into
    # private pages.
    from tests.cases import shared_prefix_case
    shared, private = shared_prefix_case()
    a = oracle.decode(shared["q"], shared["pool"], shared["bt"], shared["seq_lens"], 0, 0.125)
    b = oracle.decode(private["q"], private["pool"], private["bt"], private["seq_lens"], 0, 0.125)
    assert (shared["bt"][0, :, :3] == shared["bt"][0, 0, :3]).all()   # really shared
    assert len(np.unique(private["bt"][0, :, :3])) == 3 * shared["bt"].shape[1]
    assert np.array_equal(a, b)
