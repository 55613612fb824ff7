"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the
CPU), builds it, swaps it in for the real oracle, and runs the pins of
tests/test_oracle_pins.py: at least one pin must fail for every mutant.
"""
import os
import subprocess

import pytest

import oracle
import oracle.oracle as oo
from oracle import build as obuild
from tests import test_oracle_pins as pins

MUTANTS = {
    "gqa_mod_instead_of_div": ("int g = h / O_Q_PER_KV;", "int g = h % O_KV_HEADS;"),
    "slot_off_by_one": ("int slot = (int)(t % O_TOKENS_PER_PAGE);\n      double acc",
                        "int slot = (int)((t + 1) % O_TOKENS_PER_PAGE);\n      double acc"),
    "scale_dropped": ("s[t] = jb->scale * acc;", "s[t] = acc;"),
    "normalisation_perturbed": ("oh[d] /= l;", "oh[d] /= (l * 1.0000001);"),
    "scores_from_values": ("o_bf16(jb->pool[o_offset(page, 0, g, slot, d)])",
                           "o_bf16(jb->pool[o_offset(page, 1, g, slot, d)])"),
    "weights_not_per_token": ("oh[d] += w[t] * o_bf16", "oh[d] += w[0] * o_bf16"),
    "append_wrong_slot": ("int slot = (int)(pos % O_TOKENS_PER_PAGE);\n    for",
                          "int slot = (int)((pos + 1) % O_TOKENS_PER_PAGE);\n    for"),
    "fill_wrong_slot": ("int slot = (int)(pos % O_TOKENS_PER_PAGE);\n      for",
                        "int slot = (int)((pos + 1) % O_TOKENS_PER_PAGE);\n      for"),
    "fill_source_row_not_offset": ("((int64_t)(cu[b] + i) * O_KV_HEADS + g)",
                                   "((int64_t)(i) * O_KV_HEADS + g)"),
    "fill_v_from_k": ("pool[o_offset(page, 1, g, slot, d)] = v_src[src];",
                      "pool[o_offset(page, 1, g, slot, d)] = k_src[src];"),
    "gather_k_from_v": ("k_out[dst] = pool[o_offset(page, 0, g, slot, d)];",
                        "k_out[dst] = pool[o_offset(page, 1, g, slot, d)];"),
}

PIN_CALLS = [
    lambda: [pins.test_decode_matches_bruteforce(l) for l in pins.LEN_SETS],
    lambda: [pins.test_decode_matches_torch_sdpa_fp64(l) for l in ([1, 17, 40], [33, 64])],
    pins.test_physical_page_permutation_is_bitwise_invariant,
    pins.test_single_token_returns_v_exactly,
    lambda: [pins.test_uniform_weights_give_mean_of_v(h) for h in ("equal_keys", "zero_q",
                                                                   "zero_scale")],
    pins.test_two_token_closed_form,
    pins.test_gqa_isolation,
    pins.test_key_shift_invariance,
    pins.test_append_writes_exactly_one_slot_per_kv_head,
    pins.test_append_then_single_token_decode_returns_v_new,
    pins.test_gather_matches_fancy_indexing_and_leaves_tail,
    pins.test_fill_equals_successive_appends,
    pins.test_fill_then_gather_returns_the_tokens,
]


def _build_mutant(tmp_path, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, old
    path = tmp_path / "pkv_oracle.c"
    path.write_text(src.replace(old, new))
    (tmp_path / "pkv_oracle.h").write_text(open(obuild.HDR).read())
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-pthread", str(path), "-o",
                    str(lib), "-lm"], check=True)
    return oo.load(str(lib))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_mutant_fails_a_pin(name, tmp_path):
    oracle.oracle._lib()             # make sure the real library is loaded first
    real = oo._LIB
    oo._LIB = _build_mutant(tmp_path, *MUTANTS[name])
    failed = 0
    try:
        for call in PIN_CALLS:
            try:
                call()
            except (AssertionError, oracle.OracleError):
                failed += 1
    finally:
        oo._LIB = real
    assert failed >= 1, "mutant %s passed every pin" % name


def test_unmutated_copy_passes_every_pin(tmp_path):
    oracle.oracle._lib()
    real = oo._LIB
    oo._LIB = _build_mutant(tmp_path, "oh[d] /= l;", "oh[d] /= l;")
    try:
        for call in PIN_CALLS:
            call()
    finally:
        oo._LIB = real
