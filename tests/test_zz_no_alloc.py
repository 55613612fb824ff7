"""GPU test of the allocation-free decode entry point.

paged_attention_decode_noalloc serves callers that cannot allocate device
memory where attention runs (allocator callbacks, runtime plugins that only
get their inputs and outputs, loops that must not synchronise on
cudaMalloc/cudaFree).  It runs the same decode as paged_attention_decode but
on a fixed scratch area the library keeps in device memory, so its output
must match the workspace entry point's within the attention tolerance, on
every call -- including a second call that finds the previous call's data
still in the shared scratch.  This file is collected last so that a run
stopping at the first failure has already run every other test; it also
passes on its own in a fresh process (its first call does the per-device
set-up).
"""
import ctypes

import numpy as np
import pytest
import torch

from paged_attention_decode_pkv_b200 import pkv
from tests.cases import make_case
from tests.harness import ATOL, GpuCase, max_err, u16_to_bf16

pytestmark = pytest.mark.gpu


def _noalloc(g, scale=0.125, layer=0):
    out = torch.full((g.q.shape[0], 32, 64), float("nan"), dtype=torch.float32, device="cuda")
    pkv.decode_noalloc(g.q, g.pool, g.bt, g.sl, layer, scale, out)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def test_noalloc_matches_workspace_entry_point_twice():
    # lengths that give split (multi-CTA) sequences, whole ones and an empty one
    cases = [GpuCase(make_case([1300, 17, 0, 260, 33, 1], seed=101, spare_pages=4)),
             GpuCase(make_case([40, 2500, 7, 16], seed=202, spare_pages=2))]
    for g in cases:
        ref = g.decode()
        first = _noalloc(g)
        second = _noalloc(g)
        assert max_err(first, ref) <= ATOL
        assert max_err(second, ref) <= ATOL
        assert max_err(first, g.oracle()) <= ATOL
        assert pkv.get_device_error(g.pool) == 0


def test_noalloc_after_other_calls_keeps_results():
    # The scratch keeps the previous call's contents; a different batch and
    # a different layer must not be affected by what is left there.
    a = GpuCase(make_case([3000, 5, 900], seed=303, spare_pages=3, num_layers=2))
    b = GpuCase(make_case([12, 700], seed=404, spare_pages=3))
    for layer in (1, 0):
        assert max_err(_noalloc(a, layer=layer), a.decode(layer=layer)) <= ATOL
    assert max_err(_noalloc(b, scale=0.3), b.decode(scale=0.3)) <= ATOL


def test_noalloc_rejects_batches_beyond_the_scratch():
    g = GpuCase(make_case([16, 16], seed=505))
    big = 8192   # far beyond what 16 MiB of scratch holds
    need = g.pool.workspace_bytes(big)
    assert need > pkv.NOALLOC_SCRATCH_BYTES
    bt = torch.zeros((1, big, 1), dtype=torch.int32, device="cuda")
    sl = torch.zeros((big,), dtype=torch.int32, device="cuda")
    q = torch.zeros((big, 32, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((big, 32, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(pkv.PkvError) as e:
        pkv.decode_noalloc(q, g.pool, bt, sl, 0, 0.125, out)
    assert e.value.status == pkv.ERR_TOO_LARGE
    assert "scratch" in pkv.lib.pkv_last_error_message().decode()


def test_noalloc_long_batch_then_short_batch():
    # A long-context call leaves many more split records in the shared scratch
    # than the next, shorter call writes; the shorter call must read only its
    # own (checked against the workspace entry point and the oracle).
    long_ = GpuCase(make_case([6000, 4100, 2500], seed=606, spare_pages=2))
    short = GpuCase(make_case([700, 30, 1500, 5, 260], seed=707, spare_pages=2))
    assert max_err(_noalloc(long_), long_.oracle()) <= ATOL
    for g in (short, long_, short):
        got = _noalloc(g)
        assert max_err(got, g.decode()) <= ATOL
        assert max_err(got, g.oracle()) <= ATOL
    assert pkv.get_device_error(short.pool) == 0
