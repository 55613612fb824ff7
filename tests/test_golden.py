"""Golden case with formula-defined inputs (tests/golden/formula_case.py).

The expected values were written by tests/golden/make_golden.py, which calls
only the FP64 oracle.  On the CPU the oracle must still reproduce them to
1e-12 (a regression guard); on the GPU the CUDA path must match them to the
attention tolerance.
"""
import os

import numpy as np
import pytest

import oracle
from tests.golden import formula_case as fc

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _expected():
    rows = np.loadtxt(os.path.join(HERE, "formula_case_expected.txt"))
    return rows[:, 0].astype(int), rows[:, 1].astype(int), rows[:, 2].astype(int), rows[:, 3]


def test_oracle_reproduces_golden():
    q, pool = fc.inputs()
    out = oracle.decode(q, pool, fc.BT, fc.LENS, 0, fc.SCALE)
    b, h, d, v = _expected()
    assert np.max(np.abs(out[b, h, d] - v)) <= 1e-12
    assert not out[3].any()          # the empty sequence


@pytest.mark.gpu
@pytest.mark.parametrize("kernel", [1, 2])
def test_gpu_matches_golden(kernel):
    import torch
    from paged_attention_decode_pkv_b200 import pkv
    from tests.harness import ATOL, u16_to_bf16, to_dev
    q, pool = fc.inputs()
    pool_t = u16_to_bf16(pool)
    p = pkv.Pool(fc.NUM_PAGES, storage=pool_t)
    out = pkv.decode(u16_to_bf16(q), p, to_dev(fc.BT), to_dev(fc.LENS), 0, fc.SCALE, kernel=kernel)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    b, h, d, v = _expected()
    assert np.max(np.abs(got[b, h, d] - v)) <= ATOL
    assert not got[3].any()
    assert pkv.get_device_error(p) == 0
