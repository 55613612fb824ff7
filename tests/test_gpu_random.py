"""Seeded random sweep over the decode options together: lengths (page
boundaries, empty sequences), batch size, queries per sequence, output type,
fused append, kernel variant, grid and minimum chunk -- each case against the
FP64 oracle (and the pool bit for bit when the call appends)."""
import numpy as np
import pytest
import torch

import oracle
from paged_attention_decode_pkv_b200 import pkv
from tests.cases import NAN, bf16_bits, make_case
from tests.harness import ATOL, GpuCase, bits, max_err, u16_to_bf16

pytestmark = pytest.mark.gpu

CASES = 40


def _draw(rng):
    nq = int(rng.choice([1, 1, 1, 2, 3, 4, 6, 8]))
    B = int(rng.integers(1, 24))
    kinds = rng.integers(0, 4, B)
    lens = []
    for k in kinds:
        if k == 0:
            lens.append(0)
        elif k == 1:
            lens.append(int(16 * rng.integers(1, 6) + rng.integers(-1, 2)))   # around a boundary
        else:
            lens.append(int(rng.integers(1, 700)))
    lens = [0 if L == 0 else max(L, nq) for L in lens]
    fused = nq == 1 and bool(rng.integers(0, 2))
    kernel = pkv.KERNEL_MMA if nq > 1 else int(rng.choice([pkv.KERNEL_SIMT, pkv.KERNEL_MMA]))
    return dict(nq=nq, lens=lens, fused=fused, kernel=kernel,
                bf16=bool(rng.integers(0, 2)), grid=int(rng.choice([0, 1, 5, 77, 300])),
                min_chunk=int(rng.choice([0, 0, 1, 3])), scale=float(rng.uniform(0.05, 0.3)))


@pytest.mark.parametrize("i", range(CASES))
def test_random_option_mix(i):
    rng = np.random.default_rng(1000 + i)
    o = _draw(rng)
    c = make_case(o["lens"], seed=2000 + i, spare_pages=3)
    if o["fused"]:   # the new token's slot starts as NaN: the call must write it
        pool = c["pool"].copy()
        for b, L in enumerate(c["seq_lens"]):
            if L > 0:
                pool[c["bt"][0, b, (L - 1) // 16], :, :, (L - 1) % 16, :] = NAN
        c = dict(c, pool=pool)
    g = GpuCase(c)
    nq = o["nq"]
    q = c["q"] if nq == 1 else bf16_bits(rng.standard_normal((len(o["lens"]), nq, 32, 64)))
    kv = dict(k_new=u16_to_bf16(c["k_new"]), v_new=u16_to_bf16(c["v_new"])) if o["fused"] else {}
    out = pkv.decode_general(u16_to_bf16(q), g.pool, g.bt, g.sl, 0, o["scale"], num_queries=nq,
                             out_dtype=torch.bfloat16 if o["bf16"] else torch.float32,
                             kernel=o["kernel"], grid_ctas=o["grid"], min_chunk=o["min_chunk"],
                             **kv)
    torch.cuda.synchronize()
    assert pkv.get_device_error(g.pool) == 0, o
    host = c["pool"].copy()
    if o["fused"]:
        rows = np.nonzero(c["seq_lens"] > 0)[0]
        oracle.append(host, c["bt"][:, rows, :], c["seq_lens"][rows], c["k_new"][rows],
                      c["v_new"][rows], 0)
        assert np.array_equal(bits(g.pool_t).reshape(host.shape), host), o
    if nq == 1:
        want = oracle.decode(q, host, c["bt"], c["seq_lens"], 0, o["scale"])
    else:
        want = oracle.decode_multi(q, host, c["bt"], c["seq_lens"], 0, o["scale"])
    got = out.float().cpu().numpy().astype(np.float64)
    tol = ATOL + (np.abs(want) * 2.0 ** -8 if o["bf16"] else 0.0)
    assert np.isfinite(got).all(), o
    assert (np.abs(got - want) <= tol).all(), (o, max_err(got, want))
