"""Host-side argument checks of the decode entry points, through the raw C
ABI: every invalid call returns its documented status and launches nothing
(the output buffer keeps its sentinel), and the valid call next to each
invalid one succeeds.  The header documents these checks per call; this file
holds them to it."""
import ctypes

import numpy as np
import pytest
import torch

from paged_attention_decode_pkv_b200 import pkv
from tests.cases import make_case
from tests.harness import GpuCase, u16_to_bf16

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


@pytest.fixture(scope="module")
def setup():
    c = make_case([40, 300, 7], seed=91, spare_pages=2, num_layers=2)
    g = GpuCase(c)
    B, MB = 3, c["bt"].shape[2]
    ws = g.pool.workspace(B)
    out = torch.full((B + 1, 32, 64), 7.0, dtype=torch.float32, device="cuda")
    k = u16_to_bf16(c["k_new"])
    v = u16_to_bf16(c["v_new"])
    return dict(g=g, B=B, MB=MB, ws=ws, out=out, k=k, v=v)


def _decode_ex(s, q=None, out=None, layer=0, num_layers=2, batch=None, max_blocks=None,
               ws=None, ws_bytes=None, scale=0.125, kernel=pkv.KERNEL_AUTO, grid=0, min_chunk=0,
               pool=None):
    g = s["g"]
    return pkv.lib.paged_attention_decode_ex(
        P(g.q.data_ptr()) if q is None else q, g.pool.handle if pool is None else pool,
        P(g.bt.data_ptr()), P(g.sl.data_ptr()), layer, ctypes.c_float(scale),
        P(s["out"].data_ptr()) if out is None else out, num_layers,
        s["B"] if batch is None else batch, s["MB"] if max_blocks is None else max_blocks,
        P(s["ws"].data_ptr()) if ws is None else ws,
        s["ws"].numel() if ws_bytes is None else ws_bytes, None, kernel, grid, min_chunk)


def _untouched(s):
    torch.cuda.synchronize()
    return bool((s["out"] == 7.0).all())


BAD_DECODE = [
    ("layer == num_layers", dict(layer=2), pkv.ERR_INVALID_ARG),
    ("negative layer", dict(layer=-1), pkv.ERR_INVALID_ARG),
    ("num_layers 0", dict(num_layers=0, layer=0), pkv.ERR_INVALID_ARG),
    ("negative batch", dict(batch=-1), pkv.ERR_INVALID_ARG),
    ("max_blocks 0", dict(max_blocks=0), pkv.ERR_INVALID_ARG),
    ("NaN scale", dict(scale=float("nan")), pkv.ERR_INVALID_ARG),
    ("negative grid", dict(grid=-1), pkv.ERR_INVALID_ARG),
    ("negative min_chunk", dict(min_chunk=-3), pkv.ERR_INVALID_ARG),
    ("unknown kernel", dict(kernel=7), pkv.ERR_UNSUPPORTED),
    ("workspace too small", dict(ws_bytes=1024), pkv.ERR_WORKSPACE),
    ("no workspace", dict(ws=P(0)), pkv.ERR_WORKSPACE),
    ("null pool", dict(pool=P(0)), pkv.ERR_INVALID_ARG),
]


@pytest.mark.parametrize("what,kw,status", BAD_DECODE, ids=[b[0] for b in BAD_DECODE])
def test_invalid_decode_arguments_are_rejected_before_launch(setup, what, kw, status):
    s = setup
    assert _decode_ex(s, **kw) == status, what
    assert _untouched(s), what


def test_misaligned_pointers_are_rejected(setup):
    s = setup
    g = s["g"]
    # q and out must be 16-byte aligned, the workspace 256-byte aligned
    assert _decode_ex(s, q=P(g.q.data_ptr() + 2)) == pkv.ERR_INVALID_ARG
    assert _decode_ex(s, out=P(s["out"].data_ptr() + 4)) == pkv.ERR_INVALID_ARG
    assert _decode_ex(s, ws=P(s["ws"].data_ptr() + 16), ws_bytes=s["ws"].numel() - 16) == \
        pkv.ERR_WORKSPACE
    assert _untouched(s)


def test_the_valid_call_next_to_them_runs(setup):
    s = setup
    assert _decode_ex(s) == pkv.OK
    torch.cuda.synchronize()
    assert not (s["out"][:3] == 7.0).any()      # all three rows written
    assert (s["out"][3] == 7.0).all()           # nothing past the batch
    assert pkv.get_device_error(s["g"].pool) == 0
    s["out"].fill_(7.0)


def test_general_call_option_checks(setup):
    s = setup
    g = s["g"]

    def params(**kw):
        p = pkv.DecodeParams(struct_size=ctypes.sizeof(pkv.DecodeParams))
        p.q, p.block_tables, p.seq_lens = g.q.data_ptr(), g.bt.data_ptr(), g.sl.data_ptr()
        p.out, p.workspace, p.workspace_bytes = s["out"].data_ptr(), s["ws"].data_ptr(), \
            s["ws"].numel()
        p.scale, p.layer, p.num_layers, p.batch, p.max_blocks = 0.125, 0, 2, s["B"], s["MB"]
        p.num_queries, p.out_dtype = 1, pkv.DTYPE_F32
        for k, v in kw.items():
            setattr(p, k, v)
        return p

    def call(p):
        return pkv.lib.pkv_decode(g.pool.handle, ctypes.byref(p), None)

    assert call(params(num_queries=0)) == pkv.ERR_UNSUPPORTED
    assert call(params(num_queries=9)) == pkv.ERR_UNSUPPORTED
    assert call(params(num_queries=2, kernel=pkv.KERNEL_SIMT)) == pkv.ERR_UNSUPPORTED
    assert call(params(out_dtype=5)) == pkv.ERR_INVALID_ARG
    assert call(params(k_new=s["k"].data_ptr())) == pkv.ERR_INVALID_ARG       # k without v
    assert call(params(k_new=s["k"].data_ptr(), v_new=s["v"].data_ptr(), num_queries=2)) == \
        pkv.ERR_UNSUPPORTED                                                     # fused: 1 query
    small = params()
    small.struct_size = ctypes.sizeof(pkv.DecodeParams) - 8
    assert call(small) == pkv.ERR_INVALID_ARG                                  # older layout
    assert _untouched(s)
    assert call(params()) == pkv.OK
    torch.cuda.synchronize()
    s["out"].fill_(7.0)


def test_calls_on_another_device_are_rejected(setup):
    # the pool's device must be current; with one GPU, a device index that
    # is not current can only be simulated when a second device exists
    if torch.cuda.device_count() < 2:
        pytest.skip("one GPU: nothing else can be current")
    s = setup
    with torch.cuda.device(1):
        assert _decode_ex(s) == pkv.ERR_INVALID_ARG
    assert _untouched(s)
