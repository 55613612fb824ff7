"""ctypes wrapper around libpkv_oracle.so (TEST INFRASTRUCTURE ONLY).

Arrays are numpy: the pool is uint16 [num_pages, 2, 8, 16, 64] (BF16 bits,
layout page[kv][kv_head][slot][d]); block tables int32
[num_layers, batch, max_blocks]; seq_lens int32 [batch] (length after the
step's append); q uint16 [batch, 32, 64]; k_new / v_new uint16 [batch, 8, 64].
Outputs of decode are float64 [batch, 32, 64].  append_conflict and
fill_conflict (which writes of one call race) are plain Python on the same
arrays.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None
_CODES = {1: "bad argument", 2: "bad sequence length", 3: "block-table entry outside the pool"}


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__("oracle: %s (code %d)" % (_CODES.get(code, "?"), code))
        self.code = code


def load(path):
    """Open an oracle library at `path` and declare its functions."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i32 = ctypes.c_int32
    lib.pkvo_append.argtypes = [P, i32, P, i32, i32, i32, P, P, P, i32]
    lib.pkvo_gather.argtypes = [P, i32, P, i32, i32, i32, P, i32, P, P, i32]
    lib.pkvo_fill.argtypes = [P, i32, P, i32, i32, i32, P, P, P, P, i32]
    lib.pkvo_fill.restype = ctypes.c_int
    lib.pkvo_decode.argtypes = [P, P, i32, P, i32, i32, i32, P, i32, ctypes.c_double,
                                P, P, i32, i32]
    for f in (lib.pkvo_append, lib.pkvo_gather, lib.pkvo_decode):
        f.restype = ctypes.c_int
    return lib


def _lib():
    global _LIB
    if _LIB is None:
        _LIB = load(_build.build())
    return _LIB


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError("expected %s, got %s" % (np.dtype(dtype), a.dtype))
    return a


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc):
    if rc != 0:
        raise OracleError(rc)


def append(pool, block_tables, seq_lens, k_new, v_new, layer):
    """In-place append of one token per sequence (see pkv_oracle.h)."""
    if not (pool.flags.c_contiguous and pool.dtype == np.uint16):
        raise TypeError("pool must be C-contiguous uint16")
    bt = _c(block_tables, np.int32)
    sl = _c(seq_lens, np.int32)
    k = _c(k_new, np.uint16)
    v = _c(v_new, np.uint16)
    L, B, MB = bt.shape
    _check(_lib().pkvo_append(_p(pool), pool.shape[0], _p(bt), L, B, MB, _p(sl), _p(k), _p(v),
                              int(layer)))


def fill(pool, block_tables, cu, start, k_src, v_src, layer):
    """In-place prefill write of a ragged token batch (see pkv_oracle.h)."""
    if not (pool.flags.c_contiguous and pool.dtype == np.uint16):
        raise TypeError("pool must be C-contiguous uint16")
    bt = _c(block_tables, np.int32)
    cu = _c(cu, np.int32)
    st = _c(start, np.int32)
    k = _c(k_src, np.uint16)
    v = _c(v_src, np.uint16)
    L, B, MB = bt.shape
    _check(_lib().pkvo_fill(_p(pool), pool.shape[0], _p(bt), L, B, MB, _p(cu), _p(st), _p(k),
                            _p(v), int(layer)))


def gather(pool, block_tables, seq_lens, layer, max_seq_len, k_out=None, v_out=None):
    """Contiguous copy-out of K and V, [batch, 8, max_seq_len, 64] uint16 each."""
    pool = _c(pool, np.uint16)
    bt = _c(block_tables, np.int32)
    sl = _c(seq_lens, np.int32)
    L, B, MB = bt.shape
    if k_out is None:
        k_out = np.zeros((B, 8, max_seq_len, 64), np.uint16)
    if v_out is None:
        v_out = np.zeros((B, 8, max_seq_len, 64), np.uint16)
    _check(_lib().pkvo_gather(_p(pool), pool.shape[0], _p(bt), L, B, MB, _p(sl), int(layer),
                              _p(k_out), _p(v_out), int(max_seq_len)))
    return k_out, v_out


def decode(q, pool, block_tables, seq_lens, layer, scale, rows=None, nthreads=None, out=None):
    """FP64 decode attention; returns float64 [batch, 32, 64].

    rows: optional list of sequence indices to compute (others stay as in
    ``out``, zeros by default).  nthreads: worker threads (default: all cores).
    """
    q = _c(q, np.uint16)
    pool = _c(pool, np.uint16)
    bt = _c(block_tables, np.int32)
    sl = _c(seq_lens, np.int32)
    L, B, MB = bt.shape
    if out is None:
        out = np.zeros((B, 32, 64), np.float64)
    if rows is None:
        rp, nr = None, B
    else:
        rows_a = _c(np.asarray(rows, np.int32), np.int32)
        rp, nr = _p(rows_a), rows_a.size
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    _check(_lib().pkvo_decode(_p(q), _p(pool), pool.shape[0], _p(bt), L, B, MB, _p(sl),
                              int(layer), float(scale), _p(out), rp, nr, int(nthreads)))
    return out


def decode_multi(q, pool, block_tables, seq_lens, layer, scale, nthreads=None):
    """FP64 decode of several queries per sequence, causal among them.

    q: uint16 [batch, T, 32, 64].  Query i of sequence b sees the tokens
    t < seq_lens[b] - T + 1 + i (query T-1 sees the whole context, each
    earlier query one token fewer), so its output is single-query decode at
    that shorter length -- which is how it is computed here, one decode()
    call per query.  A sequence with 0 < seq_lens[b] < T has a query with no
    token: OracleError (bad length).  Returns float64 [batch, T, 32, 64].
    """
    q = np.asarray(q, np.uint16)
    B, T = q.shape[0], q.shape[1]
    sl = np.asarray(seq_lens, np.int64)
    if ((sl > 0) & (sl < T)).any():
        raise OracleError(2)
    out = np.zeros((B, T, 32, 64), np.float64)
    for i in range(T):
        li = np.where(sl > 0, sl - T + 1 + i, 0).astype(np.int32)
        out[:, i] = decode(np.ascontiguousarray(q[:, i]), pool, block_tables, li, layer, scale,
                           nthreads=nthreads)
    return out


def append_conflict(block_tables, seq_lens, layer, num_pages, fused):
    """True when the appends of one call race, by the definition of an append.

    Sequence b with 1 <= L_b <= 16 * max_blocks writes position L_b - 1: slot
    (L_b - 1) % 16 of page block_tables[layer][b][(L_b - 1) // 16] ("Curso
    gratuito recorre la inferencia de LLM...", section on the KV cache), when
    that page lies in the pool; other sequences write nothing.
      plain append (fused=False): two sequences write the same (page, slot).
      fused append + decode (fused=True): some written (page, slot) is read by
        the call, other than by its writer at its own new position: sequence
        c (1 <= L_c <= 16 * max_blocks) reads slot t % 16 of page
        block_tables[layer][c][t // 16] for every t < L_c.  Two writes to one
        slot are the case where one writer reads the other's new position.
    Plain Python over the (page -> writes) map; fine up to full workload sizes.
    """
    bt = np.asarray(block_tables)[layer]
    lens = np.asarray(seq_lens)
    batch, max_blocks = bt.shape
    writes = {}   # page -> [(slot, writer)]
    for b in range(batch):
        L = int(lens[b])
        if not 1 <= L <= 16 * max_blocks:
            continue
        page = int(bt[b, (L - 1) // 16])
        if 0 <= page < num_pages:
            writes.setdefault(page, []).append(((L - 1) % 16, b))
    if not fused:
        for lst in writes.values():
            slots = [s for s, _ in lst]
            if len(set(slots)) != len(slots):
                return True
        return False
    for c in range(batch):
        L = int(lens[c])
        if not 1 <= L <= 16 * max_blocks:
            continue
        for j in range((L + 15) // 16):
            for s, b in writes.get(int(bt[c, j]), ()):
                t = 16 * j + s
                if t < L and not (b == c and t == L - 1):
                    return True
    return False


def fill_conflict(block_tables, cu, start, layer, num_pages):
    """True when two tokens of one fill call are written to the same slot.

    Token i of sequence b (i < cu[b+1] - cu[b]) goes to position start[b] + i,
    slot (start[b] + i) % 16 of page block_tables[layer][b][(start[b] + i) // 16]
    ("Curso gratuito recorre la inferencia de LLM...", section on the KV
    cache).  A sequence with start[b] < 0 or an end beyond 16 * max_blocks
    writes nothing, nor does a token whose page lies outside the pool; when
    cu does not start at 0 the call writes nothing at all.  cu must be
    non-decreasing (ValueError otherwise: which tokens are written is then
    unspecified).
    """
    bt = np.asarray(block_tables)[layer]
    cu = np.asarray(cu)
    st = np.asarray(start)
    batch, max_blocks = bt.shape
    if np.any(np.diff(cu) < 0):
        raise ValueError("cu_tokens decreases")
    if cu[0] != 0:
        return False
    seen = set()
    for b in range(batch):
        n = int(cu[b + 1] - cu[b])
        s0 = int(st[b])
        if s0 < 0 or s0 + n > 16 * max_blocks:
            continue
        for pos in range(s0, s0 + n):
            page = int(bt[b, pos // 16])
            if not 0 <= page < num_pages:
                continue
            if (page, pos % 16) in seen:
                return True
            seen.add((page, pos % 16))
    return False
