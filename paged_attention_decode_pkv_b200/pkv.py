"""Python binding of libpkv (the C ABI in include/pkv.h).

Argument marshalling only: every step of append, fill, gather and decode
runs in the CUDA kernels of libpkv.so (the page allocator is host C code in
the same library).  Tensors are torch CUDA tensors; torch is used
for device memory and streams, nothing else.  There is no CPU fallback: if
libpkv.so is missing or cannot be loaded, importing this module raises.
"""
from __future__ import annotations

import atexit
import ctypes
import os
import sys
import weakref
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("PKV_LIBRARY") or os.path.join(_HERE, "libpkv.so")

PAGE_TOKENS = 16
NUM_KV_HEADS = 8
NUM_Q_HEADS = 32
HEAD_DIM = 64
PAGE_BYTES = 32768

KERNEL_AUTO, KERNEL_SIMT, KERNEL_MMA = 0, 1, 2
DTYPE_F32, DTYPE_BF16 = 0, 1
MAX_QUERIES = 8
LAUNCH_PDL = 1
LAUNCH_EARLY_TABLES = 2
LAUNCH_EARLY_PAGES = 4
LAUNCH_CHECK_APPENDS = 8
LAUNCH_TEST_STALL = 1 << 30

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_CUDA = -3
ERR_OUT_OF_PAGES = -4
ERR_BAD_PAGE = -5
ERR_WORKSPACE = -6
ERR_DEVICE_TIMEOUT = -7
ERR_BAD_SEQ_LEN = -8
ERR_TOO_LARGE = -9
ERR_APPEND_CONFLICT = -10
NOALLOC_SCRATCH_BYTES = 16 << 20

EXPORTS = (
    "pkv_pool_create", "pkv_pool_destroy", "pkv_pool_data", "pkv_pool_num_pages", "pkv_append",
    "pkv_decode_workspace_bytes", "pkv_decode_workspace_bytes_ex", "paged_attention_decode",
    "paged_attention_decode_ex", "pkv_gather", "pkv_get_device_error", "pkv_status_string",
    "pkv_last_error_message", "pkv_pool_set_launch_flags", "paged_attention_decode_noalloc",
    "pkv_fill", "pkv_allocator_create", "pkv_allocator_destroy", "pkv_allocator_free_count",
    "pkv_allocator_alloc", "pkv_allocator_free", "paged_attention_decode_append",
    "paged_attention_decode_append_ex", "pkv_decode", "pkv_decode_params_workspace_bytes",
)


class DecodeParams(ctypes.Structure):
    """pkv_decode_params (include/pkv.h), field for field."""
    _fields_ = [
        ("struct_size", ctypes.c_size_t), ("q", ctypes.c_void_p), ("k_new", ctypes.c_void_p),
        ("v_new", ctypes.c_void_p), ("block_tables", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p), ("out", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t), ("scale", ctypes.c_float),
        ("layer", ctypes.c_int32), ("num_layers", ctypes.c_int32), ("batch", ctypes.c_int32),
        ("max_blocks", ctypes.c_int32), ("num_queries", ctypes.c_int32),
        ("out_dtype", ctypes.c_int32), ("kernel", ctypes.c_int32), ("grid_ctas", ctypes.c_int32),
        ("min_chunk", ctypes.c_int32),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libpkv.so not built at %s (run python -m "
                          "paged_attention_decode_pkv_b200.build)" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    sig = {
        "pkv_pool_create": ([i32, i32, i32, i32, P, sz, ctypes.POINTER(P)], ctypes.c_int),
        "pkv_pool_destroy": ([P], ctypes.c_int),
        "pkv_pool_data": ([P], P),
        "pkv_pool_num_pages": ([P], i32),
        "pkv_append": ([P, P, P, P, P, i32, i32, i32, i32, P], ctypes.c_int),
        "pkv_decode_workspace_bytes": ([P, i32, ctypes.POINTER(sz)], ctypes.c_int),
        "pkv_decode_workspace_bytes_ex": ([P, i32, i32, i32, ctypes.POINTER(sz)], ctypes.c_int),
        "paged_attention_decode": ([P, P, P, P, i32, ctypes.c_float, P, i32, i32, i32, P, sz, P],
                                   ctypes.c_int),
        "paged_attention_decode_ex": ([P, P, P, P, i32, ctypes.c_float, P, i32, i32, i32, P, sz,
                                       P, i32, i32, i32], ctypes.c_int),
        "pkv_gather": ([P, P, P, i32, P, P, i32, i32, i32, i32, P], ctypes.c_int),
        "pkv_get_device_error": ([P, P, ctypes.POINTER(i32)], ctypes.c_int),
        "pkv_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "pkv_last_error_message": ([], ctypes.c_char_p),
        "pkv_pool_set_launch_flags": ([P, i32], ctypes.c_int),
        "paged_attention_decode_noalloc": ([P, P, P, P, i32, ctypes.c_float, P, i32, i32, i32, P],
                                           ctypes.c_int),
        "pkv_fill": ([P, P, P, P, P, P, i32, i32, i32, i32, i32, P], ctypes.c_int),
        "paged_attention_decode_append": ([P, P, P, P, P, P, i32, ctypes.c_float, P, i32, i32,
                                           i32, P, sz, P], ctypes.c_int),
        "paged_attention_decode_append_ex": ([P, P, P, P, P, P, i32, ctypes.c_float, P, i32, i32,
                                              i32, P, sz, P, i32, i32, i32], ctypes.c_int),
        "pkv_decode": ([P, ctypes.POINTER(DecodeParams), P], ctypes.c_int),
        "pkv_decode_params_workspace_bytes": ([P, ctypes.POINTER(DecodeParams),
                                               ctypes.POINTER(sz)], ctypes.c_int),
        "pkv_allocator_create": ([i32, ctypes.POINTER(P)], ctypes.c_int),
        "pkv_allocator_destroy": ([P], ctypes.c_int),
        "pkv_allocator_free_count": ([P], i32),
        "pkv_allocator_alloc": ([P, i32, ctypes.POINTER(i32)], ctypes.c_int),
        "pkv_allocator_free": ([P, ctypes.POINTER(i32), i32], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


lib = _load()


class PkvError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        msg = lib.pkv_status_string(status).decode()
        if status == ERR_CUDA:
            msg += " [%s]" % lib.pkv_last_error_message().decode()
        super().__init__("%s%s (status %d)" % (what + ": " if what else "", msg, status))
        self.status = status


def status_string(status: int) -> str:
    return lib.pkv_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != OK:
        raise PkvError(status, what)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor, dtype, shape, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return ctypes.c_void_p(t.data_ptr())


# Pools still open.  They are closed by an exit hook that runs before the
# interpreter starts tearing modules down (and before torch's and the CUDA
# runtime's own shutdown), while the device, the library and every object
# the pool refers to are still alive; a pool that is only garbage-collected
# during interpreter shutdown makes no CUDA call at all (its device memory
# goes with the process).
_LIVE_POOLS = weakref.WeakSet()


@atexit.register
def _close_live_pools():
    for p in list(_LIVE_POOLS):
        try:
            p.close()
        except Exception:
            pass


class Pool:
    """A pool of 32 KiB pages ([K|V][8 kv heads][16 slots][64] BF16 each).

    The page storage is a torch tensor owned by this object
    (``self.storage``, bfloat16 [num_pages, 2, 8, 16, 64]) or one the caller
    passes in; the C library only borrows it.  CUDA graphs that captured
    calls on a pool hold the addresses of its storage and workspaces:
    release them before those tensors are freed.
    """

    def __init__(self, num_pages: int, storage: Optional[torch.Tensor] = None, device=None):
        if storage is None:
            storage = torch.empty((num_pages, 2, NUM_KV_HEADS, PAGE_TOKENS, HEAD_DIM),
                                  dtype=torch.bfloat16, device=device or "cuda")
        _dev(storage, torch.bfloat16, (num_pages, 2, NUM_KV_HEADS, PAGE_TOKENS, HEAD_DIM),
             "storage")
        self.storage = storage
        self.num_pages = int(num_pages)
        self.device = storage.device
        self._h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(lib.pkv_pool_create(num_pages, PAGE_TOKENS, NUM_KV_HEADS, HEAD_DIM,
                                       ctypes.c_void_p(storage.data_ptr()),
                                       storage.numel() * 2, ctypes.byref(self._h)),
                   "pkv_pool_create")
        self._ws = {}
        _LIVE_POOLS.add(self)

    @property
    def handle(self) -> ctypes.c_void_p:
        if not self._h:
            raise RuntimeError("pool destroyed")
        return self._h

    def reset_workspaces(self):
        """Zero every cached workspace."""
        for ws in self._ws.values():
            ws.zero_()

    def close(self):
        """Destroy the C pool (synchronises its device).  Idempotent."""
        if self._h:
            with torch.cuda.device(self.device):
                lib.pkv_pool_destroy(self._h)
            self._h = ctypes.c_void_p()
        self._ws.clear()
        _LIVE_POOLS.discard(self)

    def __del__(self, _finalizing=sys.is_finalizing):
        # During interpreter shutdown the CUDA runtime, torch's CUDA state or
        # this module's globals (sys included: hence the bound default) may
        # already be gone: make no device call then.
        if _finalizing():
            return
        try:
            self.close()
        except Exception:
            pass

    def set_launch_flags(self, flags: int):
        """PKV_LAUNCH_* bits for this pool's later kernel launches (see
        pkv_pool_set_launch_flags in include/pkv.h).  LAUNCH_CHECK_APPENDS
        makes append, fill and the fused calls report racing writes as
        ERR_APPEND_CONFLICT through get_device_error; setting it allocates the
        pool's slot bitmap once."""
        _check(lib.pkv_pool_set_launch_flags(self.handle, int(flags)), "pkv_pool_set_launch_flags")

    def workspace_bytes(self, batch: int, kernel: int = KERNEL_AUTO, grid_ctas: int = 0) -> int:
        n = ctypes.c_size_t()
        with torch.cuda.device(self.device):
            _check(lib.pkv_decode_workspace_bytes_ex(self.handle, int(batch), int(kernel),
                                                     int(grid_ctas), ctypes.byref(n)),
                   "pkv_decode_workspace_bytes")
        return n.value

    def workspace_bytes_for(self, batch: int, num_queries: int = 1, kernel: int = KERNEL_AUTO,
                            grid_ctas: int = 0) -> int:
        p = DecodeParams(struct_size=ctypes.sizeof(DecodeParams), batch=int(batch),
                         num_queries=int(num_queries), kernel=int(kernel),
                         grid_ctas=int(grid_ctas))
        n = ctypes.c_size_t()
        with torch.cuda.device(self.device):
            _check(lib.pkv_decode_params_workspace_bytes(self.handle, ctypes.byref(p),
                                                         ctypes.byref(n)),
                   "pkv_decode_params_workspace_bytes")
        return n.value

    def workspace(self, batch: int, kernel: int = KERNEL_AUTO, grid_ctas: int = 0,
                  num_queries: int = 1) -> torch.Tensor:
        """A decode workspace, cached per (batch, kernel, grid, queries)."""
        key = (int(batch), int(kernel), int(grid_ctas), int(num_queries))
        ws = self._ws.get(key)
        if ws is None:
            n = (self.workspace_bytes(*key[:3]) if num_queries == 1 else
                 self.workspace_bytes_for(batch, num_queries, kernel, grid_ctas))
            ws = torch.zeros(max(256, n), dtype=torch.uint8, device=self.device)
            self._ws[key] = ws
        return ws


def append(pool: Pool, block_tables: torch.Tensor, seq_lens: torch.Tensor, k_new: torch.Tensor,
           v_new: torch.Tensor, layer: int, stream=None):
    L, B, MB = block_tables.shape
    _check(lib.pkv_append(pool.handle, _dev(block_tables, torch.int32, None, "block_tables"),
                          _dev(seq_lens, torch.int32, (B,), "seq_lens"),
                          _dev(k_new, torch.bfloat16, (B, NUM_KV_HEADS, HEAD_DIM), "k_new"),
                          _dev(v_new, torch.bfloat16, (B, NUM_KV_HEADS, HEAD_DIM), "v_new"),
                          int(layer), L, B, MB, _stream(stream)), "pkv_append")


def decode(q: torch.Tensor, pool: Pool, block_tables: torch.Tensor, seq_lens: torch.Tensor,
           layer: int, scale: float, out: Optional[torch.Tensor] = None,
           workspace: Optional[torch.Tensor] = None, kernel: int = KERNEL_AUTO,
           grid_ctas: int = 0, min_chunk: int = 0, stream=None) -> torch.Tensor:
    L, B, MB = block_tables.shape
    if out is None:
        out = torch.empty((B, NUM_Q_HEADS, HEAD_DIM), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = pool.workspace(B, kernel, grid_ctas)
    _check(lib.paged_attention_decode_ex(
        _dev(q, torch.bfloat16, (B, NUM_Q_HEADS, HEAD_DIM), "q"), pool.handle,
        _dev(block_tables, torch.int32, None, "block_tables"),
        _dev(seq_lens, torch.int32, (B,), "seq_lens"), int(layer), float(scale),
        _dev(out, torch.float32, (B, NUM_Q_HEADS, HEAD_DIM), "out"), L, B, MB,
        _dev(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream),
        int(kernel), int(grid_ctas), int(min_chunk)), "paged_attention_decode")
    return out


def decode_append(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, pool: Pool,
                  block_tables: torch.Tensor, seq_lens: torch.Tensor, layer: int, scale: float,
                  out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  kernel: int = KERNEL_AUTO, grid_ctas: int = 0, min_chunk: int = 0,
                  stream=None) -> torch.Tensor:
    """append(k_new, v_new) then decode, fused into one launch
    (paged_attention_decode_append_ex)."""
    L, B, MB = block_tables.shape
    if out is None:
        out = torch.empty((B, NUM_Q_HEADS, HEAD_DIM), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = pool.workspace(B, kernel, grid_ctas)
    _check(lib.paged_attention_decode_append_ex(
        _dev(q, torch.bfloat16, (B, NUM_Q_HEADS, HEAD_DIM), "q"),
        _dev(k_new, torch.bfloat16, (B, NUM_KV_HEADS, HEAD_DIM), "k_new"),
        _dev(v_new, torch.bfloat16, (B, NUM_KV_HEADS, HEAD_DIM), "v_new"), pool.handle,
        _dev(block_tables, torch.int32, None, "block_tables"),
        _dev(seq_lens, torch.int32, (B,), "seq_lens"), int(layer), float(scale),
        _dev(out, torch.float32, (B, NUM_Q_HEADS, HEAD_DIM), "out"), L, B, MB,
        _dev(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream),
        int(kernel), int(grid_ctas), int(min_chunk)), "paged_attention_decode_append")
    return out


def decode_general(q: torch.Tensor, pool: Pool, block_tables: torch.Tensor,
                   seq_lens: torch.Tensor, layer: int, scale: float, num_queries: int = 1,
                   out_dtype=torch.float32, out: Optional[torch.Tensor] = None,
                   k_new: Optional[torch.Tensor] = None, v_new: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, kernel: int = KERNEL_AUTO,
                   grid_ctas: int = 0, min_chunk: int = 0, stream=None) -> torch.Tensor:
    """pkv_decode: q and out are [B, num_queries, 32, 64] ([B, 32, 64] when
    num_queries is 1); out_dtype torch.float32 or torch.bfloat16."""
    L, B, MB = block_tables.shape
    T = int(num_queries)
    shape = (B, NUM_Q_HEADS, HEAD_DIM) if T == 1 else (B, T, NUM_Q_HEADS, HEAD_DIM)
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out_dtype must be torch.float32 or torch.bfloat16")
    if out is None:
        out = torch.empty(shape, dtype=out_dtype, device=q.device)
    if workspace is None:
        workspace = pool.workspace(B, kernel, grid_ctas, T)
    p = DecodeParams(struct_size=ctypes.sizeof(DecodeParams))
    p.q = _dev(q, torch.bfloat16, shape, "q")
    if k_new is not None or v_new is not None:
        p.k_new = _dev(k_new, torch.bfloat16, (B, NUM_KV_HEADS, HEAD_DIM), "k_new")
        p.v_new = _dev(v_new, torch.bfloat16, (B, NUM_KV_HEADS, HEAD_DIM), "v_new")
    p.block_tables = _dev(block_tables, torch.int32, None, "block_tables")
    p.seq_lens = _dev(seq_lens, torch.int32, (B,), "seq_lens")
    p.out = _dev(out, out_dtype, shape, "out")
    p.workspace = _dev(workspace, torch.uint8, None, "workspace")
    p.workspace_bytes = workspace.numel()
    p.scale = float(scale)
    p.layer, p.num_layers, p.batch, p.max_blocks = int(layer), L, B, MB
    p.num_queries = T
    p.out_dtype = DTYPE_BF16 if out_dtype == torch.bfloat16 else DTYPE_F32
    p.kernel, p.grid_ctas, p.min_chunk = int(kernel), int(grid_ctas), int(min_chunk)
    _check(lib.pkv_decode(pool.handle, ctypes.byref(p), _stream(stream)), "pkv_decode")
    return out


def decode_noalloc(q: torch.Tensor, pool: Pool, block_tables: torch.Tensor,
                   seq_lens: torch.Tensor, layer: int, scale: float, out: torch.Tensor,
                   stream=None) -> torch.Tensor:
    """Decode through paged_attention_decode_noalloc: no workspace argument,
    nothing allocated by the library (it uses its own fixed device scratch).
    For callers that cannot allocate device memory where attention runs;
    `out` must therefore be passed in.  Calls that overlap on the GPU share
    the scratch and race."""
    L, B, MB = block_tables.shape
    _check(lib.paged_attention_decode_noalloc(
        _dev(q, torch.bfloat16, (B, NUM_Q_HEADS, HEAD_DIM), "q"), pool.handle,
        _dev(block_tables, torch.int32, None, "block_tables"),
        _dev(seq_lens, torch.int32, (B,), "seq_lens"), int(layer), float(scale),
        _dev(out, torch.float32, (B, NUM_Q_HEADS, HEAD_DIM), "out"), L, B, MB, _stream(stream)),
        "paged_attention_decode_noalloc")
    return out


def fill(pool: Pool, block_tables: torch.Tensor, cu_tokens: torch.Tensor,
         start_pos: torch.Tensor, k_src: torch.Tensor, v_src: torch.Tensor, layer: int,
         stream=None):
    """Write a ragged batch of tokens into the pages (prefill): sequence b's
    tokens k_src/v_src[cu_tokens[b]:cu_tokens[b+1]] go to positions
    start_pos[b], start_pos[b]+1, ..."""
    L, B, MB = block_tables.shape
    T = k_src.shape[0]
    _check(lib.pkv_fill(pool.handle, _dev(block_tables, torch.int32, None, "block_tables"),
                        _dev(cu_tokens, torch.int32, (B + 1,), "cu_tokens"),
                        _dev(start_pos, torch.int32, (B,), "start_pos"),
                        _dev(k_src, torch.bfloat16, (T, NUM_KV_HEADS, HEAD_DIM), "k_src"),
                        _dev(v_src, torch.bfloat16, (T, NUM_KV_HEADS, HEAD_DIM), "v_src"),
                        T, int(layer), L, B, MB, _stream(stream)), "pkv_fill")


class PageAllocator:
    """Host page allocator over page ids 0..num_pages-1 (pkv_allocator_*).

    alloc(n) returns n page ids or raises PkvError with status
    ERR_OUT_OF_PAGES (not enough free now: wait) or ERR_TOO_LARGE (more than
    the whole pool: reject); free(pages) returns them."""

    def __init__(self, num_pages: int):
        h = ctypes.c_void_p()
        _check(lib.pkv_allocator_create(int(num_pages), ctypes.byref(h)), "pkv_allocator_create")
        self.handle = h
        self.num_pages = int(num_pages)

    @property
    def free_count(self) -> int:
        return int(lib.pkv_allocator_free_count(self.handle))

    def alloc(self, count: int) -> list:
        buf = (ctypes.c_int32 * max(int(count), 1))()
        _check(lib.pkv_allocator_alloc(self.handle, int(count), buf), "pkv_allocator_alloc")
        return list(buf[:int(count)])

    def free(self, pages) -> None:
        pages = [int(p) for p in pages]
        buf = (ctypes.c_int32 * max(len(pages), 1))(*pages)
        _check(lib.pkv_allocator_free(self.handle, buf, len(pages)), "pkv_allocator_free")

    def close(self):
        if self.handle:
            lib.pkv_allocator_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def gather(pool: Pool, block_tables: torch.Tensor, seq_lens: torch.Tensor, layer: int,
           max_seq_len: int, k_out: Optional[torch.Tensor] = None,
           v_out: Optional[torch.Tensor] = None, stream=None):
    L, B, MB = block_tables.shape
    shape = (B, NUM_KV_HEADS, max_seq_len, HEAD_DIM)
    if k_out is None:
        k_out = torch.zeros(shape, dtype=torch.bfloat16, device=pool.device)
    if v_out is None:
        v_out = torch.zeros(shape, dtype=torch.bfloat16, device=pool.device)
    _check(lib.pkv_gather(pool.handle, _dev(block_tables, torch.int32, None, "block_tables"),
                          _dev(seq_lens, torch.int32, (B,), "seq_lens"), int(layer),
                          _dev(k_out, torch.bfloat16, shape, "k_out"),
                          _dev(v_out, torch.bfloat16, shape, "v_out"), L, B, MB,
                          int(max_seq_len), _stream(stream)), "pkv_gather")
    return k_out, v_out


def get_device_error(pool: Pool, stream=None) -> int:
    """Synchronise the stream; return and clear the pool's sticky device error."""
    v = ctypes.c_int32()
    _check(lib.pkv_get_device_error(pool.handle, _stream(stream), ctypes.byref(v)),
           "pkv_get_device_error")
    return v.value
