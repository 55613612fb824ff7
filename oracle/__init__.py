"""FP64 CPU oracle for paged decode attention (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
binding) never does.
"""
from .oracle import (append, append_conflict, fill, fill_conflict, gather, decode,  # noqa: F401
                     decode_multi, OracleError)
