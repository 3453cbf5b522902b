"""B200-native (sm_100a) Dual Chunk Attention prefill.

The compute path is the CUDA library ``libdca_b200.so`` (C ABI in
``include/dca.h``); this package is its Python binding.  Importing the package
does not load the library; the first call does, and fails loudly if it was not
built.
"""
from .api import (  # noqa: F401
    SparsePattern,
    SparseWorkspace,
    Workspace,
    attend,
    decode,
    decode_scratch_size,
    decode_step,
    host_arena_size,
    prefill,
    prefill_chunked,
    prefill_host,
    prepare,
    set_debug_flags,
    sparse_attend,
    sparse_pattern_get,
    sparse_prefill,
    sparse_prepare,
    sparse_select,
    set_wait_timeout_ns,
    workspace_size,
)

__all__ = [
    "SparsePattern", "SparseWorkspace", "Workspace", "attend", "decode", "decode_scratch_size", "decode_step", "host_arena_size", "prefill", "prefill_chunked", "prefill_host",
    "prepare", "set_debug_flags", "set_wait_timeout_ns", "sparse_attend", "sparse_pattern_get", "sparse_prefill",
    "sparse_prepare", "sparse_select",
    "workspace_size",
]
