"""ctypes loader for the in-tree CUDA library (libdca_b200.so).

The library must exist: there is no fallback.  Build it with
``python -m length_extrapolation_b200.build`` (``__graft_entry__.build()``
does the same).
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdca_b200.so")

DCA_BF16, DCA_F32 = 0, 1
DCA_WINDOW_QUERY_OFFSET, DCA_WINDOW_TRUE_DISTANCE = 0, 1
DCA_OK, DCA_ERR_ARG, DCA_ERR_UNSUPPORTED, DCA_ERR_CUDA, DCA_ERR_WORKSPACE, DCA_ERR_TIMEOUT = (
    0, -1, -2, -3, -4, -5)

# (name, restype, argtypes) for every symbol declared in include/dca.h
_i64, _i32, _dbl, _vp, _sz = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p, ctypes.c_size_t
SIGNATURES = {
    "dca_version": (_i32, []),
    "dca_status_string": (ctypes.c_char_p, [_i32]),
    "dca_workspace_size": (_sz, [_i64, _i32, _i32, _i32, _i64, _i64, _i64, _i32]),
    "dca_workspace_init": (_i32, [_vp, _sz, _vp]),
    "dca_prefill": (_i32, [_vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _i64, _i64, _i64, _dbl,
                           _dbl, _i32, _vp, _sz, _vp]),
    "dca_prefill_chunked": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _i64,
                                   _i64, _i64, _dbl, _dbl, _i32, _vp, _sz, _vp]),
    "dca_prepare": (_i32, [_vp, _i64, _i64, _i32, _i32, _i64, _i64, _i64, _dbl, _i32, _vp, _sz,
                           _vp]),
    "dca_attend": (_i32, [_vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _i64, _i64, _i64,
                          _dbl, _i32, _vp, _sz, _vp]),
    "dca_device_status": (_i32, [_vp, _vp]),
    "dca_host_arena_size": (_sz, [_i64, _i64, _i32, _i32, _i32, _i64, _i64, _i64, _i32]),
    "dca_prefill_host": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i32, _i32, _i32, _i64, _i64,
                                _i64, _dbl, _dbl, _i32, _vp, _sz, _vp]),
    "dca_plan_items": (_i32, [_i64, _i64, _i64, _i64, _i64, _i32, _i32, _vp, _i32]),
    "dca_class_rows": (_i32, [_i64, _i64, _i32, _i64, _i64, _i64, _i32, _i32, _i64, _vp]),
    "dca_prefill_chunked_ex": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _i64,
                                      _i64, _i64, _dbl, _dbl, _i32, _vp, _vp, _sz, _vp]),
    "dca_attend_ex": (_i32, [_vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _i64, _i64, _i64,
                             _dbl, _i32, _vp, _vp, _sz, _vp]),
    "dca_prefill_noalloc": (_i32, [_vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _i64, _i64, _i64,
                                   _dbl, _dbl, _i32, _vp]),
    "dca_row_keys": (_i32, [_i64, _i32, _i64, _i64, _i32, _vp]),
    "dca_noalloc_prepare": (_i32, []),
    "dca_noalloc_device_status": (_i32, [_vp]),
    "dca_decode_scratch_size": (_sz, [_i64, _i32, _i32]),
    "dca_decode": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _i64, _i64,
                          _i64, _dbl, _i32, _vp, _vp, _sz, _vp, _sz, _vp]),
    "dca_sparse_workspace_size": (_sz, [_vp, _i32]),
    "dca_sparse_prepare": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _i64, _i64,
                                  _i64, _i32, _vp, _vp, _sz, _vp, _sz, _vp]),
    "dca_sparse_attend": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _i64,
                                 _i64, _i64, _dbl, _i32, _vp, _vp, _sz, _vp, _sz, _vp]),
    "dca_sparse_plan_items": (_i32, [_vp, _i64, _vp, _i64, _i64, _i64, _i64, _i64, _i32, _vp,
                                     _i32]),
    "dca_sparse_select_scratch_size": (_sz, [_i64, _i32, _i64]),
    "dca_sparse_select": (_i32, [_vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _i64, _i64,
                                 _i64, _dbl, _dbl, _i32, _vp, _i32, _i32, _i64, _i64, _vp, _sz,
                                 _vp, _sz, _vp, _sz, _vp]),
    "dca_sparse_pattern_get": (_i32, [_vp, _i32, _vp, _sz, _vp, _vp, _vp, _vp, _vp]),
    "dca_set_wait_timeout_ns": (None, [_i64]),
    "dca_set_debug_flags": (None, [_i32]),
}

_lock = threading.Lock()
_lib = None


DCA_DECODE_MAX_TOKENS = 256


DCA_SPARSE_MAX_RUNS = 1023


class DCASparseConfig(ctypes.Structure):
    """Mirror of dca_sparse_config (include/dca.h)."""
    _fields_ = [("kv_capacity", ctypes.c_int64), ("max_vertical", ctypes.c_int64),
                ("max_slash", ctypes.c_int64)]


class DCAOptions(ctypes.Structure):
    """Mirror of dca_options (include/dca.h)."""
    _fields_ = [("window_reading", ctypes.c_int32), ("reserved", ctypes.c_int32 * 7)]


class DCAError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})" if what else status_string(status))


def lib():
    """Load libdca_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"CUDA library missing: {LIB_PATH}; run "
                        "`python -m length_extrapolation_b200.build` (there is no CPU fallback)")
                L = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in SIGNATURES.items():
                    fn = getattr(L, name)
                    fn.restype = res
                    fn.argtypes = args
                _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().dca_status_string(int(status)).decode()


def check(status: int, what: str = ""):
    if status != DCA_OK:
        raise DCAError(status, what)
