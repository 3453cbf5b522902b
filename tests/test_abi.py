"""The C ABI library loads on a machine without a GPU, exports every symbol
declared in include/dca.h, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import os
import re

import pytest

from length_extrapolation_b200 import _native as N
from length_extrapolation_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return N.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "dca.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dca_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
        assert n in N.SIGNATURES, f"{n} has no Python signature"


def test_version_and_status_strings(lib):
    assert lib.dca_version() >= 100
    for st in (0, -1, -2, -3, -4, -5):
        assert N.status_string(st).startswith("DCA_")
    assert "unknown" in N.status_string(42)


BASE = dict(Hq=28, Hkv=4, d=128, s=8192, w=1024, c=16384, dtype=0)


def ws_size(L, **kw):
    a = {**BASE, **kw}
    return N.lib().dca_workspace_size(L, a["Hq"], a["Hkv"], a["d"], a["s"], a["w"], a["c"],
                                      a["dtype"])


def test_workspace_size_layout(lib):
    # header + table (s + w + 1 rows of 64 (cos, sin) fp32) + rotated keys (L*Hkv*128 bf16)
    L = 32768
    table = (8192 + 1024 + 1) * 64 * 8
    keys = L * 4 * 128 * 2
    n = ws_size(L)
    assert n >= 1024 + table + keys
    assert n <= 1024 + table + keys + 3 * 1024
    assert ws_size(L, dtype=1) > n                     # fp32 keys are twice as large
    assert ws_size(100, s=1 << 40, w=0, c=1) > 0        # chunk_size beyond L: table sized by L
    assert ws_size(100, s=1 << 40, w=0, c=1) < 1024 + 102 * 512 + 100 * 4 * 256 + 4096


@pytest.mark.parametrize("bad", [dict(Hq=30), dict(Hkv=0), dict(d=127), dict(s=0), dict(w=-1),
                                 dict(w=9000), dict(c=0), dict(dtype=7)])
def test_workspace_size_rejects(lib, bad):
    assert ws_size(1024, **bad) == 0


def _prefill(lib, L=256, Hq=4, Hkv=2, d=128, s=64, w=16, c=128, base=1e7, yarn=1.0, dtype=0,
             ptr=1 << 20, ws=None, ws_bytes=None, q_ptr=None):
    if ws_bytes is None:
        ws_bytes = lib.dca_workspace_size(L, Hq, Hkv, 128, s, max(0, min(w, s)), max(c, 1), 0) or 1 << 30
    q = ptr if q_ptr is None else q_ptr
    return lib.dca_prefill(q, ptr, ptr, ptr, L, Hq, Hkv, d, s, w, c, base, yarn, dtype,
                           ptr if ws is None else ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=5, Hkv=2), N.DCA_ERR_ARG),          # Hq % Hkv
    (dict(w=65), N.DCA_ERR_ARG),                 # w > s
    (dict(w=-1), N.DCA_ERR_ARG),
    (dict(s=0), N.DCA_ERR_ARG),
    (dict(c=70), N.DCA_ERR_ARG),                 # L > s and s + w > c
    (dict(yarn=0.0), N.DCA_ERR_ARG),
    (dict(yarn=float("nan")), N.DCA_ERR_ARG),
    (dict(base=-1.0), N.DCA_ERR_ARG),
    (dict(dtype=3), N.DCA_ERR_ARG),
    (dict(d=64), N.DCA_ERR_UNSUPPORTED),
    (dict(ws=0), N.DCA_ERR_WORKSPACE),
    (dict(ws=(1 << 20) + 16), N.DCA_ERR_WORKSPACE),   # not 256-byte aligned
    (dict(ws_bytes=1000), N.DCA_ERR_WORKSPACE),       # too small
    (dict(q_ptr=(1 << 20) + 2), N.DCA_ERR_ARG),       # misaligned tensor
    (dict(q_ptr=0), N.DCA_ERR_ARG),                   # null tensor
])
def test_prefill_rejects_before_launch(lib, kw, status):
    assert _prefill(lib, **kw) == status


def test_chunked_rejects_bad_ranges(lib):
    ws = lib.dca_workspace_size(512, 4, 2, 128, 64, 16, 128, 0)
    p = 1 << 20
    call = lambda q0, lq, lk: lib.dca_prefill_chunked(p, p, p, p, q0, lq, lk, 4, 2, 128, 64, 16,
                                                      128, 1e7, 1.0, 0, p, ws, None)
    assert call(-1, 10, 100) == N.DCA_ERR_ARG
    assert call(0, -1, 100) == N.DCA_ERR_ARG
    assert call(95, 10, 100) == N.DCA_ERR_ARG      # q_start + Lq > Lk
    assert call(0, 10, 600) == N.DCA_ERR_WORKSPACE  # Lk beyond the workspace capacity
    assert call(5, 0, 100) == N.DCA_OK              # empty block: nothing to do, no launch


def test_prepare_attend_reject(lib):
    p = 1 << 20
    ws = lib.dca_workspace_size(512, 4, 2, 128, 64, 16, 128, 0)
    assert lib.dca_prepare(p, 100, 101, 2, 128, 64, 16, 128, 1e7, 0, p, ws, None) == N.DCA_ERR_ARG
    assert lib.dca_prepare(p, 100, -1, 2, 128, 64, 16, 128, 1e7, 0, p, ws, None) == N.DCA_ERR_ARG
    assert lib.dca_prepare(0, 100, 0, 2, 128, 64, 16, 128, 1e7, 0, p, ws, None) == N.DCA_ERR_ARG
    assert lib.dca_attend(p, p, p, 0, 10, 5, 4, 2, 128, 64, 16, 128, 1.0, 0, p, ws, None) == N.DCA_ERR_ARG
    assert lib.dca_attend(p, p, p, 0, 0, 5, 4, 2, 128, 64, 16, 128, 1.0, 0, p, ws, None) == N.DCA_OK


def test_window_reading_options(lib):
    """dca_options: an unknown reading or a non-zero reserved field is an
    argument error, found before any launch; NULL selects the default."""
    import ctypes
    p = 1 << 20
    ws = lib.dca_workspace_size(512, 4, 2, 128, 64, 16, 128, 0)

    def chunked(opts, lq=10):
        return lib.dca_prefill_chunked_ex(p, p, p, p, 0, lq, 100, 4, 2, 128, 64, 16, 128, 1e7,
                                          1.0, 0, opts, p, ws, None)

    def attend(opts, lq=10):
        return lib.dca_attend_ex(p, p, p, 0, lq, 100, 4, 2, 128, 64, 16, 128, 1.0, 0, opts, p,
                                 ws, None)

    for bad_reading, bad_reserved in [(2, 0), (-1, 0), (0, 1), (1, 7)]:
        o = N.DCAOptions()
        o.window_reading = bad_reading
        o.reserved[3] = bad_reserved
        assert chunked(ctypes.byref(o)) == N.DCA_ERR_ARG
        assert attend(ctypes.byref(o)) == N.DCA_ERR_ARG
    for reading in (N.DCA_WINDOW_QUERY_OFFSET, N.DCA_WINDOW_TRUE_DISTANCE):
        o = N.DCAOptions()
        o.window_reading = reading
        assert chunked(ctypes.byref(o), lq=0) == N.DCA_OK   # empty block: valid, no launch
        assert attend(ctypes.byref(o), lq=0) == N.DCA_OK
    assert chunked(None, lq=0) == N.DCA_OK
    assert ctypes.sizeof(N.DCAOptions) == 32


def test_python_api_rejects_unknown_window_reading():
    from length_extrapolation_b200 import api
    with pytest.raises(ValueError):
        api._options("window")
    assert api._options("true_distance").window_reading == N.DCA_WINDOW_TRUE_DISTANCE


def test_host_entry_rejects(lib):
    need = lib.dca_host_arena_size(1000, 256, 4, 2, 128, 64, 16, 128, 0)
    assert need > lib.dca_workspace_size(1000, 4, 2, 128, 64, 16, 128, 0)
    p = 1 << 20
    assert lib.dca_prefill_host(p, p, p, p, 1000, 256, 4, 2, 128, 64, 16, 128, 1e7, 1.0, 0,
                                p, need - 1, None) == N.DCA_ERR_WORKSPACE
    assert lib.dca_prefill_host(0, p, p, p, 1000, 256, 4, 2, 128, 64, 16, 128, 1e7, 1.0, 0,
                                p, need, None) == N.DCA_ERR_ARG
    assert lib.dca_host_arena_size(1000, 256, 4, 3, 128, 64, 16, 128, 0) == 0


def test_python_api_refuses_cpu_tensors():
    import torch

    import length_extrapolation_b200 as dca
    q = torch.zeros(8, 2, 128, dtype=torch.bfloat16)
    k = torch.zeros(8, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        dca.prefill(q, k, k, chunk_size=4, local_window=1, pretrain_window=8)
