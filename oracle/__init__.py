"""Float64 CPU oracle for Dual Chunk Attention (DCA) prefill.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the CPU-baseline leg
of the benchmark are the only callers.  The product path (the CUDA library and
its Python binding) never imports this package.

The arithmetic lives in ``dca_oracle.c`` (plain C, fp64, one thread per
(row, head) work item); this module compiles it with gcc on first use and
wraps it with ctypes.  Page citations for every step are in the C file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dca_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libdca_oracle.so")
_lock = threading.Lock()
_lib = None

DT_BF16, DT_F32, DT_F64 = 0, 1, 2

# Mutation codes planted by the pin tests (mirror of the C defines).
MUTATIONS = {
    "sin_sign": 1,
    "key_not_periodic": 2,
    "query_c": 3,
    "window_le": 4,
    "pair_adjacent": 5,
    "no_mscale_sq": 6,
    "succ_as_inter": 7,
    "noncausal_diag": 8,
    "gqa_interleaved": 9,
    "theta_d": 10,
    # sparse variant
    "sp_no_dedup": 11,
    "sp_vert_acausal": 12,
    "sp_offset_off1": 13,
    "sp_no_self": 14,
}


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc -O2, pthreads)."""
    with _lock:
        if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
        ):
            tmp = _LIB_PATH + f".tmp{os.getpid()}"
            subprocess.check_call(
                ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC,
                 "-lm", "-lpthread"]
            )
            os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        i64, i32, dbl, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        lib.dca_oracle_attention_mut.argtypes = [
            vp, vp, vp, i32, i64, i64, i64, i32, i32, i32, i64, i64, i64, dbl, dbl,
            i32, i32, vp, i64, vp, i32, vp, vp, i32]
        lib.dca_oracle_attention_mut.restype = i32
        lib.dca_oracle_sparse_attention.argtypes = [
            vp, vp, vp, i32, i64, i64, i64, i32, i32, i32, i64, i64, i64, dbl, dbl,
            i32, i32, vp, vp, vp, vp, vp, i64, vp, i32, vp, vp, i32]
        lib.dca_oracle_sparse_attention.restype = i32
        lib.dca_oracle_vs_scores.argtypes = [vp, vp, i32, i64, i64, i64, i32, i32, i32, i64, i64,
                                             i64, dbl, dbl, i32, i64, i32, vp, vp, i32]
        lib.dca_oracle_vs_scores.restype = i32
        lib.dca_oracle_topk.argtypes = [vp, i64, i64, vp]
        lib.dca_oracle_topk.restype = i32
        lib.dca_oracle_position.argtypes = [i64, i64, i64, i64, i64, i32, i32,
                                            ctypes.POINTER(i64), ctypes.POINTER(i64)]
        lib.dca_oracle_position.restype = i32
        lib.dca_oracle_mscale.argtypes = [dbl]
        lib.dca_oracle_mscale.restype = dbl
        _lib = lib
    return _lib


def _as_input(x):
    """Return (contiguous numpy array, dtype code).  bf16 torch tensors are
    passed as their raw 16-bit patterns; the C side widens them exactly."""
    try:
        import torch
    except ImportError:  # pragma: no cover
        torch = None
    if torch is not None and isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy(), DT_BF16
        if x.dtype == torch.float32:
            return x.numpy(), DT_F32
        if x.dtype == torch.float64:
            return x.numpy(), DT_F64
        raise TypeError(f"unsupported dtype {x.dtype}")
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, DT_F32
    if x.dtype == np.float64:
        return x, DT_F64
    if x.dtype in (np.uint16, np.int16):
        return x, DT_BF16
    raise TypeError(f"unsupported dtype {x.dtype}")


def mscale(f: float) -> float:
    return _load().dca_oracle_mscale(float(f))


def position(i, j, s, w, c, reading=0, mutation=0):
    """(class, Pq, Pk) of the DCA position map for query i, key j <= i."""
    pq, pk = ctypes.c_int64(), ctypes.c_int64()
    cls = _load().dca_oracle_position(int(i), int(j), int(s), int(w), int(c),
                                      int(reading), int(mutation),
                                      ctypes.byref(pq), ctypes.byref(pk))
    return cls, pq.value, pk.value


def attention(q, k, v, *, chunk_size, local_window, pretrain_window,
              rope_base=1e7, yarn_scale=1.0, q_start=0, rows=None, heads=None,
              reading=0, mutation=0, n_threads=None, return_lse=False):
    """DCA attention in fp64 for the selected block rows and query heads.

    q: [Lq, Hq, d] query block (absolute row index = q_start + t);
    k, v: [Lk, Hkv, d] KV cache.  Returns out [len(rows), len(heads), d]
    (fp64 numpy) and, if requested, the natural-log LSE [len(rows), len(heads)].
    """
    qa, dt = _as_input(q)
    ka, dtk = _as_input(k)
    va, dtv = _as_input(v)
    if not (dt == dtk == dtv):
        raise TypeError("q, k, v must share a dtype")
    Lq, Hq, d = qa.shape
    Lk, Hkv, dk = ka.shape
    if va.shape != ka.shape or dk != d:
        raise ValueError("shape mismatch")
    rows = np.arange(Lq, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    heads = np.arange(Hq, dtype=np.int32) if heads is None else np.ascontiguousarray(heads, dtype=np.int32)
    out = np.zeros((len(rows), len(heads), d), dtype=np.float64)
    lse = np.zeros((len(rows), len(heads)), dtype=np.float64) if return_lse else None
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    rc = _load().dca_oracle_attention_mut(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, dt, int(q_start), Lq, Lk, Hq,
        Hkv, d, int(chunk_size), int(local_window), int(pretrain_window),
        float(rope_base), float(yarn_scale), int(reading), int(mutation),
        rows.ctypes.data, len(rows), heads.ctypes.data, len(heads), out.ctypes.data,
        lse.ctypes.data if lse is not None else None, int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle returned {rc}")
    return (out, lse) if return_lse else out


def csr(lists, Lk):
    """Per-head index lists -> (ptr int64 [H+1], idx int64), each list sorted,
    without repeats, inside [0, Lk)."""
    ptr = [0]
    flat = []
    for a in lists:
        a = np.asarray(a, dtype=np.int64).ravel()
        if a.size and (np.any(np.diff(a) <= 0) or a[0] < 0 or a[-1] >= Lk):
            raise ValueError("index lists must be sorted, unique and inside [0, Lk)")
        flat.append(a)
        ptr.append(ptr[-1] + a.size)
    idx = np.concatenate(flat) if flat else np.zeros(0, np.int64)
    return np.asarray(ptr, dtype=np.int64), np.ascontiguousarray(idx, dtype=np.int64)


def sparse_attention(q, k, v, *, vertical, slash, chunk_size, local_window, pretrain_window,
                     rope_base=1e7, yarn_scale=1.0, q_start=0, rows=None, heads=None,
                     reading=0, mutation=0, n_threads=None, return_lse=False):
    """Vertical-slash sparse DCA attention in fp64 (definition in dca_oracle.c).

    vertical[h], slash[h]: sorted key indices / diagonal offsets of query head
    h.  Row i of head h attends keys {j <= i in vertical[h]} U {i - o : o in
    slash[h], o <= i} U {i}.  Other arguments as ``attention``.
    """
    qa, dt = _as_input(q)
    ka, dtk = _as_input(k)
    va, dtv = _as_input(v)
    if not (dt == dtk == dtv):
        raise TypeError("q, k, v must share a dtype")
    Lq, Hq, d = qa.shape
    Lk, Hkv, dk = ka.shape
    if va.shape != ka.shape or dk != d or len(vertical) != Hq or len(slash) != Hq:
        raise ValueError("shape mismatch")
    v_ptr, v_idx = csr(vertical, Lk)
    s_ptr, s_off = csr(slash, Lk)
    rows = np.arange(Lq, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    heads = np.arange(Hq, dtype=np.int32) if heads is None else np.ascontiguousarray(heads, dtype=np.int32)
    out = np.zeros((len(rows), len(heads), d), dtype=np.float64)
    lse = np.zeros((len(rows), len(heads)), dtype=np.float64) if return_lse else None
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    rc = _load().dca_oracle_sparse_attention(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, dt, int(q_start), Lq, Lk, Hq, Hkv, d,
        int(chunk_size), int(local_window), int(pretrain_window), float(rope_base),
        float(yarn_scale), int(reading), int(mutation), v_ptr.ctypes.data,
        v_idx.ctypes.data if v_idx.size else None, s_ptr.ctypes.data,
        s_off.ctypes.data if s_off.size else None, rows.ctypes.data, len(rows),
        heads.ctypes.data, len(heads), out.ctypes.data,
        lse.ctypes.data if lse is not None else None, int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle returned {rc}")
    return (out, lse) if return_lse else out


def vs_scores(q, k, *, chunk_size, local_window, pretrain_window, rope_base=1e7, yarn_scale=1.0,
              q_start=0, kv_len=None, n_last=64, continuous=False, reading=0, n_threads=None):
    """Key-selection scores (definition in dca_oracle.c): vertical [Hq, Lk]
    and slash [Hq, Lk] fp64 from the last n_last rows of the query block,
    with DCA logits or (continuous=True) RoPE logits at the true positions."""
    qa, dt = _as_input(q)
    ka, dtk = _as_input(k)
    if dt != dtk:
        raise TypeError("q, k must share a dtype")
    Lq, Hq, d = qa.shape
    Lk = ka.shape[0] if kv_len is None else int(kv_len)
    vert = np.zeros((Hq, Lk), dtype=np.float64)
    slash = np.zeros((Hq, Lk), dtype=np.float64)
    rc = _load().dca_oracle_vs_scores(
        qa.ctypes.data, ka.ctypes.data, dt, int(q_start), Lq, Lk, Hq, ka.shape[1], d,
        int(chunk_size), int(local_window), int(pretrain_window), float(rope_base),
        float(yarn_scale), int(reading), int(n_last), 1 if continuous else 0, vert.ctypes.data,
        slash.ctypes.data, int(n_threads or os.cpu_count() or 1))
    if rc != 0:
        raise ValueError(f"oracle returned {rc}")
    return vert, slash


def topk(score, n):
    """The n indices of largest score (ties: smaller index), ascending."""
    score = np.ascontiguousarray(score, dtype=np.float64)
    out = np.zeros(max(1, n), dtype=np.int64)
    m = _load().dca_oracle_topk(score.ctypes.data, score.size, int(n), out.ctypes.data)
    if m != n:
        raise ValueError("bad top-k arguments")
    return out[:n]
