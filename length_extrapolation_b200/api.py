"""Python API over the C ABI of the DCA prefill library.

Argument marshalling only: torch provides device memory and the current CUDA
stream; every step of the computation runs in the library's kernels.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _native as N

_DTYPES = {torch.bfloat16: N.DCA_BF16, torch.float32: N.DCA_F32}


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype} (bfloat16 or float32)")
    return _DTYPES[t.dtype]


def _check_cuda(*ts):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors (the library has no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _stream_ptr(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


WINDOW_READINGS = {"query_offset": N.DCA_WINDOW_QUERY_OFFSET,
                   "true_distance": N.DCA_WINDOW_TRUE_DISTANCE}


def _options(window_reading):
    """dca_options for a window reading ('query_offset' (default) or 'true_distance')."""
    if window_reading not in WINDOW_READINGS:
        raise ValueError(f"window_reading must be one of {sorted(WINDOW_READINGS)}")
    o = N.DCAOptions()
    o.window_reading = WINDOW_READINGS[window_reading]
    return o


def workspace_size(kv_capacity, Hq, Hkv, d, chunk_size, local_window, pretrain_window,
                   dtype) -> int:
    code = _DTYPES[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    n = N.lib().dca_workspace_size(int(kv_capacity), int(Hq), int(Hkv), int(d), int(chunk_size),
                                   int(local_window), int(pretrain_window), code)
    if n == 0:
        raise N.DCAError(N.DCA_ERR_ARG, "dca_workspace_size")
    return n


class Workspace:
    """Caller-owned device workspace (RoPE table, rotated keys, status word).

    One workspace serves every call whose key length is <= its capacity and
    whose (Hkv, d, chunk_size, local_window, dtype) match.
    """

    def __init__(self, kv_capacity, Hq, Hkv, d, chunk_size, local_window, pretrain_window,
                 dtype, device="cuda"):
        self.nbytes = workspace_size(kv_capacity, Hq, Hkv, d, chunk_size, local_window,
                                     pretrain_window, dtype)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        self.device = self.buf.device
        N.check(N.lib().dca_workspace_init(self.buf.data_ptr(), self.nbytes,
                                           _stream_ptr(self.device)), "dca_workspace_init")

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()

    def status(self) -> int:
        """Synchronise the current stream and read/clear the device status word."""
        return N.lib().dca_device_status(self.ptr, _stream_ptr(self.device))


def _ws_for(ws: Optional[Workspace], Lk, Hq, Hkv, d, p, dtype, device) -> Workspace:
    if ws is not None:
        return ws
    return Workspace(Lk, Hq, Hkv, d, p["chunk_size"], p["local_window"], p["pretrain_window"],
                     dtype, device)


def prefill(q, k, v, *, chunk_size, local_window, pretrain_window, rope_base=1e7,
            yarn_scale=1.0, out=None, workspace: Optional[Workspace] = None,
            window_reading="query_offset"):
    """One-shot DCA prefill.  q [L,Hq,d], k, v [L,Hkv,d] (CUDA, bf16 or fp32)."""
    return prefill_chunked(q, k, v, q_start=0, chunk_size=chunk_size, local_window=local_window,
                           pretrain_window=pretrain_window, rope_base=rope_base,
                           yarn_scale=yarn_scale, out=out, workspace=workspace,
                           window_reading=window_reading)


def prefill_chunked(q_block, k_cache, v_cache, *, q_start, chunk_size, local_window,
                    pretrain_window, rope_base=1e7, yarn_scale=1.0, kv_len=None, out=None,
                    workspace: Optional[Workspace] = None, window_reading="query_offset"):
    """A query block (absolute rows q_start ..) against the KV cache rows [0, kv_len)."""
    _check_cuda(q_block, k_cache, v_cache)
    Lq, Hq, d = q_block.shape
    Lk = k_cache.shape[0] if kv_len is None else int(kv_len)
    Hkv = k_cache.shape[1]
    dt = _dtype_code(q_block)
    if not (k_cache.dtype == v_cache.dtype == q_block.dtype):
        raise TypeError("q, k, v must share a dtype")
    if out is None:
        out = torch.empty_like(q_block)
    p = dict(chunk_size=chunk_size, local_window=local_window, pretrain_window=pretrain_window)
    ws = _ws_for(workspace, Lk, Hq, Hkv, d, p, q_block.dtype, q_block.device)
    opts = _options(window_reading)
    rc = N.lib().dca_prefill_chunked_ex(
        q_block.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), out.data_ptr(), int(q_start),
        Lq, Lk, Hq, Hkv, d, int(chunk_size), int(local_window), int(pretrain_window),
        float(rope_base), float(yarn_scale), dt, ctypes.byref(opts), ws.ptr, ws.nbytes,
        _stream_ptr(q_block.device))
    N.check(rc, "dca_prefill_chunked_ex")
    return out


def prepare(k_cache, *, kv_len, k_rows_valid, chunk_size, local_window, pretrain_window,
            rope_base, workspace: Workspace):
    """Stage 1: RoPE table (when k_rows_valid == 0) and rotated keys [k_rows_valid, kv_len)."""
    _check_cuda(k_cache)
    rc = N.lib().dca_prepare(k_cache.data_ptr(), int(kv_len), int(k_rows_valid), k_cache.shape[1],
                             k_cache.shape[2], int(chunk_size), int(local_window),
                             int(pretrain_window), float(rope_base), _dtype_code(k_cache),
                             workspace.ptr, workspace.nbytes, _stream_ptr(k_cache.device))
    N.check(rc, "dca_prepare")


def attend(q_block, v_cache, out, *, q_start, kv_len, chunk_size, local_window, pretrain_window,
           yarn_scale, workspace: Workspace, window_reading="query_offset"):
    """Stage 2: the fused attention kernel over one query block."""
    _check_cuda(q_block, v_cache, out)
    Lq, Hq, d = q_block.shape
    opts = _options(window_reading)
    rc = N.lib().dca_attend_ex(q_block.data_ptr(), v_cache.data_ptr(), out.data_ptr(),
                               int(q_start), Lq, int(kv_len), Hq, v_cache.shape[1], d,
                               int(chunk_size), int(local_window), int(pretrain_window),
                               float(yarn_scale), _dtype_code(q_block), ctypes.byref(opts),
                               workspace.ptr, workspace.nbytes, _stream_ptr(q_block.device))
    N.check(rc, "dca_attend_ex")


def decode_scratch_size(Lq, Hq, Hkv) -> int:
    n = N.lib().dca_decode_scratch_size(int(Lq), int(Hq), int(Hkv))
    if n == 0:
        raise N.DCAError(N.DCA_ERR_ARG, "dca_decode_scratch_size")
    return n


def decode(q_block, v_cache, out=None, *, q_start, kv_len, chunk_size, local_window,
           pretrain_window, yarn_scale=1.0, workspace: Workspace, scratch=None, lse=None,
           window_reading="query_offset"):
    """Decode-stage attention of a few query tokens (absolute rows q_start ..,
    Lq <= DCA_DECODE_MAX_TOKENS = 256) against the rotated keys [0, kv_len)
    in `workspace` and v_cache, split over the key range and merged.  `lse`
    (optional fp32 [Lq, Hq]) receives the natural-log LSE of each row.
    Returns out [Lq, Hq, 128]."""
    _check_cuda(q_block, v_cache)
    Lq, Hq, d = q_block.shape
    if out is None:
        out = torch.empty_like(q_block)
    _check_cuda(out)
    if scratch is None:
        scratch = torch.empty(decode_scratch_size(Lq, Hq, v_cache.shape[1]), dtype=torch.uint8,
                              device=q_block.device)
    if lse is not None:
        _check_cuda(lse)
        if lse.dtype != torch.float32 or tuple(lse.shape) != (Lq, Hq):
            raise ValueError("lse must be fp32 [Lq, Hq]")
    opts = _options(window_reading)
    rc = N.lib().dca_decode(q_block.data_ptr(), v_cache.data_ptr(), out.data_ptr(),
                            lse.data_ptr() if lse is not None else None, int(q_start), Lq,
                            int(kv_len), Hq, v_cache.shape[1], d, int(chunk_size),
                            int(local_window), int(pretrain_window), float(yarn_scale),
                            _dtype_code(q_block), ctypes.byref(opts), workspace.ptr,
                            workspace.nbytes, scratch.data_ptr(), scratch.numel(),
                            _stream_ptr(q_block.device))
    N.check(rc, "dca_decode")
    return out


def decode_step(q_new, k_cache, v_cache, *, kv_len, chunk_size, local_window, pretrain_window,
                rope_base=1e7, yarn_scale=1.0, workspace: Workspace, scratch=None, out=None,
                lse=None, window_reading="query_offset"):
    """One generation step: the Lq new keys (cache rows [kv_len - Lq, kv_len))
    are rotated into the workspace, whose rows [0, kv_len - Lq) already hold
    the earlier keys, then the Lq new query tokens attend the whole cache."""
    Lq = q_new.shape[0]
    prepare(k_cache, kv_len=kv_len, k_rows_valid=kv_len - Lq, chunk_size=chunk_size,
            local_window=local_window, pretrain_window=pretrain_window, rope_base=rope_base,
            workspace=workspace)
    return decode(q_new, v_cache, out, q_start=kv_len - Lq, kv_len=kv_len, chunk_size=chunk_size,
                  local_window=local_window, pretrain_window=pretrain_window,
                  yarn_scale=yarn_scale, workspace=workspace, scratch=scratch, lse=lse,
                  window_reading=window_reading)


class SparsePattern:
    """Per-query-head vertical keys and slash offsets (host CSR arrays) for
    the vertical-slash sparse attention.  Lists are sorted, without repeats."""

    def __init__(self, vertical, slash):
        import numpy as np
        if len(vertical) != len(slash):
            raise ValueError("one vertical and one slash list per query head")
        self.Hq = len(vertical)

        def csr(lists):
            ptr = np.zeros(len(lists) + 1, dtype=np.int64)
            arrs = [np.asarray(a, dtype=np.int64).ravel() for a in lists]
            for h, a in enumerate(arrs):
                ptr[h + 1] = ptr[h] + a.size
            idx = np.concatenate(arrs).astype(np.int32) if ptr[-1] else np.zeros(1, np.int32)
            return ptr, np.ascontiguousarray(idx)

        self.v_ptr, self.v_idx = csr(vertical)
        self.s_ptr, self.s_off = csr(slash)
        self.vertical = [np.asarray(a, dtype=np.int64) for a in vertical]
        self.slash = [np.asarray(a, dtype=np.int64) for a in slash]

    def max_vertical(self):
        return int((self.v_ptr[1:] - self.v_ptr[:-1]).max())

    def max_slash(self):
        return int((self.s_ptr[1:] - self.s_ptr[:-1]).max())

    def restricted(self, Lk):
        """The pattern with vertical keys and slash offsets below Lk."""
        return SparsePattern([a[a < Lk] for a in self.vertical], [a[a < Lk] for a in self.slash])


class SparseWorkspace:
    """Device memory for the sparse index structures (bitmaps, gathered
    vertical rows); its layout is fixed by (kv_capacity, max_vertical,
    max_slash, Hq)."""

    def __init__(self, kv_capacity, Hq, max_vertical, max_slash, device="cuda"):
        self.cfg = N.DCASparseConfig(int(kv_capacity), int(max_vertical), int(max_slash))
        n = N.lib().dca_sparse_workspace_size(ctypes.byref(self.cfg), int(Hq))
        if n == 0:
            raise N.DCAError(N.DCA_ERR_ARG, "dca_sparse_workspace_size")
        # 1 KiB alignment for the gathered rows' tensor maps
        self.raw = torch.empty(n + 1024, dtype=torch.uint8, device=device)
        off = (-self.raw.data_ptr()) % 1024
        self.buf = self.raw[off:off + n]
        self.nbytes = n
        self.device = self.buf.device

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()


def sparse_prepare(pattern: SparsePattern, v_cache, *, kv_len, chunk_size, local_window,
                   pretrain_window, workspace: Workspace, sparse: SparseWorkspace):
    """Copy the pattern (restricted to keys < kv_len), build the bitmaps and
    gather the vertical rows from the rotated keys in `workspace` (which
    must hold rows [0, kv_len): call prepare first).  The lists are checked
    on the host: sorted, no repeats, at most 1023 runs of consecutive slash
    offsets per head; per-head sizes within sparse's configuration."""
    _check_cuda(v_cache)
    pat = pattern.restricted(kv_len)
    rc = N.lib().dca_sparse_prepare(
        ctypes.byref(sparse.cfg), pat.v_ptr.ctypes.data, pat.v_idx.ctypes.data,
        pat.s_ptr.ctypes.data, pat.s_off.ctypes.data, int(kv_len), pattern.Hq,
        v_cache.shape[1], v_cache.shape[2], int(chunk_size), int(local_window),
        int(pretrain_window), _dtype_code(v_cache), v_cache.data_ptr(), workspace.ptr,
        workspace.nbytes, sparse.ptr, sparse.nbytes, _stream_ptr(v_cache.device))
    N.check(rc, "dca_sparse_prepare")


def sparse_attend(q_block, v_cache, out=None, *, q_start, kv_len, chunk_size, local_window,
                  pretrain_window, yarn_scale=1.0, workspace: Workspace, sparse: SparseWorkspace,
                  window_reading="query_offset"):
    """Sparse DCA attention of a query block over the prepared structures.

    q_block [Lq, Hq, 128] bf16 holds the rows q_start .. q_start + Lq - 1;
    row i attends, per head, only its pattern's members among keys j <= i:
    the vertical keys, the keys i - o for the slash offsets o, and j = i,
    each counted once, with the DCA positions of the pair.  `sparse` must
    hold a pattern prepared (sparse_prepare) or selected (sparse_select)
    for kv_len >= q_start + Lq keys.  Returns out [Lq, Hq, 128]."""
    _check_cuda(q_block, v_cache)
    Lq, Hq, d = q_block.shape
    if out is None:
        out = torch.empty_like(q_block)
    opts = _options(window_reading)
    rc = N.lib().dca_sparse_attend(
        ctypes.byref(sparse.cfg), q_block.data_ptr(), v_cache.data_ptr(), out.data_ptr(),
        int(q_start), Lq, int(kv_len), Hq, v_cache.shape[1], d, int(chunk_size),
        int(local_window), int(pretrain_window), float(yarn_scale), _dtype_code(q_block),
        ctypes.byref(opts), workspace.ptr, workspace.nbytes, sparse.ptr, sparse.nbytes,
        _stream_ptr(q_block.device))
    N.check(rc, "dca_sparse_attend")
    return out


def sparse_select(q_block, v_cache, *, q_start, kv_len, chunk_size, local_window,
                  pretrain_window, rope_base=1e7, yarn_scale=1.0, n_vertical, n_slash,
                  n_last=64, continuous=True, workspace: Workspace, sparse: SparseWorkspace,
                  scratch=None, window_reading="query_offset"):
    """Online key selection into `sparse` from the last n_last rows of the
    block (continuous=True: true positions, the refinement; False: DCA).

    For each query head, the softmax of the last n_last (<= 64) rows over
    keys j < kv_len gives per-key column sums (vertical) and per-offset
    diagonal sums (slash); the n_vertical keys and n_slash offsets of
    largest sum (ties: the smaller index) become the head's pattern, ready
    for sparse_attend.  n_vertical <= sparse's max_vertical, n_slash <=
    max_slash and <= 1023.  bf16 only.  sparse_pattern_get reads it back."""
    _check_cuda(q_block, v_cache)
    Lq, Hq, d = q_block.shape
    if scratch is None:
        n = N.lib().dca_sparse_select_scratch_size(int(kv_len), Hq, int(chunk_size))
        if n == 0:
            raise N.DCAError(N.DCA_ERR_ARG, "dca_sparse_select_scratch_size")
        scratch = torch.empty(n, dtype=torch.uint8, device=q_block.device)
    opts = _options(window_reading)
    rc = N.lib().dca_sparse_select(
        ctypes.byref(sparse.cfg), q_block.data_ptr(), v_cache.data_ptr(), int(q_start), Lq,
        int(kv_len), Hq, v_cache.shape[1], d, int(chunk_size), int(local_window),
        int(pretrain_window), float(rope_base), float(yarn_scale), _dtype_code(q_block),
        ctypes.byref(opts), int(n_last), 1 if continuous else 0, int(n_vertical), int(n_slash),
        workspace.ptr, workspace.nbytes, sparse.ptr, sparse.nbytes, scratch.data_ptr(),
        scratch.numel(), _stream_ptr(q_block.device))
    N.check(rc, "dca_sparse_select")


def sparse_pattern_get(sparse: SparseWorkspace, Hq):
    """(vertical, slash) lists per head currently held by `sparse` (syncs)."""
    import numpy as np
    mv, ms = int(sparse.cfg.max_vertical), int(sparse.cfg.max_slash)
    vc = np.zeros(Hq, np.int32)
    sc = np.zeros(Hq, np.int32)
    vi = np.zeros(max(1, Hq * mv), np.int32)
    so = np.zeros(max(1, Hq * ms), np.int32)
    rc = N.lib().dca_sparse_pattern_get(ctypes.byref(sparse.cfg), Hq, sparse.ptr, sparse.nbytes,
                                        vc.ctypes.data, vi.ctypes.data, sc.ctypes.data,
                                        so.ctypes.data, _stream_ptr(sparse.device))
    N.check(rc, "dca_sparse_pattern_get")
    V = [vi[h * mv:h * mv + vc[h]].astype(np.int64) for h in range(Hq)]
    S = [so[h * ms:h * ms + sc[h]].astype(np.int64) for h in range(Hq)]
    return V, S


def sparse_prefill(q, k, v, pattern: SparsePattern, *, chunk_size, local_window,
                   pretrain_window, rope_base=1e7, yarn_scale=1.0, out=None,
                   window_reading="query_offset"):
    """One-shot sparse DCA prefill: rotate the keys, prepare the pattern, attend."""
    L, Hq, d = q.shape
    ws = Workspace(L, Hq, k.shape[1], d, chunk_size, local_window, pretrain_window, q.dtype,
                   q.device)
    kw = dict(chunk_size=chunk_size, local_window=local_window, pretrain_window=pretrain_window)
    prepare(k, kv_len=L, k_rows_valid=0, rope_base=rope_base, workspace=ws, **kw)
    sp = SparseWorkspace(L, Hq, max(1, pattern.max_vertical()), max(1, pattern.max_slash()),
                         q.device)
    sparse_prepare(pattern, v, kv_len=L, workspace=ws, sparse=sp, **kw)
    return sparse_attend(q, v, out, q_start=0, kv_len=L, yarn_scale=yarn_scale, workspace=ws,
                         sparse=sp, window_reading=window_reading, **kw)


def host_arena_size(L, block, Hq, Hkv, d, chunk_size, local_window, pretrain_window, dtype):
    code = _DTYPES[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    n = N.lib().dca_host_arena_size(int(L), int(block), int(Hq), int(Hkv), int(d),
                                    int(chunk_size), int(local_window), int(pretrain_window), code)
    if n == 0:
        raise N.DCAError(N.DCA_ERR_ARG, "dca_host_arena_size")
    return n


def prefill_host(q_h, k_h, v_h, out_h, *, block, chunk_size, local_window, pretrain_window,
                 rope_base=1e7, yarn_scale=1.0, arena: torch.Tensor, stream=None):
    """Whole prefill from host (CPU, ideally pinned) tensors through the C ABI."""
    for t in (q_h, k_h, v_h, out_h):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host tensors must be contiguous CPU tensors")
    L, Hq, d = q_h.shape
    Hkv = k_h.shape[1]
    st = (stream or torch.cuda.current_stream(arena.device)).cuda_stream
    rc = N.lib().dca_prefill_host(q_h.data_ptr(), k_h.data_ptr(), v_h.data_ptr(), out_h.data_ptr(),
                                  L, int(block), Hq, Hkv, d, int(chunk_size), int(local_window),
                                  int(pretrain_window), float(rope_base), float(yarn_scale),
                                  _dtype_code(q_h), arena.data_ptr(), arena.numel(), st)
    N.check(rc, "dca_prefill_host")


def set_wait_timeout_ns(ns: int):
    N.lib().dca_set_wait_timeout_ns(int(ns))


def set_debug_flags(flags: int):
    N.lib().dca_set_debug_flags(int(flags))
