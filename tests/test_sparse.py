"""Vertical-slash sparse DCA: work-list coverage (CPU), argument checks (CPU)
and parity of the CUDA path with the oracle's sparse variant (GPU).

Row i of query head h attends M_h(i) = {j <= i in V_h} U {i - o : o in S_h,
o <= i} U {i}.  The kernel visits 128-key items (vertical tiles of the
gathered keys, cache tiles crossed by slash diagonals) class by class and
masks each to its class and its members; the CPU test checks on the host
copy of the same plan that every member pair is visited exactly once.
"""
import ctypes
from collections import defaultdict

import numpy as np
import pytest
import torch

import oracle
import length_extrapolation_b200 as dca
from length_extrapolation_b200 import _native as N
from length_extrapolation_b200.workloads import Workload, generate, sparse_pattern


@pytest.fixture(scope="module")
def lib():
    from length_extrapolation_b200 import build as B
    B.build()
    return N.lib()


def plan(lib, V, S, i0, i_last, s, w, reading):
    va = np.ascontiguousarray(V, dtype=np.int32)
    sa = np.ascontiguousarray(S, dtype=np.int32)
    buf = (ctypes.c_int32 * (3 * 20000))()
    n = lib.dca_sparse_plan_items(va.ctypes.data if va.size else None, va.size,
                                  sa.ctypes.data if sa.size else None, sa.size, i0, i_last, s, w,
                                  reading, buf, 20000)
    assert 0 <= n <= 20000, n
    return [(buf[3 * k], buf[3 * k + 1], buf[3 * k + 2]) for k in range(n)]


def check_cover(lib, V, S, i0, i_last, s, w, reading):
    items = plan(lib, V, S, i0, i_last, s, w, reading)
    Vset, Sset = set(int(x) for x in V), set(int(x) for x in S)

    def klass(i, j):
        """Work-list class: 0 intra, 1 adjacent chunks with the true distance
        kept (every adjacent-chunk pair under the query-offset reading, the
        row choosing s + r_i or c - 1), 2 the inter-chunk rule."""
        dn = i // s - j // s
        if dn <= 0:
            return 0
        if dn == 1 and (reading == 0 or i - j < w):
            return 1
        return 2

    count = defaultdict(int)
    for src, start, cls in items:
        if src == 0:
            assert start % 128 == 0 and 0 <= start < len(V), (start, len(V))
            keys = [int(x) for x in V[start:start + 128]]
            for i in range(i0, i_last + 1):
                for j in keys:
                    if j <= i and klass(i, j) == cls:
                        count[(i, j)] += 1
        else:
            assert 0 <= start <= i_last
            for i in range(i0, i_last + 1):
                for j in range(start, start + 128):
                    if j > i or j in Vset:
                        continue
                    if (i - j) not in Sset and j != i:
                        continue
                    if klass(i, j) == cls:
                        count[(i, j)] += 1
    for i in range(i0, i_last + 1):
        mem = {j for j in Vset if j <= i} | {i - o for o in Sset if o <= i} | {i}
        for j in mem:
            assert count[(i, j)] == 1, (i, j, count[(i, j)])
        extra = [j for (ii, j) in count if ii == i and j not in mem]
        assert not extra, (i, extra[:5])
    return items


# ------------------------------------------------------------------ CPU

CASES = [  # L, s, w, n_vertical, n_band, n_far
    (1500, 256, 64, 40, 16, 12),
    (1300, 200, 50, 300, 5, 30),     # verticals span several gathered tiles
    (900, 3, 2, 20, 4, 10),          # tiny chunks: every tile mixes classes
    (1100, 512, 0, 10, 1, 0),        # w = 0, self + offset 0 only on the slash side
    (700, 128, 128, 0, 300, 0),      # band only: dense near the diagonal
]


@pytest.mark.parametrize("reading", [0, 1], ids=["query_offset", "true_distance"])
@pytest.mark.parametrize("L,s,w,nv,nb,nf", CASES)
def test_plan_covers_every_member_once(lib, L, s, w, nv, nb, nf, reading):
    V, S = sparse_pattern(L, 1, nv, nb, nf, seed=L + s)
    rng = np.random.default_rng(7)
    tiles = sorted({0, (L - 1) // 128, *rng.integers(0, (L + 127) // 128, 3).tolist()})
    for t in tiles:
        i0 = 128 * t
        i_last = min(i0 + 127, L - 1)
        check_cover(lib, V[0], S[0], i0, i_last, s, w, reading)


@pytest.mark.parametrize("reading", [0, 1])
def test_plan_windows_near_each_other(lib, reading):
    """Far diagonals 100, 129 and 130 keys apart: windows that start at a
    range's first key may run past its end but never into the next range."""
    S = [0, 1, 2, 3, 300, 400, 529, 530, 659, 789, 1000]
    V = [5, 77, 640, 641]
    for i0 in (896, 1024, 1152):
        check_cover(lib, V, S, i0, i0 + 127, 512, 64, reading)


def test_plan_empty_pattern_is_the_diagonal(lib):
    items = check_cover(lib, [], [], 256, 383, 100, 10, 0)
    assert all(src == 1 for src, _, _ in items)


def test_sparse_abi_rejects(lib):
    cfg = N.DCASparseConfig(1000, 16, 16)
    n = lib.dca_sparse_workspace_size(ctypes.byref(cfg), 4)
    assert n > 0
    assert lib.dca_sparse_workspace_size(None, 4) == 0
    assert lib.dca_sparse_workspace_size(ctypes.byref(N.DCASparseConfig(0, 1, 1)), 4) == 0
    p = 1 << 20
    ws = lib.dca_workspace_size(2000, 4, 2, 128, 64, 16, 128, 0)  # dense capacity above cfg's

    def prep(v, s, cfg=cfg, Lk=1000, dtype=0, sbytes=n, sws=p):
        vp = np.array([0] + list(np.cumsum([len(a) for a in v])), dtype=np.int64)
        sp = np.array([0] + list(np.cumsum([len(a) for a in s])), dtype=np.int64)
        vi = np.array([x for a in v for x in a] or [0], dtype=np.int32)
        so = np.array([x for a in s for x in a] or [0], dtype=np.int32)
        return lib.dca_sparse_prepare(ctypes.byref(cfg), vp.ctypes.data, vi.ctypes.data,
                                      sp.ctypes.data, so.ctypes.data, Lk, 4, 2, 128, 64, 16, 128,
                                      dtype, p, p, ws, sws, sbytes, None)

    ok = [[1, 5]] * 4
    assert prep([[5, 1]] + ok[1:], ok) == N.DCA_ERR_ARG          # unsorted
    assert prep([[1, 1]] + ok[1:], ok) == N.DCA_ERR_ARG          # repeat
    assert prep(ok, [[1000]] + ok[1:]) == N.DCA_ERR_ARG          # outside [0, Lk)
    assert prep([list(range(17))] + ok[1:], ok) == N.DCA_ERR_ARG  # more than max_vertical
    assert prep(ok, ok, Lk=1001) == N.DCA_ERR_ARG                # Lk beyond the capacity
    assert prep(ok, ok, dtype=1) == N.DCA_ERR_UNSUPPORTED        # fp32
    assert prep(ok, ok, sbytes=n - 1) == N.DCA_ERR_WORKSPACE
    assert prep(ok, ok, sws=p + 256) == N.DCA_ERR_WORKSPACE       # not 1 KiB aligned
    many = N.DCASparseConfig(5000, 16, 4000)
    runs = [list(range(0, 2 * 1030, 2))] + [[1]] * 3             # 1030 runs > DCA_SPARSE_MAX_RUNS
    n2 = lib.dca_sparse_workspace_size(ctypes.byref(many), 4)
    ws2 = lib.dca_workspace_size(5000, 4, 2, 128, 64, 16, 128, 0)
    vp = np.zeros(5, np.int64)
    sp = np.array([0, 1030, 1031, 1032, 1033], np.int64)
    so = np.array(runs[0] + [1, 1, 1], np.int32)
    assert lib.dca_sparse_prepare(ctypes.byref(many), vp.ctypes.data, None, sp.ctypes.data,
                                  so.ctypes.data, 5000, 4, 2, 128, 64, 16, 128, 0, p, p, ws2, p,
                                  n2, None) == N.DCA_ERR_ARG
    # attend: fp32 unsupported, bad options, Lq = 0 is a no-op
    o = N.DCAOptions()
    o.window_reading = 9
    att = lambda lq=10, dtype=0, opts=None: lib.dca_sparse_attend(
        ctypes.byref(cfg), p, p, p, 0, lq, 100, 4, 2, 128, 64, 16, 128, 1.0, dtype, opts, p, ws,
        p, n, None)
    assert att(dtype=1) == N.DCA_ERR_UNSUPPORTED
    assert att(opts=ctypes.byref(o)) == N.DCA_ERR_ARG
    assert att(lq=0) == N.DCA_OK


# ------------------------------------------------------------------ GPU

DEV = "cuda:0"


def wl(name, L, Hq, Hkv, s, w, c, yarn=1.0, sqrt_d=True):
    return Workload(name, L=L, Hq=Hq, Hkv=Hkv, d=128, dtype="bf16", chunk_size=s,
                    local_window=w, pretrain_window=c, yarn_scale=yarn, scale_by_sqrt_d=sqrt_d)


GPU_CASES = [  # workload, (n_vertical, n_band, n_far)
    (wl("sp_mixed", 1500, 4, 1, 300, 50, 400), (60, 64, 20)),
    (wl("sp_g7_yarn", 2100, 7, 1, 512, 128, 1024, yarn=4.0), (200, 256, 40)),
    (wl("sp_vert_heavy", 1300, 4, 2, 256, 32, 512, sqrt_d=False), (500, 8, 4)),
    (wl("sp_slash_far", 1700, 2, 1, 384, 100, 640, sqrt_d=False), (4, 32, 300)),
    (wl("sp_tiny_chunks", 600, 2, 1, 3, 2, 5), (30, 5, 10)),
    (wl("sp_self_only", 500, 2, 2, 128, 16, 256), (0, 0, 0)),
]


def run_sparse(w, pat, seed=0, reading="query_offset"):
    q, k, v = generate(w, device=DEV, seed=seed)
    V, S = pat
    out = dca.sparse_prefill(q, k, v, dca.SparsePattern(V, S), window_reading=reading,
                             **w.params())
    torch.cuda.synchronize()
    return q, k, v, out


@pytest.mark.gpu
@pytest.mark.parametrize("reading", [0, 1], ids=["query_offset", "true_distance"])
@pytest.mark.parametrize("w,sizes", GPU_CASES, ids=lambda x: x.name if hasattr(x, "name") else "")
def test_sparse_parity(w, sizes, reading):
    from tests.gpu_helpers import assert_close
    pat = sparse_pattern(w.L, w.Hq, *sizes, seed=11)
    q, k, v, out = run_sparse(w, pat, reading=["query_offset", "true_distance"][reading])
    want = oracle.sparse_attention(q.cpu(), k.cpu(), v.cpu(), vertical=pat[0], slash=pat[1],
                                   reading=reading, **w.params())
    assert_close(out.double().cpu().numpy(), want, torch.bfloat16, w.name)


def _sparse_staged(w, pat, q, k, v):
    kw = dict(chunk_size=w.chunk_size, local_window=w.local_window,
              pretrain_window=w.pretrain_window)
    ws = dca.Workspace(w.L, w.Hq, w.Hkv, 128, w.chunk_size, w.local_window, w.pretrain_window,
                       q.dtype, DEV)
    sp = dca.SparseWorkspace(w.L, w.Hq, pat.max_vertical(), pat.max_slash(), DEV)
    dca.prepare(k, kv_len=w.L, k_rows_valid=0, rope_base=w.rope_base, workspace=ws, **kw)
    dca.sparse_prepare(pat, v, kv_len=w.L, workspace=ws, sparse=sp, **kw)

    def attend(out):
        dca.sparse_attend(q, v, out, q_start=0, kv_len=w.L, yarn_scale=w.yarn_scale,
                          workspace=ws, sparse=sp, **kw)
        return ws.status()
    return attend


@pytest.mark.gpu
def test_sparse_bounded_wait_timeout_reports_and_recovers():
    """Withhold the first key tile (flag 1): the waits of every role of that
    CTA run out after the short limit, the CTA drains its copies and MMAs
    and exits, the status word reports the timeout, and the next launch on
    the same workspace is correct."""
    from tests.gpu_helpers import assert_close
    w = wl("sp_timeout", 1100, 4, 2, 256, 64, 512)
    V, S = sparse_pattern(w.L, w.Hq, 60, 32, 12, seed=5)
    pat = dca.SparsePattern(V, S)
    q, k, v = generate(w, device=DEV, seed=2)
    attend = _sparse_staged(w, pat, q, k, v)
    out = torch.zeros_like(q)
    dca.set_wait_timeout_ns(20_000_000)
    try:
        dca.set_debug_flags(1)
        assert attend(out) == N.DCA_ERR_TIMEOUT
    finally:
        dca.set_debug_flags(0)
        dca.set_wait_timeout_ns(0)
    out2 = torch.empty_like(q)
    assert attend(out2) == N.DCA_OK
    want = oracle.sparse_attention(q.cpu(), k.cpu(), v.cpu(), vertical=V, slash=S, **w.params())
    assert_close(out2.double().cpu().numpy(), want, torch.bfloat16, "after timeout")


@pytest.mark.gpu
def test_sparse_all_offsets_equals_dense():
    """Every offset selected: the sparse path computes dense DCA attention."""
    from tests.gpu_helpers import assert_close
    w = wl("sp_dense", 1200, 4, 2, 256, 64, 512)
    pat = ([np.arange(0)] * w.Hq, [np.arange(w.L)] * w.Hq)
    q, k, v, out = run_sparse(w, pat)
    dense = dca.prefill(q, k, v, **w.params())
    torch.cuda.synchronize()
    assert_close(out.double().cpu().numpy(), dense.double().cpu().numpy(), torch.bfloat16)


@pytest.mark.gpu
def test_sparse_chunked_blocks():
    """Chunked prefill: per block, the pattern restricted to the cache."""
    from tests.gpu_helpers import assert_close
    w = wl("sp_chunked", 1536, 4, 2, 256, 64, 512)
    V, S = sparse_pattern(w.L, w.Hq, 80, 64, 16, seed=3)
    pat = dca.SparsePattern(V, S)
    q, k, v = generate(w, device=DEV, seed=1)
    kw = dict(chunk_size=w.chunk_size, local_window=w.local_window,
              pretrain_window=w.pretrain_window)
    ws = dca.Workspace(w.L, w.Hq, w.Hkv, 128, w.chunk_size, w.local_window, w.pretrain_window,
                       q.dtype, DEV)
    sp = dca.SparseWorkspace(w.L, w.Hq, pat.max_vertical(), pat.max_slash(), DEV)
    out = torch.empty_like(q)
    for q0 in range(0, w.L, 512):
        lk = q0 + 512
        dca.prepare(k, kv_len=lk, k_rows_valid=q0, rope_base=w.rope_base, workspace=ws, **kw)
        dca.sparse_prepare(pat, v, kv_len=lk, workspace=ws, sparse=sp, **kw)
        dca.sparse_attend(q[q0:lk], v, out[q0:lk], q_start=q0, kv_len=lk,
                          yarn_scale=w.yarn_scale, workspace=ws, sparse=sp, **kw)
    torch.cuda.synchronize()
    assert ws.status() == N.DCA_OK
    want = oracle.sparse_attention(q.cpu(), k.cpu(), v.cpu(), vertical=V, slash=S, **w.params())
    assert_close(out.double().cpu().numpy(), want, torch.bfloat16, "chunked")


@pytest.mark.gpu
def test_sparse_full_size_1m_sampled():
    """1M tokens, the 7B DCA parameters, the sparse benchmark's pattern:
    sampled rows and heads against the oracle (each row costs the oracle only
    its member keys)."""
    from length_extrapolation_b200.workloads import SPARSE_WORKLOADS, generate_sparse, sample_heads
    from tests.gpu_helpers import assert_close, gather
    sw = SPARSE_WORKLOADS["qwen7b_1m_sparse"]
    w = sw.base
    q, k, v = generate(w, device=DEV, seed=0)
    V, S = generate_sparse(sw)
    out = dca.sparse_prefill(q, k, v, dca.SparsePattern(V, S), **w.params())
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, w.L - 1, w.chunk_size, w.chunk_size + 5],
                                     rng.integers(0, w.L, 24)]))
    heads = sample_heads(w).numpy()
    got = gather(out, rows, heads)
    want = oracle.sparse_attention(q.cpu(), k.cpu(), v.cpu(), vertical=V, slash=S, rows=rows,
                                   heads=heads, **w.params())
    assert_close(got, want, torch.bfloat16, "1m sparse")
