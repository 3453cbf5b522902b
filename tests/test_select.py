"""Online key selection for the sparse attention (DCA or continuous positions).

CPU: argument checks of dca_sparse_select.
GPU: the selected keys and offsets are a top-k of the fp64 oracle's scores
(vertical column sums and slash diagonal sums of the last rows' softmax);
where several answers are correct (scores within the rounding of the bf16
keys of each other) any of them passes, everything else must match.  Then
the sparse attention over the selected pattern against the oracle.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import length_extrapolation_b200 as dca
from length_extrapolation_b200 import _native as N
from length_extrapolation_b200.workloads import Workload, generate


@pytest.fixture(scope="module")
def lib():
    from length_extrapolation_b200 import build as B
    B.build()
    return N.lib()


def test_select_rejects(lib):
    cfg = N.DCASparseConfig(1000, 64, 64)
    n = lib.dca_sparse_workspace_size(ctypes.byref(cfg), 4)
    ws = lib.dca_workspace_size(1000, 4, 2, 128, 64, 16, 128, 0)
    sc = lib.dca_sparse_select_scratch_size(1000, 4, 64)
    assert sc > 0 and lib.dca_sparse_select_scratch_size(0, 4, 64) == 0
    p = 1 << 20

    def call(n_last=16, cont=1, nv=8, ns=8, dtype=0, sbytes=sc, Lq=100):
        return lib.dca_sparse_select(ctypes.byref(cfg), p, p, 900, Lq, 1000, 4, 2, 128, 64, 16,
                                     128, 1e7, 1.0, dtype, None, n_last, cont, nv, ns, p, ws, p,
                                     n, p, sbytes, None)

    assert call(n_last=65) == N.DCA_ERR_ARG
    assert call(n_last=0) == N.DCA_ERR_ARG
    assert call(cont=2) == N.DCA_ERR_ARG
    assert call(nv=65) == N.DCA_ERR_ARG                  # more than cfg.max_vertical
    assert call(dtype=1) == N.DCA_ERR_UNSUPPORTED
    assert call(sbytes=sc - 1) == N.DCA_ERR_WORKSPACE
    big = N.DCASparseConfig(1000, 64, 2000)
    nb = lib.dca_sparse_workspace_size(ctypes.byref(big), 4)
    assert lib.dca_sparse_select(ctypes.byref(big), p, p, 900, 100, 1000, 4, 2, 128, 64, 16, 128,
                                 1e7, 1.0, 0, None, 16, 1, 8, 1024, p, ws, p, nb, p, sc,
                                 None) == N.DCA_ERR_ARG   # n_slash above DCA_SPARSE_MAX_RUNS


DEV = "cuda:0"


def wl(name, L, Hq, Hkv, s, w, c, yarn=1.0, sqrt_d=False):
    return Workload(name, L=L, Hq=Hq, Hkv=Hkv, d=128, dtype="bf16", chunk_size=s,
                    local_window=w, pretrain_window=c, yarn_scale=yarn, scale_by_sqrt_d=sqrt_d)


def select_on_gpu(w, n_v, n_s, n_last, continuous, seed=0, q_start=None):
    q, k, v = generate(w, device=DEV, seed=seed)
    kw = dict(chunk_size=w.chunk_size, local_window=w.local_window,
              pretrain_window=w.pretrain_window)
    ws = dca.Workspace(w.L, w.Hq, w.Hkv, 128, w.chunk_size, w.local_window, w.pretrain_window,
                       q.dtype, DEV)
    dca.prepare(k, kv_len=w.L, k_rows_valid=0, rope_base=w.rope_base, workspace=ws, **kw)
    sp = dca.SparseWorkspace(w.L, w.Hq, max(1, n_v), max(1, n_s), DEV)
    q0 = 0 if q_start is None else q_start
    dca.sparse_select(q[q0:], v, q_start=q0, kv_len=w.L, rope_base=w.rope_base,
                      yarn_scale=w.yarn_scale, n_vertical=n_v, n_slash=n_s, n_last=n_last,
                      continuous=continuous, workspace=ws, sparse=sp, **kw)
    V, S = dca.sparse_pattern_get(sp, w.Hq)
    return q, k, v, ws, sp, V, S


def check_topk(sel, score, k, rel=3e-3):
    """`sel` is a valid top-k of `score` up to ties within the tolerance."""
    sel = np.asarray(sel)
    assert len(sel) == k and np.all(np.diff(sel) > 0)
    if k == 0:
        return
    thr = np.sort(score)[-k]
    tol = rel * max(thr, 1e-12) + 1e-7
    chosen = np.zeros(score.size, bool)
    chosen[sel] = True
    assert np.all(score[chosen] >= thr - tol), (score[chosen].min(), thr)
    assert np.all(score[~chosen] <= thr + tol), (score[~chosen].max(), thr)


CASES = [  # workload, n_vertical, n_slash, n_last
    (wl("sel_mixed", 2000, 4, 2, 512, 64, 1024, yarn=2.0), 100, 60, 64),
    (wl("sel_one_chunk", 900, 2, 1, 1024, 64, 2048), 50, 30, 32),
    (wl("sel_small_chunks", 1500, 3, 1, 200, 50, 300), 300, 200, 64),
    (wl("sel_g7", 3000, 7, 1, 1024, 128, 2048, sqrt_d=True), 128, 512, 64),
]


@pytest.mark.gpu
@pytest.mark.parametrize("continuous", [True, False], ids=["continuous", "dca"])
@pytest.mark.parametrize("w,nv,ns,nl", CASES, ids=lambda x: getattr(x, "name", ""))
def test_selection_is_a_topk_of_the_oracle_scores(w, nv, ns, nl, continuous):
    q, k, v, ws, sp, V, S = select_on_gpu(w, nv, ns, nl, continuous)
    vert, slash = oracle.vs_scores(q.cpu(), k.cpu(), n_last=nl, continuous=continuous,
                                   **w.params())
    for h in range(w.Hq):
        check_topk(V[h], vert[h], min(nv, w.L))
        check_topk(S[h], slash[h], min(ns, w.L))


# Key ranges beyond one score slice (4096 keys per CTA of the score passes) and
# beyond one top-k span (16,384 keys per CTA of the radix select): the slices'
# row statistics are merged across CTAs and the spans' counts place each
# span's part of the ordered output.
#   sel_50k_g7:  13 slices, 4 spans (the last ragged), G = 7, n_last = 64
#   sel_70k_gqa: 18 slices, 5 spans (the last ragged), G = 2, YaRN 2, n_last = 48
MULTI = [
    (wl("sel_50k_g7", 50000, 7, 1, 4096, 512, 8192, sqrt_d=True), 1000, 1000, 64),
    (wl("sel_70k_gqa", 70000, 4, 2, 16384, 2048, 32768, yarn=2.0), 700, 900, 48),
]


@pytest.mark.gpu
@pytest.mark.parametrize("continuous", [True, False], ids=["continuous", "dca"])
@pytest.mark.parametrize("w,nv,ns,nl", MULTI, ids=lambda x: getattr(x, "name", ""))
def test_selection_spanning_slices_and_spans(w, nv, ns, nl, continuous):
    assert w.L > 2 * 16384 and w.L % 16384 != 0 and w.L > 4 * 4096
    q, k, v, ws, sp, V, S = select_on_gpu(w, nv, ns, nl, continuous)
    vert, slash = oracle.vs_scores(q.cpu(), k.cpu(), n_last=nl, continuous=continuous,
                                   **w.params())
    for h in range(w.Hq):
        check_topk(V[h], vert[h], nv)
        check_topk(S[h], slash[h], ns)
        # the selections reach into every span, not only the first
        assert V[h].max() >= 2 * 16384 and S[h].max() >= 16384


def _rope(x, pos, base=1e7):
    """Rotate the last axis of x (d = 128, pairs (k, k + 64)) by position pos (fp64)."""
    d = x.shape[-1]
    th = base ** (-2.0 * np.arange(d // 2) / d)
    c, sn = np.cos(pos * th), np.sin(pos * th)
    a, b = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([a * c - b * sn, a * sn + b * c], axis=-1)


@pytest.mark.gpu
def test_exact_ties_across_topk_spans():
    """Seven bit-identical keys with the same j mod s (12000 + 4096 n,
    n = 0..6), all inter-chunk for the estimate rows, straddle the first three
    16,384-key spans (two in span 0, four in span 1, one in span 2).  The last
    rows' queries point along the keys' rotated direction, so these keys
    score highest, exactly alike on both sides; a top-k that cuts through
    them takes the smaller indices (the oracle's rule), across spans."""
    w = wl("sel_span_ties", 50000, 2, 1, 4096, 512, 8192)
    q, k, v = generate(w, device=DEV, seed=9)
    dup = [12000 + 4096 * n for n in range(7)]
    assert [j // 16384 for j in dup] == [0, 0, 1, 1, 1, 1, 2]
    rng = np.random.default_rng(9)
    u = rng.standard_normal(128)
    key = _rope(0.5 * u, w.pretrain_window - 1 - dup[0] % w.chunk_size)   # R(j mod s) key = R(c-1) u / 2
    q[-64:] = torch.as_tensor(u, dtype=torch.float32).to(q.dtype).to(DEV)
    kb = torch.as_tensor(key, dtype=torch.float32).to(k.dtype).to(DEV)
    for j in dup:
        k[j, 0] = kb
    kw = dict(chunk_size=w.chunk_size, local_window=w.local_window,
              pretrain_window=w.pretrain_window)
    ws = dca.Workspace(w.L, w.Hq, w.Hkv, 128, w.chunk_size, w.local_window, w.pretrain_window,
                       q.dtype, DEV)
    dca.prepare(k, kv_len=w.L, k_rows_valid=0, rope_base=w.rope_base, workspace=ws, **kw)
    sp = dca.SparseWorkspace(w.L, w.Hq, 8, 8, DEV)
    vert, _ = oracle.vs_scores(q.cpu(), k.cpu(), n_last=64, continuous=False, **w.params())
    for h in range(w.Hq):
        assert len({vert[h][j] for j in dup}) == 1
        assert set(oracle.topk(vert[h], 7).tolist()) == set(dup)
    for n_v in (1, 2, 3, 6):
        dca.sparse_select(q, v, q_start=0, kv_len=w.L, rope_base=w.rope_base,
                          yarn_scale=w.yarn_scale, n_vertical=n_v, n_slash=4, n_last=64,
                          continuous=False, workspace=ws, sparse=sp, **kw)
        V, _ = dca.sparse_pattern_get(sp, w.Hq)
        for h in range(w.Hq):
            assert oracle.topk(vert[h], n_v).tolist() == dup[:n_v]
            assert V[h].tolist() == dup[:n_v], (n_v, h, V[h])


@pytest.mark.gpu
def test_selected_pattern_attention_matches_oracle():
    from tests.gpu_helpers import assert_close
    w = wl("sel_e2e", 2500, 4, 2, 512, 64, 1024, yarn=2.0, sqrt_d=True)
    q, k, v, ws, sp, V, S = select_on_gpu(w, 120, 400, 64, True, seed=4)
    kw = dict(chunk_size=w.chunk_size, local_window=w.local_window,
              pretrain_window=w.pretrain_window)
    out = dca.sparse_attend(q, v, q_start=0, kv_len=w.L, yarn_scale=w.yarn_scale, workspace=ws,
                            sparse=sp, **kw)
    torch.cuda.synchronize()
    assert ws.status() == N.DCA_OK
    want = oracle.sparse_attention(q.cpu(), k.cpu(), v.cpu(), vertical=V, slash=S, **w.params())
    assert_close(out.double().cpu().numpy(), want, torch.bfloat16, "selected pattern")


@pytest.mark.gpu
def test_continuous_and_dca_selections_differ_across_chunks():
    """Several chunks: the true-position estimate selects other keys than the
    DCA estimate (the motivation of the refinement)."""
    w = wl("sel_modes", 2048, 2, 1, 256, 32, 512)
    a = select_on_gpu(w, 64, 64, 64, True)
    b = select_on_gpu(w, 64, 64, 64, False)
    diff = sum(len(set(x.tolist()) ^ set(y.tolist())) for x, y in zip(a[5] + a[6], b[5] + b[6]))
    assert diff > 0


@pytest.mark.gpu
def test_exact_ties_take_the_smaller_index():
    """Equal cached keys of one class for every row score exactly alike (on
    both sides); a top-k that cuts through them takes the smaller indices,
    the oracle's rule.  Key 100 is made a sink and copied to 612, 1124, 1636
    (same j mod s, all inter-chunk for rows in chunk 5)."""
    w = wl("sel_ties", 3000, 2, 1, 512, 64, 1024)
    q, k, v = generate(w, device=DEV, seed=5)
    dup = [100, 612, 1124, 1636]
    k[100] = (k[100].float() * 8).to(k.dtype)
    for j in dup[1:]:
        k[j] = k[100]
    kw = dict(chunk_size=w.chunk_size, local_window=w.local_window,
              pretrain_window=w.pretrain_window)
    ws = dca.Workspace(w.L, w.Hq, w.Hkv, 128, w.chunk_size, w.local_window, w.pretrain_window,
                       q.dtype, DEV)
    dca.prepare(k, kv_len=w.L, k_rows_valid=0, rope_base=w.rope_base, workspace=ws, **kw)
    sp = dca.SparseWorkspace(w.L, w.Hq, 8, 8, DEV)
    vert, _ = oracle.vs_scores(q.cpu(), k.cpu(), n_last=64, continuous=False, **w.params())
    for n_v in (1, 2, 3):
        dca.sparse_select(q, v, q_start=0, kv_len=w.L, rope_base=w.rope_base,
                          yarn_scale=w.yarn_scale, n_vertical=n_v, n_slash=4, n_last=64,
                          continuous=False, workspace=ws, sparse=sp, **kw)
        V, _ = dca.sparse_pattern_get(sp, w.Hq)
        for h in range(w.Hq):
            assert vert[h][dup[0]] == vert[h][dup[3]] and set(oracle.topk(vert[h], 4)) == set(dup)
            assert V[h].tolist() == dup[:n_v], (n_v, h, V[h])
            assert oracle.topk(vert[h], n_v).tolist() == dup[:n_v]
