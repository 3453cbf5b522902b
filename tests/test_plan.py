"""The tile plan of the CUDA kernels (host-side introspection through the C ABI)
against the oracle's per-pair DCA positions, on CPU.

For every query tile of a sweep of small configurations:
  * coverage: every causal pair (i, j) of a real row is admitted by exactly one
    work item -- the item of its key tile whose class is the pair's chunk
    distance class -- and that class's query rotation equals the oracle's query
    position for the pair;
  * full items really are uniform: every pair of a 'full' tile is causal and of
    the item's class (so skipping the mask is safe).
"""
import ctypes

import numpy as np
import pytest

import oracle
from length_extrapolation_b200 import _native as N
from length_extrapolation_b200 import build as B


@pytest.fixture(scope="module")
def lib():
    B.build()
    return N.lib()


def plan(lib, i0, i_last, rows, s, bn, w=0, reading=0):
    buf = (ctypes.c_int32 * (3 * 16384))()
    n = lib.dca_plan_items(i0, i_last, rows, s, w, reading, bn, buf, 16384)
    assert 0 <= n <= 16384
    a = np.frombuffer(buf, dtype=np.int32)[: 3 * n].reshape(n, 3)
    return a


def chunk_class(i, j, s, w=0, reading=0):
    """Work-list class of a pair: 0 intra, 1 successive with its true distance
    kept (reading A: every adjacent-chunk pair), 2 inter-chunk rule."""
    dn = i // s - j // s
    if dn == 0:
        return 0
    if dn == 1 and (reading == 0 or i - j < w):
        return 1
    return 2


def query_position(i, cls, s, w, c):
    """Query rotation of a row in a plan class, as stated in include/dca.h."""
    r = i % s
    if cls == 0:
        return r
    if cls == 1 and r < w:
        return s + r
    return c - 1


CASES = [  # (L, s, w, c, bm, bn)
    (300, 64, 16, 100, 64, 64),
    (300, 100, 30, 140, 64, 64),
    (520, 37, 5, 50, 128, 128),
    (700, 128, 128, 256, 128, 128),
    (700, 200, 0, 200, 128, 128),
    (260, 1, 1, 2, 128, 128),
    (260, 3, 2, 5, 64, 64),
    (400, 1000, 7, 1, 128, 128),    # single chunk (L <= s): everything intra
    (1100, 256, 128, 512, 128, 128),
]


@pytest.mark.parametrize("reading", [0, 1], ids=["query_offset", "true_distance"])
@pytest.mark.parametrize("L,s,w,c,bm,bn", CASES)
def test_plan_matches_oracle_positions(lib, L, s, w, c, bm, bn, reading):
    for q_start, Lq in [(0, L), (L // 3, L - L // 3)]:
        for t0 in range(0, Lq, bm):
            i0 = q_start + t0
            i_last = min(i0 + bm - 1, q_start + Lq - 1)
            items = plan(lib, i0, i_last, bm, s, bn, w, reading)
            # phases in order INTER, SUCC, INTRA
            assert list(items[:, 1]) == sorted(items[:, 1], reverse=True)
            seen = {}
            for kt, cls, full in items:
                assert (kt, cls) not in seen
                seen[(kt, cls)] = full
                if full:
                    for i in range(i0, i0 + bm):
                        for j in range(kt * bn, kt * bn + bn):
                            assert j <= i and chunk_class(i, j, s, w, reading) == cls
            for i in range(i0, i_last + 1):
                for j in range(0, i + 1):
                    cls = chunk_class(i, j, s, w, reading)
                    assert (j // bn, cls) in seen, (i, j)
                    _, pq, pk = oracle.position(i, j, s, w, c, reading=reading)
                    assert pk == j % s
                    assert query_position(i, cls, s, w, c) == pq, (i, j, cls)


def test_plan_rejects_bad_args(lib):
    buf = (ctypes.c_int32 * 3)()
    assert lib.dca_plan_items(10, 5, 128, 64, 8, 0, 128, buf, 1) == N.DCA_ERR_ARG
    assert lib.dca_plan_items(0, 200, 128, 64, 8, 0, 128, buf, 1) == N.DCA_ERR_ARG
    assert lib.dca_plan_items(0, 5, 128, 0, 0, 0, 128, buf, 1) == N.DCA_ERR_ARG
    assert lib.dca_plan_items(0, 5, 128, 64, 65, 0, 128, buf, 1) == N.DCA_ERR_ARG
    assert lib.dca_plan_items(0, 5, 128, 64, 8, 2, 128, buf, 1) == N.DCA_ERR_ARG


def test_big_config_phase_counts(lib):
    """Last query tile of the 1M chunked workload: INTER keys of chunks 0-3,
    SUCC tiles of chunk 4, INTRA tiles of chunk 5 up to the diagonal, all full
    except the diagonal tile."""
    s, L = 196608, 1048576
    i0 = L - 128
    items = plan(lib, i0, L - 1, 128, s, 128)
    n_inter = (items[:, 1] == 2).sum()
    n_succ = (items[:, 1] == 1).sum()
    n_intra = (items[:, 1] == 0).sum()
    assert n_inter == 4 * s // 128
    assert n_succ == s // 128
    assert n_intra == (L - 5 * s) // 128
    assert items[:, 2].sum() == len(items) - 1


def test_selection_row_ranges_brute_force(lib):
    """The key selection masks each key's rows to one contiguous range per
    work-list class (or key chunk, continuous positions); against the
    per-pair class over random small configurations."""
    rng = np.random.default_rng(7)
    rg = (ctypes.c_int32 * 2)()
    for _ in range(3000):
        s = int(rng.integers(1, 300))
        w = int(rng.integers(0, s + 1))
        reading = int(rng.integers(0, 2))
        n_rows = int(rng.integers(1, 65))
        i_first = int(rng.integers(0, 2000))
        kv_len = i_first + n_rows - int(rng.integers(0, n_rows)) if rng.random() < 0.3 \
            else i_first + n_rows + int(rng.integers(0, 50))
        j = int(rng.integers(0, i_first + 200))
        cls = int(rng.integers(-1, 3))
        chunk = j // s if rng.random() < 0.5 else int(rng.integers(0, 20))
        assert lib.dca_class_rows(j, i_first, n_rows, kv_len, s, w, reading, cls, chunk, rg) == 0
        ra, rb = rg[0], rg[1]
        assert 0 <= ra <= rb <= n_rows
        for r in range(n_rows):
            i = i_first + r
            want = j <= i and j < kv_len
            want = want and (chunk_class(i, j, s, w, reading) == cls if cls >= 0 else j // s == chunk)
            assert want == (ra <= r < rb), (s, w, reading, i_first, j, cls, r, ra, rb)


def test_selection_row_ranges_reject(lib):
    rg = (ctypes.c_int32 * 2)()
    ok = dict(j=5, i_first=0, n_rows=8, kv_len=100, s=16, w=4, reading=0, cls=0, chunk=0)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.dca_class_rows(a["j"], a["i_first"], a["n_rows"], a["kv_len"], a["s"], a["w"],
                                  a["reading"], a["cls"], a["chunk"], rg)
    assert call() == 0
    for bad in (dict(j=-1), dict(j=1 << 31), dict(n_rows=0), dict(n_rows=65), dict(s=0),
                dict(w=17), dict(cls=3), dict(cls=-2), dict(reading=2), dict(i_first=-1)):
        assert call(**bad) == N.DCA_ERR_ARG, bad
    assert lib.dca_class_rows(5, 0, 8, 100, 16, 4, 0, 0, 0, None) == N.DCA_ERR_ARG


@pytest.mark.parametrize("s,w,q_start,L", [
    (128, 0, 0, 1000), (256, 128, 128, 1500), (384, 200, 256, 2600), (1024, 1024, 0, 4200),
    (512, 77, 1024, 3000), (128, 128, 384, 900)])
def test_consecutive_tiles_share_an_ascending_key_order(lib, s, w, q_start, L):
    """Under reading A with s a multiple of 128 and a 128-aligned q_start (the
    condition under which the attention kernel runs a group's last head on two
    consecutive query tiles in one CTA), every tile's work list is its key
    tiles 0, 1, 2, ... in order, each once, and tile t's list is a prefix of
    tile t + 1's, with its own class per key tile."""
    rows = 128
    prev = None
    for q0 in range(q_start, L, rows):
        i_last = min(q0 + rows - 1, L - 1)
        a = plan(lib, q0, i_last, rows, s, 128, w=w, reading=0)
        assert a[:, 0].tolist() == list(range(len(a)))
        for kt, cls, _ in a:
            js = range(kt * 128, min(kt * 128 + 128, i_last + 1))
            want = {chunk_class(i, j, s, w) for i in range(q0, i_last + 1) for j in js if j <= i}
            assert want == {cls}
        if prev is not None:
            assert len(a) == len(prev) + 1
            assert a[:len(prev), 0].tolist() == prev[:, 0].tolist()
        prev = a


@pytest.mark.parametrize("s,w,reading", [(1, 0, 0), (3, 2, 0), (3, 2, 1), (7, 0, 1), (7, 7, 1),
                                         (10, 4, 0), (10, 4, 1), (16, 1, 1), (64, 63, 1)])
def test_row_key_ranges_match_pair_classes(lib, s, w, reading):
    """The attention kernel masks a tile to one contiguous key range per row
    and class; brute force over rows and keys: key j is inside row i's range
    for class c exactly when j <= i and the pair's class is c."""
    rng = ctypes.c_int64 * 2
    for i in range(0, 6 * s + 5):
        for c in range(3):
            r = rng()
            assert lib.dca_row_keys(i, c, s, w, reading, r) == N.DCA_OK
            want = [j for j in range(i + 1) if chunk_class(i, j, s, w, reading) == c]
            got = list(range(r[0], r[1]))
            assert got == want, (i, c, r[0], r[1], want[:3], want[-3:])
    r = rng()
    assert lib.dca_row_keys(5, 3, 4, 1, 0, r) == N.DCA_ERR_ARG
    assert lib.dca_row_keys(5, 0, 4, 5, 0, r) == N.DCA_ERR_ARG
