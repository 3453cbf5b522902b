"""Pins of the oracle's key-selection scores (the estimate behind the sparse
pattern) and of its top-k.

vertical_h[j] = sum over the last n_last rows i of p_ij, slash_h[o] = sum of
p_{i, i-o}, with p the softmax over j <= i of the DCA logits, or of RoPE
logits at the true positions (continuous=True).  Pinned to:
  - the dense oracle: with one-hot values v_j = e_j (key count <= d) its
    output row is the probability row p_i., a separate code path;
  - continuous positions = the dense oracle on a single chunk (chunk size
    >= key count, where DCA keeps every true position);
  - each probability row sums to one, so each score vector sums to n_last;
  - continuous and DCA scores agree on one chunk and differ across chunks.
Top-k: the n largest by value, ties to the smaller index, against a sort.
"""
import numpy as np
import pytest
import torch

import oracle

D = 128


def qk(L, Hq, Hkv, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(L, Hq, D, generator=g, dtype=torch.float64)
    k = torch.randn(L, Hkv, D, generator=g, dtype=torch.float64)
    return q, k


def onehot_v(L, Hkv):
    v = torch.zeros(L, Hkv, D, dtype=torch.float64)
    for j in range(L):
        v[j, :, j] = 1.0
    return v


def scores_from_dense(q, k, n_last, **P):
    """vertical, slash from the dense oracle's probability rows."""
    L, Hq, _ = q.shape
    v = onehot_v(L, k.shape[1])
    out = oracle.attention(q, k, v, **P)  # [L, Hq, D], row i = p_i. in dims 0..L-1
    vert = np.zeros((Hq, L))
    slash = np.zeros((Hq, L))
    for i in range(L - n_last, L):
        p = out[i, :, :L]
        vert += p
        for j in range(i + 1):
            slash[:, i - j] += p[:, j]
    return vert, slash


P_DCA = dict(chunk_size=24, local_window=6, pretrain_window=40, rope_base=1e4, yarn_scale=2.0)


@pytest.mark.parametrize("reading", [0, 1])
def test_dca_scores_equal_dense_probabilities(reading):
    q, k = qk(120, 4, 2, 0)
    want_v, want_s = scores_from_dense(q, k, 20, reading=reading, **P_DCA)
    v, s = oracle.vs_scores(q, k, n_last=20, reading=reading, **P_DCA)
    assert np.abs(v - want_v).max() < 1e-12 and np.abs(s - want_s).max() < 1e-12


def test_continuous_scores_equal_single_chunk_dense():
    q, k = qk(110, 2, 1, 1)
    one_chunk = dict(chunk_size=128, local_window=8, pretrain_window=256, rope_base=1e4,
                     yarn_scale=2.0)
    want_v, want_s = scores_from_dense(q, k, 16, **one_chunk)
    v, s = oracle.vs_scores(q, k, n_last=16, continuous=True, **P_DCA)  # chunking ignored
    assert np.abs(v - want_v).max() < 1e-12 and np.abs(s - want_s).max() < 1e-12


def test_scores_sum_to_rows():
    q, k = qk(200, 3, 1, 2)
    for cont in (False, True):
        v, s = oracle.vs_scores(q[150:], k, q_start=150, n_last=30, continuous=cont, **P_DCA)
        assert np.allclose(v.sum(1), 30.0) and np.allclose(s.sum(1), 30.0)
        assert (v >= 0).all() and (s >= 0).all()
        assert np.all(s[:, 200:] == 0)          # no offset beyond the last row


def test_modes_agree_on_one_chunk_and_differ_across_chunks():
    q, k = qk(90, 2, 2, 3)
    one = dict(P_DCA, chunk_size=100, pretrain_window=120)
    a = oracle.vs_scores(q, k, n_last=10, **one)
    b = oracle.vs_scores(q, k, n_last=10, continuous=True, **one)
    assert np.abs(a[0] - b[0]).max() < 1e-12
    c = oracle.vs_scores(q, k, n_last=10, **P_DCA)
    d = oracle.vs_scores(q, k, n_last=10, continuous=True, **P_DCA)
    assert np.abs(c[0] - d[0]).max() > 1e-3


def test_topk_against_sort():
    rng = np.random.default_rng(0)
    for _ in range(20):
        n = int(rng.integers(1, 60))
        x = rng.integers(0, 8, size=n).astype(np.float64)  # many ties
        k = int(rng.integers(0, n + 1))
        order = sorted(range(n), key=lambda j: (-x[j], j))[:k]
        assert oracle.topk(x, k).tolist() == sorted(order)
