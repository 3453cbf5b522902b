"""Pins of the oracle's vertical-slash sparse variant.

The sparse oracle attends, for query head h and row i, the member keys
M_h(i) = {j <= i in V_h} U {i - o : o in S_h, o <= i} U {i} (each once).  The
pins tie it to things other than itself:
  - reductions to the dense oracle: every offset selected, every key vertical,
    both at once (a key reachable twice counts once);
  - rows that a band of offsets or a prefix of vertical keys covers entirely
    equal the dense rows, and a row outside differs;
  - a single member (the row's own key): out_i = v_i exactly;
  - a slash offset o seen from row i and the vertical key i - o are the same
    member (the two membership paths agree);
  - out is a softmax-weighted mean of values: adding a constant to every v
    adds it to every output.
Each planted mistake of the sparse variant fails at least one pin.
"""
import numpy as np
import pytest
import torch

import oracle

P = dict(chunk_size=16, local_window=5, pretrain_window=24, rope_base=10000.0, yarn_scale=2.0)
L, HQ, HKV, D = 70, 4, 2, 128


def inputs(seed=0, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(L, HQ, D, generator=g, dtype=torch.float64).to(dtype)
    k = torch.randn(L, HKV, D, generator=g, dtype=torch.float64).to(dtype)
    v = torch.randn(L, HKV, D, generator=g, dtype=torch.float64).to(dtype)
    return q, k, v


def sparse(q, k, v, vert, slash, mutation=0, **kw):
    return oracle.sparse_attention(q, k, v, vertical=vert, slash=slash, mutation=mutation,
                                   **{**P, **kw})


ALL = list(range(L))
NONE = []


def pin_full_slash(q, k, v, mutation=0):
    got = sparse(q, k, v, [NONE] * HQ, [ALL] * HQ, mutation)
    return np.abs(got - oracle.attention(q, k, v, **P)).max() < 1e-12


def pin_full_vertical(q, k, v, mutation=0):
    got = sparse(q, k, v, [ALL] * HQ, [NONE] * HQ, mutation)
    return np.abs(got - oracle.attention(q, k, v, **P)).max() < 1e-12


def pin_both_full(q, k, v, mutation=0):
    got = sparse(q, k, v, [ALL] * HQ, [ALL] * HQ, mutation)
    return np.abs(got - oracle.attention(q, k, v, **P)).max() < 1e-12


def pin_self_only(q, k, v, mutation=0):
    got = sparse(q, k, v, [NONE] * HQ, [NONE] * HQ, mutation)
    want = np.repeat(v.double().numpy(), HQ // HKV, axis=1)  # head h reads KV head h // G
    return np.abs(got - want).max() == 0.0


def pin_band(q, k, v, mutation=0, W=9):
    got = sparse(q, k, v, [NONE] * HQ, [list(range(W))] * HQ, mutation)
    dense = oracle.attention(q, k, v, **P)
    inside = np.abs(got[:W] - dense[:W]).max() < 1e-12
    outside = np.abs(got[W:] - dense[W:]).max(axis=(1, 2)).min() > 1e-6
    return inside and outside


def pin_vertical_prefix(q, k, v, mutation=0, Pn=12):
    got = sparse(q, k, v, [list(range(Pn))] * HQ, [NONE] * HQ, mutation)
    dense = oracle.attention(q, k, v, **P)
    inside = np.abs(got[:Pn] - dense[:Pn]).max() < 1e-12
    outside = np.abs(got[Pn + 1:] - dense[Pn + 1:]).max(axis=(1, 2)).min() > 1e-6
    return inside and outside


def pin_slash_is_vertical(q, k, v, mutation=0):
    ok = True
    for i, o in [(40, 7), (63, 33), (17, 16), (69, 1)]:
        rows = np.array([i])
        a = sparse(q, k, v, [NONE] * HQ, [[o]] * HQ, mutation, rows=rows)
        b = sparse(q, k, v, [[i - o]] * HQ, [NONE] * HQ, mutation, rows=rows)
        ok = ok and np.abs(a - b).max() < 1e-12
    return ok


def pin_shift(q, k, v, mutation=0):
    rng = np.random.default_rng(3)
    vert = [sorted(rng.choice(L, 6, replace=False).tolist()) for _ in range(HQ)]
    sl = [sorted(rng.choice(L, 5, replace=False).tolist()) for _ in range(HQ)]
    a = sparse(q, k, v, vert, sl, mutation)
    b = sparse(q, k, v + 3.25, vert, sl, mutation)
    return np.abs(b - (a + 3.25)).max() < 1e-10


PINS = [pin_full_slash, pin_full_vertical, pin_both_full, pin_self_only, pin_band,
        pin_vertical_prefix, pin_slash_is_vertical, pin_shift]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin_holds(pin):
    assert pin(*inputs())


@pytest.mark.parametrize("name", ["sp_no_dedup", "sp_vert_acausal", "sp_offset_off1",
                                  "sp_no_self"])
def test_planted_mistake_is_caught(name):
    q, k, v = inputs(1)
    caught = [p.__name__ for p in PINS if not p(q, k, v, oracle.MUTATIONS[name])]
    assert caught, f"mutation {name} passes every pin"


def test_chunked_rows_equal_one_shot():
    """A query block with q_start gives the same rows as the one-shot call."""
    q, k, v = inputs(2)
    rng = np.random.default_rng(5)
    vert = [sorted(rng.choice(L, 8, replace=False).tolist()) for _ in range(HQ)]
    sl = [sorted({0, 1, 2, *rng.choice(L, 6, replace=False).tolist()}) for _ in range(HQ)]
    full = sparse(q, k, v, vert, sl)
    q0 = 29
    blk = sparse(q[q0:], k, v, vert, sl, q_start=q0)
    assert np.abs(blk - full[q0:]).max() < 1e-12


def test_rejects_unsorted_or_out_of_range():
    q, k, v = inputs()
    with pytest.raises(ValueError):
        sparse(q, k, v, [[3, 2]] + [NONE] * (HQ - 1), [NONE] * HQ)
    with pytest.raises(ValueError):
        sparse(q, k, v, [NONE] * HQ, [[L]] + [NONE] * (HQ - 1))
