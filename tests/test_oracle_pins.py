"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each check below is also run against deliberately broken copies of the oracle
(the ``mutation`` knob of the C oracle) to show that a plausible mistake in
the oracle fails at least one pin.
"""
import math

import numpy as np
import pytest

import oracle
from tests import oracle_refs as R

RNG = np.random.default_rng(1234)


def _rand(shape, rng=None, scale=1.0):
    rng = RNG if rng is None else rng
    return rng.standard_normal(shape) * scale


# ----------------------------------------------------------------------------
# individual pins (each returns True when the oracle agrees); mutation=0 is the
# real oracle, other values plant one known mistake in it
# ----------------------------------------------------------------------------

def pin_single_chunk_reduces_to_rope(mutation=0):
    """chunk_size >= L and no YaRN: DCA is plain causal RoPE attention."""
    rng = np.random.default_rng(1)
    L, Hq, Hkv, d, base = 37, 4, 2, 16, 100.0
    q, k, v = _rand((L, Hq, d), rng), _rand((L, Hkv, d), rng), _rand((L, Hkv, d), rng)
    want = R.rope_attention(q, k, v, base, 1.0 / math.sqrt(d))
    ok = True
    for s in (L, L + 5):
        got = oracle.attention(q, k, v, chunk_size=s, local_window=3, pretrain_window=2 * s + 7,
                               rope_base=base, yarn_scale=1.0, mutation=mutation)
        ok &= np.allclose(got, want, rtol=0, atol=1e-12)
    return bool(ok)


def pin_full_window_reduces_to_rope(mutation=0):
    """w = s, L <= 2s, 2s <= c: every pair keeps its true distance (successive branch)."""
    rng = np.random.default_rng(2)
    L, Hq, Hkv, d, base, s = 40, 2, 1, 16, 50.0, 24
    q, k, v = _rand((L, Hq, d), rng), _rand((L, Hkv, d), rng), _rand((L, Hkv, d), rng)
    want = R.rope_attention(q, k, v, base, 1.0 / math.sqrt(d))
    got = oracle.attention(q, k, v, chunk_size=s, local_window=s, pretrain_window=2 * s,
                           rope_base=base, yarn_scale=1.0, mutation=mutation)
    return bool(np.allclose(got, want, rtol=0, atol=1e-12))


def _golden_check(fname, reading, mutation):
    for i, pq, pk, cls in R.read_golden_map(fname):
        for j in range(i + 1):
            c, a, b = oracle.position(i, j, 4, 2, 7, reading=reading, mutation=mutation)
            if (c, a, b) != (cls[j], pq[j], pk[j]):
                return False
    return True


def pin_golden_position_map(mutation=0):
    return _golden_check("position_map_L12_s4_w2_c7.txt", 0, mutation)


def pin_golden_logits(mutation=0, reading=0, fname="position_map_L12_s4_w2_c7.txt"):
    """Attention probabilities of the oracle on the hand-worked toy case equal the
    softmax of RoPE logits taken at the hand-worked positions.  V is one-hot per key,
    so out[i, :, j] is the probability of key j."""
    rng = np.random.default_rng(3)
    L, d, base = 12, 16, 7.0
    q = _rand((L, 1, d), rng)
    k = _rand((L, 1, d), rng)
    v = np.zeros((L, 1, d))
    for j in range(L):
        v[j, 0, j] = 1.0
    got = oracle.attention(q, k, v, chunk_size=4, local_window=2, pretrain_window=7,
                           rope_base=base, reading=reading, mutation=mutation)[:, 0, :]
    for i, pq, pk, _ in R.read_golden_map(fname):
        qi = R.rope_complex(q[i:i + 1].repeat(i + 1, 0), np.array(pq), base)[:, 0, :]
        kj = R.rope_complex(k[:i + 1], np.array(pk), base)[:, 0, :]
        lg = np.sum(qi * kj, axis=-1) / math.sqrt(d)
        p = np.exp(lg - lg.max())
        p /= p.sum()
        if not np.allclose(got[i, :i + 1], p, rtol=0, atol=1e-12):
            return False
        if not np.allclose(got[i, i + 1:L], 0.0, atol=0):
            return False
    return True


def pin_first_row_and_zero_query(mutation=0):
    """Closed forms: row 0 attends only to key 0; q = 0 gives the running mean of v."""
    rng = np.random.default_rng(4)
    L, Hq, Hkv, d = 30, 2, 1, 8
    q, k, v = _rand((L, Hq, d), rng), _rand((L, Hkv, d), rng), _rand((L, Hkv, d), rng)
    kw = dict(chunk_size=7, local_window=3, pretrain_window=12, rope_base=1e4, yarn_scale=3.0,
              mutation=mutation)
    got = oracle.attention(q, k, v, **kw)
    ok = np.allclose(got[0, 0], v[0, 0], atol=1e-14) and np.allclose(got[0, 1], v[0, 0], atol=1e-14)
    got0 = oracle.attention(np.zeros_like(q), k, v, **kw)
    mean = np.cumsum(v[:, 0, :], axis=0) / np.arange(1, L + 1)[:, None]
    ok &= np.allclose(got0[:, 0, :], mean, atol=1e-13)
    return bool(ok)


def pin_yarn_temperature(mutation=0):
    """YaRN only rescales logits: out(q, f) == out(q * m(f)^2, f = 1), m(f) = 0.1 ln f + 1."""
    rng = np.random.default_rng(5)
    L, Hq, Hkv, d = 33, 2, 1, 16
    q, k, v = _rand((L, Hq, d), rng), _rand((L, Hkv, d), rng), _rand((L, Hkv, d), rng)
    kw = dict(chunk_size=8, local_window=3, pretrain_window=16, rope_base=300.0, mutation=mutation)
    f = 5.0
    m = 0.1 * math.log(f) + 1.0
    a = oracle.attention(q, k, v, yarn_scale=f, **kw)
    b = oracle.attention(q * m * m, k, v, yarn_scale=1.0, **kw)
    return bool(np.allclose(a, b, rtol=0, atol=1e-12))


def pin_gqa_expansion(mutation=0):
    """Grouped call == call with every KV head repeated G times (consecutive groups)."""
    rng = np.random.default_rng(6)
    L, Hq, Hkv, d = 26, 6, 2, 8
    q, k, v = _rand((L, Hq, d), rng), _rand((L, Hkv, d), rng), _rand((L, Hkv, d), rng)
    kw = dict(chunk_size=6, local_window=2, pretrain_window=11, rope_base=1e3, mutation=mutation)
    a = oracle.attention(q, k, v, **kw)
    b = oracle.attention(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), **kw)
    return bool(np.allclose(a, b, rtol=0, atol=1e-13))


def pin_relative_logits_bruteforce(mutation=0, reading=0):
    """Explicit L x L position matrices (rules re-derived here, vectorised) and the
    relative form of RoPE vs the oracle's factored computation, over a sweep."""
    rng = np.random.default_rng(7)
    d, base = 64, 20.0
    for L, s, w, c in [(1, 1, 0, 1), (5, 2, 1, 3), (17, 4, 0, 4), (17, 4, 4, 9), (31, 5, 2, 7),
                       (32, 8, 3, 14), (40, 6, 6, 12), (40, 13, 5, 18), (64, 16, 8, 24)]:
        q = _rand((L, 1, d), rng)
        k = _rand((L, 1, d), rng)
        v = np.zeros((L, 1, d))
        v[np.arange(L), 0, np.arange(L)] = 1.0
        got = oracle.attention(q, k, v, chunk_size=s, local_window=w, pretrain_window=c,
                               rope_base=base, reading=reading, mutation=mutation)[:, 0, :]
        i = np.arange(L)[:, None]
        j = np.arange(L)[None, :]
        ni, nj, ri = i // s, j // s, i % s
        win = (ri < w) if reading == 0 else ((i - j) < w)
        Pq = np.where(ni == nj, ri, np.where((ni - nj == 1) & win, s + ri, c - 1))
        Pk = j % s + 0 * i
        lg = R.relative_logits(q[:, 0], k[:, 0], (Pq - Pk).astype(np.float64), base,
                               1.0 / math.sqrt(d))
        lg = np.where(j <= i, lg, -np.inf)
        p = np.exp(lg - lg.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        if not np.allclose(got[:, :L], p, rtol=0, atol=1e-12):
            return False
    return True


def pin_distance_invariant(mutation=0):
    """Every remapped relative distance lies in [0, c) (exhaustive on small cases)."""
    for L in (1, 7, 20, 33):
        for s in range(1, 12):
            for w in sorted({0, 1, s // 2, s}):
                for c in (s + w, s + w + 3):
                    if c < 1:
                        continue
                    for i in range(L):
                        for j in range(i + 1):
                            _, pq, pk = oracle.position(i, j, s, w, c, mutation=mutation)
                            if not (0 <= pq - pk < c):
                                return False
    return True


def pin_chunked_equals_oneshot(mutation=0):
    rng = np.random.default_rng(8)
    L, Hq, Hkv, d, blk = 50, 2, 1, 8, 16
    q, k, v = _rand((L, Hq, d), rng), _rand((L, Hkv, d), rng), _rand((L, Hkv, d), rng)
    kw = dict(chunk_size=9, local_window=4, pretrain_window=20, rope_base=1e3, yarn_scale=2.0,
              mutation=mutation)
    full = oracle.attention(q, k, v, **kw)
    for q0 in range(0, L, blk):
        lq = min(blk, L - q0)
        part = oracle.attention(q[q0:q0 + lq], k[:q0 + lq], v[:q0 + lq], q_start=q0, **kw)
        if not np.allclose(part, full[q0:q0 + lq], rtol=0, atol=1e-13):
            return False
    return True


PINS = [
    pin_single_chunk_reduces_to_rope,
    pin_full_window_reduces_to_rope,
    pin_golden_position_map,
    pin_golden_logits,
    pin_first_row_and_zero_query,
    pin_yarn_temperature,
    pin_gqa_expansion,
    pin_relative_logits_bruteforce,
    pin_distance_invariant,
    pin_chunked_equals_oneshot,
]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    assert pin(0)


def test_golden_position_map_reading_b():
    assert _golden_check("position_map_B_L12_s4_w2_c7.txt", 1, 0)
    assert pin_golden_logits(0, reading=1, fname="position_map_B_L12_s4_w2_c7.txt")
    assert pin_relative_logits_bruteforce(0, reading=1)


def test_readings_differ_on_toy_case():
    """The two window readings give different maps (so the choice is visible)."""
    a = R.read_golden_map("position_map_L12_s4_w2_c7.txt")
    b = R.read_golden_map("position_map_B_L12_s4_w2_c7.txt")
    assert a != b


def test_mscale_values():
    assert oracle.mscale(1.0) == 1.0
    assert oracle.mscale(0.5) == 1.0
    assert oracle.mscale(math.exp(10.0)) == pytest.approx(2.0, abs=1e-15)
    assert oracle.mscale(math.exp(5.0)) == pytest.approx(1.5, abs=1e-15)


def test_large_logits_stable():
    """Two-pass softmax: logits in the hundreds stay finite and match the library."""
    rng = np.random.default_rng(9)
    L, d, base = 24, 16, 100.0
    q, k, v = _rand((L, 1, d), rng, 30.0), _rand((L, 1, d), rng, 30.0), _rand((L, 1, d), rng)
    got = oracle.attention(q, k, v, chunk_size=L, local_window=0, pretrain_window=L,
                           rope_base=base)
    want = R.rope_attention(q, k, v, base, 1.0 / math.sqrt(d))
    assert np.all(np.isfinite(got))
    assert np.allclose(got, want, rtol=0, atol=1e-10)


def test_dca_differs_from_rope_beyond_one_chunk():
    rng = np.random.default_rng(10)
    L, d, base = 40, 16, 10.0
    q, k, v = _rand((L, 1, d), rng), _rand((L, 1, d), rng), _rand((L, 1, d), rng)
    got = oracle.attention(q, k, v, chunk_size=8, local_window=2, pretrain_window=12, rope_base=base)
    want = R.rope_attention(q, k, v, base, 1.0 / math.sqrt(d))
    assert np.allclose(got[:8], want[:8], atol=1e-12)       # first chunk: unchanged
    assert not np.allclose(got[16:], want[16:], atol=1e-3)  # far rows: remapped


def test_page_constants_used_by_workloads():
    from length_extrapolation_b200 import workloads as W
    pc = R.read_page_constants()
    big = W.WORKLOADS["qwen7b_1m_chunked"]
    assert big.rope_base == pc["rope_base"]
    assert big.block == pc["chunked_prefill_block"]
    assert big.pretrain_window == pc["pretrain_window_1m_model"]
    assert big.L == pc["target_context"]


# the dense oracle's mutations (the sparse variant's are pinned in test_sparse_oracle_pins.py)
@pytest.mark.parametrize("name,code", sorted((n, c) for n, c in oracle.MUTATIONS.items()
                                             if not n.startswith("sp_")))
def test_planted_mistake_is_caught(name, code):
    failed = [p.__name__ for p in PINS if not p(code)]
    assert failed, f"mutation {name} passes every pin"
