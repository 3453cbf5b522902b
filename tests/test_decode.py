"""Decode step (a few new query tokens against the whole cache).

CPU: the scratch-size rule and the argument checks of dca_decode (no launch).
GPU: parity of the split-KV decode kernel (bf16) and of the fp32 path with the
fp64 oracle, whose rows q_start .. q_start + Lq - 1 are the same definition as
the prefill rows (decode = the last rows of a chunked prefill), including the
natural-log LSE; the generation-step composition (rotate the new keys, then
decode); the bounded-wait timeout path; a full 1M-token cache.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import length_extrapolation_b200 as dca
from length_extrapolation_b200 import _native as N
from length_extrapolation_b200.workloads import (DECODE_WORKLOADS, DecodeWorkload, Workload,
                                                 generate_decode)

DEV = "cuda:0"


@pytest.fixture(scope="module")
def lib():
    from length_extrapolation_b200 import build as B
    B.build()
    return N.lib()


# ------------------------------------------------------------------ CPU


def test_scratch_size_rule(lib):
    # (Hkv * row groups * slices) CTAs, each nr rows x (128 + 2) fp32 words;
    # a row group holds 16 (token, head) rows, or 32 when a KV head has more
    def expect(Lq, Hq, Hkv):
        rows = Lq * (Hq // Hkv)
        nr = 16 if rows <= 16 else 32
        n_rg = -(-rows // nr)
        n_cta = Hkv * n_rg * max(1, 148 // (Hkv * n_rg))
        return -(-n_cta * nr * 130 * 4 // 256) * 256
    for Lq, Hq, Hkv in [(1, 28, 4), (4, 28, 4), (256, 28, 4), (1, 8, 8), (3, 40, 8), (1, 1, 1)]:
        assert lib.dca_decode_scratch_size(Lq, Hq, Hkv) == expect(Lq, Hq, Hkv)
    assert lib.dca_decode_scratch_size(0, 28, 4) == 0
    assert lib.dca_decode_scratch_size(N.DCA_DECODE_MAX_TOKENS + 1, 28, 4) == 0
    assert lib.dca_decode_scratch_size(1, 28, 5) == 0


def test_decode_rejects_before_launch(lib):
    p = 1 << 20
    ws = lib.dca_workspace_size(512, 4, 2, 128, 64, 16, 128, 0)
    sc = lib.dca_decode_scratch_size(2, 4, 2)

    def call(q0=98, lq=2, lk=100, opts=None, scratch=p, sbytes=sc, lse=None, dtype=0):
        return lib.dca_decode(p, p, p, lse, q0, lq, lk, 4, 2, 128, 64, 16, 128, 1.0, dtype, opts,
                              p, ws, scratch, sbytes, None)

    bad = N.DCAOptions()
    bad.window_reading = 5
    assert call(opts=ctypes.byref(bad)) == N.DCA_ERR_ARG
    assert call(q0=99) == N.DCA_ERR_ARG                       # q_start + Lq > Lk
    assert call(scratch=0) == N.DCA_ERR_ARG                   # no scratch
    assert call(scratch=p + 8) == N.DCA_ERR_ARG               # misaligned scratch
    assert call(sbytes=sc - 1) == N.DCA_ERR_ARG               # scratch too small
    assert call(lse=p + 2) == N.DCA_ERR_ARG                   # misaligned lse
    assert call(lq=N.DCA_DECODE_MAX_TOKENS + 1, q0=0, lk=600) == N.DCA_ERR_WORKSPACE
    assert call(lq=N.DCA_DECODE_MAX_TOKENS + 1, q0=0, lk=300) == N.DCA_ERR_ARG
    assert call(lk=600, q0=598) == N.DCA_ERR_WORKSPACE        # beyond the workspace capacity
    assert call(lq=0, q0=100) == N.DCA_OK                     # nothing to do, no launch


# ------------------------------------------------------------------ GPU


def dec(name, Lk, Lq, Hq, Hkv, s, w, c, yarn=1.0, dtype="bf16", sqrt_d=True):
    base = Workload(name, L=Lk, Hq=Hq, Hkv=Hkv, d=128, dtype=dtype, chunk_size=s,
                    local_window=w, pretrain_window=c, yarn_scale=yarn, scale_by_sqrt_d=sqrt_d)
    return DecodeWorkload(name, base, Lk=Lk, Lq=Lq)


CASES = [
    dec("far_r", 5000, 1, 28, 4, 1024, 128, 2048),                 # r_i >= w: SUCC at c - 1
    dec("near_r", 4147, 1, 28, 4, 1024, 128, 2048, yarn=4.0),      # r_i = 50 < w: SUCC at s + r_i
    dec("straddle", 4098, 3, 28, 4, 1024, 128, 2048),              # rows 4095..4097 cross a chunk
    dec("rowgroups", 3000, 5, 28, 4, 512, 64, 1024, yarn=2.0),     # 35 rows: 2 groups of 32
    dec("group32", 4147, 4, 28, 4, 1024, 128, 2048),              # 28 rows: one group of 32
    dec("group16_full", 2000, 2, 16, 2, 512, 64, 1024),           # exactly 16 rows
    dec("single_chunk", 700, 2, 8, 2, 1024, 64, 2048),
    dec("tiny_chunks", 300, 2, 2, 1, 3, 2, 5),
    dec("w0", 2500, 1, 4, 2, 256, 0, 256),
    dec("g1", 1500, 2, 8, 8, 256, 32, 512, sqrt_d=False),
    dec("one_key", 1, 1, 4, 1, 64, 8, 128),
    dec("sensitive", 6000, 4, 14, 2, 1536, 256, 2048, sqrt_d=False),
    dec("max_tokens", 700, N.DCA_DECODE_MAX_TOKENS, 4, 2, 256, 64, 512),
]


def run_decode(dw, seed=0, reading="query_offset", want_lse=True):
    w = dw.base
    q, k, v = generate_decode(dw, device=DEV, seed=seed)
    ws = dca.Workspace(dw.Lk, w.Hq, w.Hkv, 128, w.chunk_size, w.local_window, w.pretrain_window,
                       q.dtype, DEV)
    dca.prepare(k, kv_len=dw.Lk, k_rows_valid=0, chunk_size=w.chunk_size,
                local_window=w.local_window, pretrain_window=w.pretrain_window,
                rope_base=w.rope_base, workspace=ws)
    lse = torch.empty((dw.Lq, w.Hq), dtype=torch.float32, device=DEV) if want_lse else None
    out = dca.decode(q, v, q_start=dw.Lk - dw.Lq, kv_len=dw.Lk, chunk_size=w.chunk_size,
                     local_window=w.local_window, pretrain_window=w.pretrain_window,
                     yarn_scale=w.yarn_scale, workspace=ws, lse=lse, window_reading=reading)
    torch.cuda.synchronize()
    assert ws.status() == N.DCA_OK
    return q, k, v, out, lse


def oracle_decode(dw, q, k, v, reading=0, rows=None, heads=None):
    w = dw.base
    return oracle.attention(q.cpu(), k.cpu(), v.cpu(), chunk_size=w.chunk_size,
                            local_window=w.local_window, pretrain_window=w.pretrain_window,
                            rope_base=w.rope_base, yarn_scale=w.yarn_scale,
                            q_start=dw.Lk - dw.Lq, reading=reading, rows=rows, heads=heads,
                            return_lse=True)


def check_lse(got, want):
    """LSE (natural log of the softmax denominator) within 1e-2 absolute.
    The kernel rounds each rotated query to bf16 (relative 2^-9 per element),
    so a logit m^2 <q', k'>/sqrt(d) carries an error of standard deviation
    about 2^-9/sqrt(3) * ||q o k|| / sqrt(d), 1.1e-3 for unit-variance q and k;
    the LSE error is a softmax-weighted mean of those, and 1e-2 is about nine
    of them (the bf16 output's max-abs bound is 2e-2)."""
    g = got.double().cpu().numpy()
    assert np.all(np.isfinite(g))
    assert np.max(np.abs(g - want)) <= 1e-2, np.max(np.abs(g - want))


@pytest.mark.gpu
@pytest.mark.parametrize("dw", CASES, ids=lambda dw: dw.name)
@pytest.mark.parametrize("reading", ["query_offset", "true_distance"])
def test_decode_parity(dw, reading):
    from tests.gpu_helpers import assert_close
    q, k, v, out, lse = run_decode(dw, reading=reading)
    want, want_lse = oracle_decode(dw, q, k, v, reading=0 if reading == "query_offset" else 1)
    assert_close(out.double().cpu().numpy(), want, torch.bfloat16, dw.name)
    check_lse(lse, want_lse)


@pytest.mark.gpu
@pytest.mark.parametrize("reading", ["query_offset", "true_distance"])
def test_decode_f32(reading):
    from tests.gpu_helpers import assert_close
    dw = dec("f32", 2100, 3, 6, 2, 512, 64, 1024, yarn=2.0, dtype="f32", sqrt_d=False)
    q, k, v, out, lse = run_decode(dw, reading=reading)
    want, want_lse = oracle_decode(dw, q, k, v, reading=0 if reading == "query_offset" else 1)
    assert_close(out.double().cpu().numpy(), want, torch.float32, dw.name)
    assert np.max(np.abs(lse.double().cpu().numpy() - want_lse)) <= 1e-4


@pytest.mark.gpu
def test_decode_negative_control():
    """The decode output is far from an oracle with a wrong position map, so
    the parity comparison sees the DCA mapping at decode time too."""
    from tests.gpu_helpers import TOL, errors
    dw = dec("neg", 4147, 2, 8, 2, 1024, 128, 2048, sqrt_d=False)
    q, k, v, out, _ = run_decode(dw)
    got = out.double().cpu().numpy()
    w = dw.base
    for name in ("query_c", "key_not_periodic", "succ_as_inter"):
        bad = oracle.attention(q.cpu(), k.cpu(), v.cpu(), chunk_size=w.chunk_size,
                               local_window=w.local_window, pretrain_window=w.pretrain_window,
                               rope_base=w.rope_base, yarn_scale=w.yarn_scale,
                               q_start=dw.Lk - dw.Lq, mutation=oracle.MUTATIONS[name])
        assert errors(got, bad)[1] > 2 * TOL[torch.bfloat16]["rel_l2"], name


@pytest.mark.gpu
def test_decode_step_after_incremental_prepare():
    """decode_step (rotate the Lq new keys into a workspace that holds the
    earlier ones, then decode) equals decode after a full rebuild, bit for bit."""
    dw = dec("step", 3333, 2, 28, 4, 1024, 128, 2048, yarn=4.0)
    w = dw.base
    q, k, v = generate_decode(dw, device=DEV, seed=4)
    kw = dict(chunk_size=w.chunk_size, local_window=w.local_window,
              pretrain_window=w.pretrain_window)
    ws = dca.Workspace(dw.Lk, w.Hq, w.Hkv, 128, w.chunk_size, w.local_window, w.pretrain_window,
                       q.dtype, DEV)
    dca.prepare(k, kv_len=dw.Lk - dw.Lq, k_rows_valid=0, rope_base=w.rope_base, workspace=ws,
                **kw)
    got = dca.decode_step(q, k, v, kv_len=dw.Lk, rope_base=w.rope_base,
                          yarn_scale=w.yarn_scale, workspace=ws, **kw)
    ws2 = dca.Workspace(dw.Lk, w.Hq, w.Hkv, 128, w.chunk_size, w.local_window,
                        w.pretrain_window, q.dtype, DEV)
    dca.prepare(k, kv_len=dw.Lk, k_rows_valid=0, rope_base=w.rope_base, workspace=ws2, **kw)
    ref = dca.decode(q, v, q_start=dw.Lk - dw.Lq, kv_len=dw.Lk, yarn_scale=w.yarn_scale,
                     workspace=ws2, **kw)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


@pytest.mark.gpu
def test_decode_matches_prefill_rows():
    """The decode kernel and the prefill kernel agree on the last rows."""
    from tests.gpu_helpers import assert_close
    dw = dec("vs_prefill", 2600, 3, 28, 4, 512, 64, 1024, yarn=2.0)
    w = dw.base
    q, k, v = generate_decode(dw, device=DEV, seed=2)
    kw = dict(chunk_size=w.chunk_size, local_window=w.local_window,
              pretrain_window=w.pretrain_window, rope_base=w.rope_base, yarn_scale=w.yarn_scale)
    pre = dca.prefill_chunked(q, k, v, q_start=dw.Lk - dw.Lq, **kw)
    _, _, _, out, _ = run_decode(dw, seed=2, want_lse=False)
    assert_close(out.double().cpu().numpy(), pre.double().cpu().numpy(), torch.bfloat16)


@pytest.mark.gpu
def test_decode_timeout_reports_and_recovers():
    dw = dec("timeout", 5000, 1, 8, 2, 1024, 64, 2048)
    try:
        dca.set_wait_timeout_ns(50_000_000)
        dca.set_debug_flags(1)   # the next launch withholds its first key tile
        w = dw.base
        q, k, v = generate_decode(dw, device=DEV)
        ws = dca.Workspace(dw.Lk, w.Hq, w.Hkv, 128, w.chunk_size, w.local_window,
                           w.pretrain_window, q.dtype, DEV)
        kw = dict(chunk_size=w.chunk_size, local_window=w.local_window,
                  pretrain_window=w.pretrain_window)
        dca.prepare(k, kv_len=dw.Lk, k_rows_valid=0, rope_base=w.rope_base, workspace=ws, **kw)
        dca.decode(q, v, q_start=dw.Lk - 1, kv_len=dw.Lk, workspace=ws, **kw)
        assert ws.status() == N.DCA_ERR_TIMEOUT
    finally:
        dca.set_debug_flags(0)
        dca.set_wait_timeout_ns(10_000_000_000)
    q2, k2, v2, out, _ = run_decode(dw)
    from tests.gpu_helpers import assert_close
    want, _ = oracle_decode(dw, q2, k2, v2)
    assert_close(out.double().cpu().numpy(), want, torch.bfloat16, "after timeout")


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["qwen7b_1m_decode", "qwen7b_1m_decode_q4"])
def test_full_size_decode(name):
    """1M-token cache, the launch configuration the decode benchmark times;
    every row and head against the oracle."""
    from tests.gpu_helpers import assert_close
    dw = DECODE_WORKLOADS[name]
    q, k, v, out, lse = run_decode(dw)
    want, want_lse = oracle_decode(dw, q, k, v)
    assert_close(out.double().cpu().numpy(), want, torch.bfloat16, name)
    check_lse(lse, want_lse)
