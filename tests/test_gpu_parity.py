"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small cases: every output element, sizes spanning several 128-row tiles with
ragged tails, chunk sizes that are not tile multiples (mixed-class tiles),
odd GQA groups, YaRN on and off.  Full-size workloads: sampled rows and heads
(the oracle computes them one by one), run in the same staged launch sequence
that the benchmark times.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import length_extrapolation_b200 as dca
from length_extrapolation_b200 import _native as N
from length_extrapolation_b200 import build as B
from length_extrapolation_b200 import runner
from length_extrapolation_b200.workloads import WORKLOADS, Workload, generate, sample_heads, sample_rows
from tests.gpu_helpers import TOL, assert_close, errors, gather

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    N.lib()


def small(name, L, Hq, Hkv, s, w, c, yarn=1.0, dtype="bf16", sqrt_d=True):
    return Workload(name, L=L, Hq=Hq, Hkv=Hkv, d=128, dtype=dtype, chunk_size=s, local_window=w,
                    pretrain_window=c, yarn_scale=yarn, scale_by_sqrt_d=sqrt_d)


SMALL = [
    small("ragged_mixed", 1000, 4, 1, 300, 50, 400),
    small("g7_yarn2", 777, 7, 1, 256, 128, 512, yarn=2.0),
    small("g5_yarn4", 2048, 10, 2, 512, 128, 1024, yarn=4.0),
    small("g1_w0", 130, 2, 2, 64, 0, 64),
    small("w_eq_s", 900, 2, 1, 200, 200, 400),
    small("single_chunk", 384, 4, 2, 384, 16, 512),
    small("tiny_chunks", 300, 2, 1, 3, 2, 5),
    small("one_token", 1, 3, 1, 64, 8, 128),
    small("sensitive_N01", 1500, 4, 1, 384, 128, 640, sqrt_d=False),
    small("f32_small", 700, 3, 1, 200, 40, 300, dtype="f32", sqrt_d=False),
]


def run_small(w, seed=0):
    q, k, v = generate(w, device=DEV, seed=seed)
    out = dca.prefill(q, k, v, **w.params())
    torch.cuda.synchronize()
    return q, k, v, out


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_all_rows(w):
    q, k, v, out = run_small(w)
    want = oracle.attention(q.cpu(), k.cpu(), v.cpu(), **w.params())
    assert_close(out.double().cpu().numpy(), want, w.torch_dtype, w.name)


def test_tiny_f32_workload_all_rows():
    w = WORKLOADS["tiny_f32_4k"]
    q, k, v, out = run_small(w)
    want = oracle.attention(q.cpu(), k.cpu(), v.cpu(), **w.params())
    ma, rl = assert_close(out.double().cpu().numpy(), want, torch.float32, w.name)
    print(f"tiny_f32_4k: max_abs {ma:.2e} rel_l2 {rl:.2e}")


def test_negative_controls_see_the_mapping():
    """On inputs with O(1) logits the GPU output differs from oracles with a
    deliberately wrong position map by far more than the tolerance, so the
    parity comparison does see the DCA mapping."""
    w = small("neg", 1024, 2, 1, 256, 64, 384, sqrt_d=False)
    q, k, v, out = run_small(w)
    got = out.double().cpu().numpy()
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    _, rl_ok = errors(got, oracle.attention(qc, kc, vc, **w.params()))
    assert rl_ok <= TOL[torch.bfloat16]["rel_l2"]
    for name in ("query_c", "key_not_periodic", "succ_as_inter", "sin_sign", "pair_adjacent"):
        bad = oracle.attention(qc, kc, vc, mutation=oracle.MUTATIONS[name], **w.params())
        _, rl = errors(got, bad)
        assert rl > 10 * rl_ok and rl > 2 * TOL[torch.bfloat16]["rel_l2"], (name, rl, rl_ok)
    # r_i <= w instead of r_i < w changes one query row per chunk: smaller, but
    # still outside the tolerance band
    bad = oracle.attention(qc, kc, vc, mutation=oracle.MUTATIONS["window_le"], **w.params())
    assert errors(got, bad)[1] > 2 * TOL[torch.bfloat16]["rel_l2"]
    bad = oracle.attention(qc, kc, vc, reading=1, **w.params())
    assert errors(got, bad)[1] > 2 * TOL[torch.bfloat16]["rel_l2"]


# Window reading B (true distance kept iff i - j < w): the same small shapes,
# plus the reading's own degenerate cases.  Reading B differs from reading A
# only in which successive-chunk pairs keep the true distance.
READING_B = [
    small("B_ragged_mixed", 1000, 4, 1, 300, 50, 400),
    small("B_g7_yarn2", 777, 7, 1, 256, 128, 512, yarn=2.0),
    small("B_w_eq_s", 900, 2, 1, 200, 200, 400),
    small("B_w0", 400, 2, 2, 64, 0, 64),          # no pair keeps its true distance across chunks
    small("B_w1", 520, 2, 1, 128, 1, 160),        # only j = i - 1 at a chunk start
    small("B_odd_window", 1100, 4, 2, 256, 77, 400, sqrt_d=False),
    small("B_tiny_chunks", 300, 2, 1, 3, 2, 5),
    small("B_single_chunk", 384, 4, 2, 384, 16, 512),
    small("B_f32", 700, 3, 1, 200, 40, 300, dtype="f32", sqrt_d=False),
]


@pytest.mark.parametrize("w", READING_B, ids=lambda w: w.name)
def test_reading_b_all_rows(w):
    q, k, v = generate(w, device=DEV, seed=3)
    out = dca.prefill(q, k, v, window_reading="true_distance", **w.params())
    torch.cuda.synchronize()
    want = oracle.attention(q.cpu(), k.cpu(), v.cpu(), reading=1, **w.params())
    assert_close(out.double().cpu().numpy(), want, w.torch_dtype, w.name)


def test_reading_b_differs_from_a():
    """The two readings give measurably different outputs on O(1) logits, and
    each kernel option matches its own oracle reading, not the other."""
    w = small("AB", 1024, 2, 1, 256, 64, 384, sqrt_d=False)
    q, k, v = generate(w, device=DEV, seed=5)
    outs = {r: dca.prefill(q, k, v, window_reading=r, **w.params()).double().cpu().numpy()
            for r in ("query_offset", "true_distance")}
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    want = {r: oracle.attention(qc, kc, vc, reading=i, **w.params())
            for i, r in enumerate(("query_offset", "true_distance"))}
    tol = TOL[torch.bfloat16]["rel_l2"]
    for r in outs:
        assert errors(outs[r], want[r])[1] <= tol
        other = "true_distance" if r == "query_offset" else "query_offset"
        assert errors(outs[r], want[other])[1] > 2 * tol


def test_reading_b_chunked_blocks_equal_oneshot():
    w = small("B_chunked", 1300, 4, 2, 256, 100, 512)
    q, k, v = generate(w, device=DEV, seed=7)
    one = dca.prefill(q, k, v, window_reading="true_distance", **w.params())
    ws = dca.Workspace(w.L, w.Hq, w.Hkv, 128, w.chunk_size, w.local_window, w.pretrain_window,
                       q.dtype, DEV)
    blk = torch.empty_like(q)
    for q0 in range(0, w.L, 256):       # tile-aligned blocks: the same tiles as one-shot
        lq = min(256, w.L - q0)
        dca.prefill_chunked(q[q0:q0 + lq], k, v, q_start=q0, kv_len=q0 + lq, workspace=ws,
                            out=blk[q0:q0 + lq], window_reading="true_distance", **w.params())
    torch.cuda.synchronize()
    assert torch.equal(one, blk)


@pytest.mark.parametrize("aligned", [True, False])
def test_chunked_blocks_equal_oneshot(aligned):
    w = small("chunk", 1280, 4, 2, 320, 64, 512, yarn=2.0)
    q, k, v, full = run_small(w)
    blk = 256 if aligned else 200
    parts = []
    for q0 in range(0, w.L, blk):
        lq = min(blk, w.L - q0)
        parts.append(dca.prefill_chunked(q[q0:q0 + lq], k[:q0 + lq], v[:q0 + lq], q_start=q0,
                                         **w.params()))
    got = torch.cat(parts)
    torch.cuda.synchronize()
    if aligned:
        assert torch.equal(got, full)
    else:
        assert_close(got.double().cpu().numpy(), full.double().cpu().numpy(), torch.bfloat16)


def test_incremental_prepare_equals_full_rebuild():
    w = Workload("inc", L=1536, Hq=4, Hkv=1, d=128, dtype="bf16", chunk_size=512,
                 local_window=64, pretrain_window=640, yarn_scale=2.0, block=384)
    q, k, v = generate(w, device=DEV)
    ws = runner.make_workspace(w, DEV)
    out = torch.empty_like(q)
    runner.run_workload(w, q, k, v, out, ws)
    ref = dca.prefill(q, k, v, **w.params())
    torch.cuda.synchronize()
    assert ws.status() == N.DCA_OK
    assert torch.equal(out, ref)


def test_host_entry_matches_device_path():
    w = Workload("host", L=1000, Hq=4, Hkv=2, d=128, dtype="bf16", chunk_size=256,
                 local_window=32, pretrain_window=384, yarn_scale=1.5, block=256)
    q, k, v = generate(w, device="cpu")
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty_like(qh).pin_memory()
    n = dca.host_arena_size(w.L, w.block, w.Hq, w.Hkv, w.d, w.chunk_size, w.local_window,
                            w.pretrain_window, torch.bfloat16)
    arena = torch.empty(n, dtype=torch.uint8, device=DEV)
    dca.prefill_host(qh, kh, vh, oh, block=w.block, arena=arena, **w.params())
    torch.cuda.synchronize()
    dev = torch.empty_like(q, device=DEV)
    ws = runner.make_workspace(w, DEV)
    runner.run_workload(w, q.to(DEV), k.to(DEV), v.to(DEV), dev, ws)
    torch.cuda.synchronize()
    assert torch.equal(oh, dev.cpu())


def test_bounded_wait_timeout_reports_and_recovers():
    """Withhold one TMA load: every wait of the kernel runs out after the short
    limit, the kernel exits cleanly and the status word reports the timeout;
    the context stays usable."""
    w = small("timeout", 512, 2, 1, 128, 32, 256)
    q, k, v = generate(w, device=DEV)
    ws = runner.make_workspace(w, DEV)
    out = torch.zeros_like(q)
    dca.set_wait_timeout_ns(20_000_000)
    try:
        dca.set_debug_flags(1)
        dca.prefill(q, k, v, workspace=ws, out=out, **w.params())
        assert ws.status() == N.DCA_ERR_TIMEOUT
    finally:
        dca.set_debug_flags(0)
        dca.set_wait_timeout_ns(0)
    out2 = dca.prefill(q, k, v, workspace=ws, **w.params())
    assert ws.status() == N.DCA_OK
    want = oracle.attention(q.cpu(), k.cpu(), v.cpu(), **w.params())
    assert_close(out2.double().cpu().numpy(), want, torch.bfloat16)


def test_empty_block_is_a_no_op():
    w = small("empty", 256, 2, 1, 128, 32, 256)
    q, k, v = generate(w, device=DEV)
    out = torch.full_like(q, 7.0)
    dca.prefill_chunked(q[:0], k, v, q_start=100, out=out[:0], **w.params())
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


# ------------------------------------------------------------------ full size
def _rows_to_check(w, q0, lq, n_random, max_rows):
    """Block-relative rows: every chunk-structure row of sample_rows (chunk
    offsets 0, 1, w-1, w, w+1, s-1 and the block's edges) first, then its
    seeded random rows up to max_rows in total."""
    structural = sample_rows(w, q0, lq, n_random=0).numpy()
    extra = np.setdiff1d(sample_rows(w, q0, lq, n_random=n_random).numpy(), structural)
    if max_rows is not None:
        extra = extra[:max(0, max_rows - len(structural))]
    return np.union1d(structural, extra)


def _full_size_check(name, max_rows=None, n_random=48, blocks_to_check=None):
    w = WORKLOADS[name]
    q, k, v = generate(w, device=DEV)
    ws = runner.make_workspace(w, DEV)
    out = torch.empty_like(q)
    runner.run_workload(w, q, k, v, out, ws)
    assert ws.status() == N.DCA_OK
    heads = sample_heads(w).numpy()
    kc, vc = k.cpu(), v.cpu()
    blocks = w.blocks()
    if blocks_to_check is not None:
        blocks = [blocks[b] for b in blocks_to_check]
    worst = (0.0, 0.0)
    for q0, lq, lk in blocks:
        rows = _rows_to_check(w, q0, lq, n_random, max_rows)
        want = oracle.attention(q[q0:q0 + lq].cpu(), kc[:lk], vc[:lk], q_start=q0, rows=rows,
                                heads=heads, **w.params())
        got = gather(out[q0:q0 + lq], rows, heads)
        ma, rl = assert_close(got, want, w.torch_dtype, f"{name} block q0={q0}")
        worst = (max(worst[0], ma), max(worst[1], rl))
    print(f"{name}: worst max_abs {worst[0]:.2e} rel_l2 {worst[1]:.2e}")


def test_full_size_qwen7b_32k():
    _full_size_check("qwen7b_32k")


def test_full_size_qwen14b_128k():
    _full_size_check("qwen14b_128k", max_rows=48, n_random=24)


def test_full_size_qwen7b_256k():
    _full_size_check("qwen7b_256k", max_rows=40, n_random=16)


def test_full_size_qwen7b_1m_chunked():
    """All 32 query blocks run on the GPU; five are checked on sampled rows.
    Block 0 lies in chunk 0 (intra pairs only).  Blocks 6 and 30 start at the
    starts of chunks 1 and 5, so every row has r_i < w: their pairs with the
    previous chunk keep the true distance, with queries rotated by s + r_i up
    to s + w - 1 = 229,375 (the largest table position below c - 1); block 30
    also has inter-chunk pairs against chunks 0-3.  Blocks 13 and 31 start at
    offset 32,768 = w of chunks 2 and 5: their previous-chunk pairs take the
    inter rule."""
    w = WORKLOADS["qwen7b_1m_chunked"]
    s, lw, blk = w.chunk_size, w.local_window, w.block
    for b, want_succ_true in ((6, True), (30, True), (13, False), (31, False)):
        q0 = b * blk
        r0, r1 = q0 % s, (q0 + blk - 1) % s
        assert (r1 < lw) == want_succ_true and (r0 >= lw) == (not want_succ_true)
    _full_size_check("qwen7b_1m_chunked", max_rows=12, n_random=4,
                     blocks_to_check=[0, 6, 13, 30, 31])
