"""Drive a whole DCA prefill workload through the library's staged C ABI.

A chunked prefill (the "Chunked Prefill" section of "Qwen2.5-1M 不重训外推
1M": 32,768-token query blocks against the growing KV cache) is, per block:
``dca_prepare`` (rotate the block's new keys into the workspace's rotated-key
cache; the RoPE table is built on the first block) then ``dca_attend`` (the
fused attention kernel).  A one-shot prefill is the single block
(0, L, L).  The benchmark and the full-size parity tests both run this.
"""
from __future__ import annotations

from typing import List, Optional

import torch

from . import api
from .workloads import Workload


def make_workspace(w: Workload, device, kv_capacity: Optional[int] = None) -> api.Workspace:
    return api.Workspace(w.L if kv_capacity is None else kv_capacity, w.Hq, w.Hkv, w.d,
                         w.chunk_size, w.local_window, w.pretrain_window, w.torch_dtype, device)


def run_workload(w: Workload, q, k, v, out, ws: api.Workspace,
                 attn_events: Optional[List] = None, L: Optional[int] = None):
    """Run every block of ``w`` (or of a shorter length ``L``).

    q, out [L, Hq, d]; k, v [L, Hkv, d] on the device.  When ``attn_events``
    is a list, a (start, end) pair of CUDA events is recorded around each
    attention launch on the current stream.
    """
    L = w.L if L is None else L
    blocks = w.blocks() if L == w.L else [
        (q0, min(w.block or L, L - q0), q0 + min(w.block or L, L - q0))
        for q0 in range(0, L, w.block or L)]
    p = w.params()
    for q0, lq, lk in blocks:
        api.prepare(k, kv_len=lk, k_rows_valid=q0, chunk_size=p["chunk_size"],
                    local_window=p["local_window"], pretrain_window=p["pretrain_window"],
                    rope_base=p["rope_base"], workspace=ws)
        ev = None
        if attn_events is not None:
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            ev[0].record()
        api.attend(q[q0:q0 + lq], v, out[q0:q0 + lq], q_start=q0, kv_len=lk,
                   chunk_size=p["chunk_size"], local_window=p["local_window"],
                   pretrain_window=p["pretrain_window"], yarn_scale=p["yarn_scale"],
                   workspace=ws)
        if ev is not None:
            ev[1].record()
            attn_events.append(ev)
    return out
