"""Named DCA prefill workloads and their seeded synthetic inputs.

This module holds sizes, parameters and random-number recipes only; none of
the attention arithmetic.  Both the CUDA path (tests, benchmark) and the fp64
oracle (tests) draw their inputs from here, so the two sides see identical
tensors.

Workload shapes follow the pages on Qwen2.5-1M: GQA head counts of the 7B
and 14B models ("Qwen-2.5 explained", section 三), RoPE base 10,000,000
(news article on the Qwen2.5-1M release, section "如何炼成的？"), and the
32,768-token query blocks of chunked prefill ("Qwen2.5-1M 不重训外推 1M",
section "Chunked Prefill").  No evaluation dataset is used: every tensor is
drawn i.i.d. from a seeded normal distribution.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

ROPE_BASE = 10_000_000.0
CHUNKED_PREFILL_BLOCK = 32_768


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    L: int                 # total sequence length
    Hq: int
    Hkv: int
    d: int
    dtype: str             # "bf16" or "f32"
    chunk_size: int
    local_window: int
    pretrain_window: int
    rope_base: float = ROPE_BASE
    yarn_scale: float = 1.0
    scale_by_sqrt_d: bool = True   # N(0,1)/sqrt(d) when True, N(0,1) otherwise
    sink_fraction: float = 0.0     # fraction of keys scaled up (attention sinks)
    sink_scale: float = 1.0
    block: Optional[int] = None    # chunked prefill: query block length

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def G(self):
        return self.Hq // self.Hkv

    def attention_flops(self) -> float:
        """4*d*Hq per unmasked causal (query, key) pair, summed over all pairs."""
        return 4.0 * self.d * self.Hq * self.L * (self.L + 1) / 2.0

    def blocks(self):
        """(q_start, Lq, Lk) of every call of a chunked prefill (one call if block is None)."""
        if self.block is None:
            return [(0, self.L, self.L)]
        out = []
        for q0 in range(0, self.L, self.block):
            lq = min(self.block, self.L - q0)
            out.append((q0, lq, q0 + lq))
        return out

    def params(self):
        return dict(chunk_size=self.chunk_size, local_window=self.local_window,
                    pretrain_window=self.pretrain_window, rope_base=self.rope_base,
                    yarn_scale=self.yarn_scale)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_f32_4k", L=4096, Hq=4, Hkv=1, d=128, dtype="f32",
                 chunk_size=1024, local_window=128, pretrain_window=2048,
                 yarn_scale=1.0, scale_by_sqrt_d=False),
        Workload("qwen7b_32k", L=32768, Hq=28, Hkv=4, d=128, dtype="bf16",
                 chunk_size=8192, local_window=1024, pretrain_window=16384,
                 yarn_scale=1.0, sink_fraction=0.01, sink_scale=8.0),
        Workload("qwen14b_128k", L=131072, Hq=40, Hkv=8, d=128, dtype="bf16",
                 chunk_size=32768, local_window=4096, pretrain_window=65536,
                 yarn_scale=2.0),
        Workload("qwen7b_256k", L=262144, Hq=28, Hkv=4, d=128, dtype="bf16",
                 chunk_size=65536, local_window=8192, pretrain_window=131072,
                 yarn_scale=2.0),
        Workload("qwen7b_1m_chunked", L=1048576, Hq=28, Hkv=4, d=128, dtype="bf16",
                 chunk_size=196608, local_window=32768, pretrain_window=262144,
                 yarn_scale=4.0, block=CHUNKED_PREFILL_BLOCK),
    ]
}

ORDER = ["tiny_f32_4k", "qwen7b_32k", "qwen14b_128k", "qwen7b_256k", "qwen7b_1m_chunked"]


def generate(w: Workload, device="cpu", seed: int = 0, L: Optional[int] = None):
    """Seeded q [L,Hq,d], k [L,Hkv,d], v [L,Hkv,d] in the workload's dtype.

    Draw order from one generator: q, then k, then v, then the sink key
    indices (the first floor(fraction*L) entries of a random permutation).
    Values are drawn in fp32, scaled, then rounded to the storage dtype
    (round-to-nearest-even).  ``L`` overrides the length (smaller test cases
    that keep the workload's other parameters).
    """
    L = w.L if L is None else L
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    q = _draw(w, g, L, w.Hq, device)
    k = _draw(w, g, L, w.Hkv, device)
    v = _draw(w, g, L, w.Hkv, device)
    _add_sinks(w, g, k, device)
    return q, k, v


def _draw(w: Workload, g, rows: int, H: int, device):
    """[rows, H, d] i.i.d. normal (scaled by 1/sqrt(d) when the workload says
    so), drawn in fp32 per slab and rounded to the storage dtype."""
    scale = 1.0 / math.sqrt(w.d) if w.scale_by_sqrt_d else 1.0
    x = torch.empty((rows, H, w.d), dtype=w.torch_dtype, device=device)
    # draw per slab to bound the fp32 temporary at full size
    step = max(1, (1 << 27) // max(1, H * w.d))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        t = torch.randn((r1 - r0, H, w.d), generator=g, device=device, dtype=torch.float32)
        if scale != 1.0:
            t.mul_(scale)
        x[r0:r1] = t.to(w.torch_dtype)
        del t
    return x


def _add_sinks(w: Workload, g, k, device):
    """Scale the keys at the first floor(fraction * rows) entries of a random permutation."""
    n = k.shape[0]
    n_sinks = int(math.floor(w.sink_fraction * n))
    if n_sinks > 0:
        idx = torch.randperm(n, generator=g, device=device)[:n_sinks]
        k[idx] = (k[idx].float() * w.sink_scale).to(w.torch_dtype)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """A decode step: Lq new query tokens at positions [Lk - Lq, Lk) against a
    cache of Lk keys, with the DCA parameters and head shapes of `base`."""
    name: str
    base: Workload
    Lk: int
    Lq: int

    def kv_bytes(self) -> int:
        """Bytes of rotated keys and values one step streams (all KV heads)."""
        esize = 2 if self.base.dtype == "bf16" else 4
        return 2 * self.Lk * self.base.Hkv * self.base.d * esize


def generate_decode(dw: DecodeWorkload, device="cpu", seed: int = 0):
    """Seeded q [Lq,Hq,d] (the new tokens), k, v [Lk,Hkv,d]: the draws of
    ``generate`` in the same order (q, k, v, sink indices) with q holding only
    the Lq new rows."""
    w = dw.base
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    q = _draw(w, g, dw.Lq, w.Hq, device)
    k = _draw(w, g, dw.Lk, w.Hkv, device)
    v = _draw(w, g, dw.Lk, w.Hkv, device)
    _add_sinks(w, g, k, device)
    return q, k, v


def sample_rows(w: Workload, q_start: int, Lq: int, n_random: int = 64, seed: int = 0):
    """Block-relative rows for sampled parity / CPU timing at full size.

    Per chunk touched by the block: offsets 0, 1, w-1, w and s-1 of the chunk,
    the block's first and last rows, plus ``n_random`` seeded uniform rows.
    """
    s, lw = w.chunk_size, w.local_window
    q_end = q_start + Lq
    rows = {q_start, q_start + 1, q_end - 1, q_end - 2}
    for n in range(q_start // s, (q_end - 1) // s + 1):
        for off in (0, 1, lw - 1, lw, lw + 1, s - 1):
            i = n * s + off
            if q_start <= i < q_end:
                rows.add(i)
    g = torch.Generator().manual_seed(seed + 1)
    for i in torch.randint(q_start, q_end, (n_random,), generator=g).tolist():
        rows.add(i)
    rows = sorted(r - q_start for r in rows if q_start <= r < q_end)
    return torch.tensor(rows, dtype=torch.int64)


def sample_heads(w: Workload):
    """Heads 0, G-1, G, Hq-1 (first/last head of the first two KV groups and the last head)."""
    hs = sorted({0, w.G - 1, min(w.G, w.Hq - 1), w.Hq - 1})
    return torch.tensor(hs, dtype=torch.int32)


# Decode steps after the prefills above: the next token (Lq = 1), and four
# tokens at once (e.g. verifying draft tokens), at the full context length.
DECODE_WORKLOADS = {
    dw.name: dw
    for dw in [
        DecodeWorkload("qwen7b_32k_decode", WORKLOADS["qwen7b_32k"], Lk=32768, Lq=1),
        DecodeWorkload("qwen7b_256k_decode", WORKLOADS["qwen7b_256k"], Lk=262144, Lq=1),
        DecodeWorkload("qwen7b_1m_decode", WORKLOADS["qwen7b_1m_chunked"], Lk=1048576, Lq=1),
        DecodeWorkload("qwen7b_1m_decode_q4", WORKLOADS["qwen7b_1m_chunked"], Lk=1048576, Lq=4),
    ]
}


def sparse_pattern(L: int, Hq: int, n_vertical: int, n_band: int, n_far: int, n_init: int = 4,
                   seed: int = 0):
    """Seeded synthetic vertical-slash pattern per query head (lists of sorted
    key indices and diagonal offsets in [0, L)).  Vertical keys: the first
    n_init tokens plus uniform random others; slash offsets: the band
    0 .. n_band - 1 (local diagonals) plus n_far uniform random far offsets.
    The real per-head patterns are searched offline on calibration data."""
    import numpy as np
    rng = np.random.default_rng(seed + 1000)
    vertical, slash = [], []
    for _ in range(Hq):
        nv = min(n_vertical, L)
        init = np.arange(min(n_init, nv))
        rest = rng.choice(np.arange(len(init), L), size=max(0, min(nv - len(init), L - len(init))),
                          replace=False) if nv > len(init) else np.zeros(0, np.int64)
        vertical.append(np.unique(np.concatenate([init, rest])).astype(np.int64))
        band = np.arange(min(n_band, L))
        far = rng.choice(np.arange(len(band), L), size=max(0, min(n_far, L - len(band))),
                         replace=False) if L > len(band) and n_far > 0 else np.zeros(0, np.int64)
        slash.append(np.unique(np.concatenate([band, far])).astype(np.int64))
    return vertical, slash


@dataclasses.dataclass(frozen=True)
class SparseWorkload:
    """A vertical-slash sparse prefill: the DCA parameters, shapes and query
    blocks of `base`, and per query head n_vertical vertical keys (the first
    4 tokens plus random others), a band of n_band local diagonals and n_far
    random far diagonals."""
    name: str
    base: Workload
    n_vertical: int
    n_band: int
    n_far: int


def generate_sparse(sw: SparseWorkload, seed: int = 0):
    """The workload's seeded per-head (vertical, slash) lists."""
    return sparse_pattern(sw.base.L, sw.base.Hq, sw.n_vertical, sw.n_band, sw.n_far, seed=seed)


# Pattern sizes in the range the sparse-attention literature uses at these
# lengths (about a thousand key columns and a few thousand diagonals per head).
SPARSE_WORKLOADS = {
    sw.name: sw
    for sw in [
        SparseWorkload("qwen7b_32k_sparse", WORKLOADS["qwen7b_32k"], 1000, 4096, 64),
        SparseWorkload("qwen7b_256k_sparse", WORKLOADS["qwen7b_256k"], 1000, 4096, 64),
        SparseWorkload("qwen7b_1m_sparse", WORKLOADS["qwen7b_1m_chunked"], 1000, 4096, 64),
    ]
}
