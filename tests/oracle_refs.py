"""Independent textbook references used to pin the oracle (test-only).

Nothing here shares code with the oracle: RoPE is written as a complex
multiplication (the RoFormer formulation) and causal attention is torch's
library ``scaled_dot_product_attention`` in float64.
"""
from __future__ import annotations

import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def rope_freqs(d: int, base: float) -> np.ndarray:
    return base ** (-np.arange(d // 2, dtype=np.float64) * 2.0 / d)


def rope_complex(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rotate [L, H, d] by per-row positions, pairs (k, k + d/2) as one complex number."""
    d = x.shape[-1]
    h = d // 2
    z = x[..., :h] + 1j * x[..., h:]
    z = z * np.exp(1j * np.asarray(pos, dtype=np.float64)[:, None, None] * rope_freqs(d, base)[None, None, :])
    return np.concatenate([z.real, z.imag], axis=-1)


def causal_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """Library causal softmax attention, GQA by consecutive head groups."""
    G = q.shape[1] // k.shape[1]
    qt = torch.from_numpy(np.ascontiguousarray(q)).permute(1, 0, 2)[None]
    kt = torch.from_numpy(np.ascontiguousarray(np.repeat(k, G, axis=1))).permute(1, 0, 2)[None]
    vt = torch.from_numpy(np.ascontiguousarray(np.repeat(v, G, axis=1))).permute(1, 0, 2)[None]
    o = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


def rope_attention(q, k, v, base, scale):
    """Standard causal RoPE attention with true positions 0..L-1."""
    L = q.shape[0]
    pos = np.arange(L)
    return causal_attention(rope_complex(q, pos, base), rope_complex(k, pos, base), v, scale)


def relative_logits(q: np.ndarray, k: np.ndarray, D: np.ndarray, base: float, scale: float):
    """logit[i, j] = scale * Re sum_k qc_k conj(kc_k) exp(i D[i,j] theta_k)  (one head each).

    Uses only the relative-distance property of RoPE: <R(a)q, R(b)k> = <R(a-b)q, k>."""
    d = q.shape[-1]
    h = d // 2
    qc = q[:, :h] + 1j * q[:, h:]
    kc = k[:, :h] + 1j * k[:, h:]
    th = rope_freqs(d, base)
    prod = qc[:, None, :] * np.conj(kc)[None, :, :]            # [Lq, Lk, h]
    return scale * np.real(np.sum(prod * np.exp(1j * D[:, :, None] * th), axis=-1))


def read_golden_map(name: str):
    """Parse a hand-worked position-map fixture -> list of (i, Pq[], Pk[], cls[])."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = [p.split() for p in line.split("|")]
            i = int(parts[0][0])
            rows.append((i, [int(x) for x in parts[1]], [int(x) for x in parts[2]],
                         [int(x) for x in parts[3]]))
    return rows


def read_page_constants():
    out = {}
    with open(os.path.join(GOLDEN, "page_constants.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, val = line.split("|")[0].split()
            out[name] = float(val)
    return out
