"""Comparison helpers and tolerances for the GPU parity tests.

Tolerances (stated for this method's outputs): bf16 inputs -> max-abs error
<= 2e-2 and relative L2 error <= 5e-3 against the fp64 oracle; fp32 inputs ->
1e-4 for both (applied strictly).
"""
import numpy as np
import torch

TOL = {
    torch.bfloat16: dict(max_abs=2e-2, rel_l2=5e-3),
    torch.float32: dict(max_abs=1e-4, rel_l2=1e-4),
}


def errors(got, want):
    g = np.asarray(got, dtype=np.float64)
    w = np.asarray(want, dtype=np.float64)
    diff = g - w
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    denom = float(np.linalg.norm(w.ravel()))
    rel = float(np.linalg.norm(diff.ravel()) / denom) if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_close(got, want, dtype, what=""):
    tol = TOL[dtype]
    ma, rl = errors(got, want)
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), f"{what}: non-finite output"
    assert ma <= tol["max_abs"] and rl <= tol["rel_l2"], (
        f"{what}: max_abs {ma:.3e} (tol {tol['max_abs']}), rel_l2 {rl:.3e} (tol {tol['rel_l2']})")
    return ma, rl


def gather(out, rows, heads):
    """out [L, Hq, d] (device) -> fp64 numpy [len(rows), len(heads), d]."""
    r = torch.as_tensor(rows, device=out.device, dtype=torch.long)
    h = torch.as_tensor(heads, device=out.device, dtype=torch.long)
    return out.index_select(0, r).index_select(1, h).double().cpu().numpy()
