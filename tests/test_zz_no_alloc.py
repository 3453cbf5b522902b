"""dca_prefill_noalloc: the one-shot prefill for callers that cannot allocate
device memory (for example a serving process whose own pool took all free HBM
at start-up, or a plugin whose host framework owns every allocation).

Called through the C ABI, it must give the same result as the workspace entry
point dca_prefill, within the parity tolerance, on two calls in a row (the
second call reuses the scratch the first one left behind), and refuse a
problem larger than its fixed scratch before launching anything.  Collected
last so that a run stopping at its first failure has run every other test.
"""
import pytest
import torch

from length_extrapolation_b200 import _native as N
from length_extrapolation_b200 import build as B
from length_extrapolation_b200.workloads import Workload, generate
from tests.gpu_helpers import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SCRATCH_BYTES = 32 * 1024 * 1024  # DCA_NOALLOC_SCRATCH_BYTES in include/dca.h


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    return N.lib()


def _stream():
    return torch.cuda.current_stream(DEV).cuda_stream


def _args(w):
    return (w.Hq, w.Hkv, w.d, w.chunk_size, w.local_window, w.pretrain_window, w.rope_base,
            w.yarn_scale, 0)


def _with_workspace(lib, w, q, k, v):
    out = torch.empty_like(q)
    n = lib.dca_workspace_size(w.L, w.Hq, w.Hkv, w.d, w.chunk_size, w.local_window,
                               w.pretrain_window, 0)
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    rc = lib.dca_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), w.L,
                         *_args(w), ws.data_ptr(), n, _stream())
    assert rc == N.DCA_OK, N.status_string(rc)
    return out


def _no_alloc(lib, w, q, k, v):
    out = torch.empty_like(q)
    rc = lib.dca_prefill_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), w.L,
                                 *_args(w), _stream())
    assert rc == N.DCA_OK, N.status_string(rc)
    return out


def test_no_alloc_matches_workspace_entry_twice(lib):
    cases = [
        Workload("na1", L=3000, Hq=7, Hkv=1, d=128, dtype="bf16", chunk_size=1024,
                 local_window=256, pretrain_window=1536, yarn_scale=2.0, scale_by_sqrt_d=False),
        Workload("na2", L=1337, Hq=4, Hkv=2, d=128, dtype="bf16", chunk_size=300,
                 local_window=64, pretrain_window=400, yarn_scale=1.0, scale_by_sqrt_d=False),
    ]
    for seed, w in enumerate(cases):  # two calls in a row, different shapes and contents
        q, k, v = generate(w, device=DEV, seed=seed)
        want = _with_workspace(lib, w, q, k, v)
        got = _no_alloc(lib, w, q, k, v)
        torch.cuda.synchronize()
        assert_close(got.double().cpu().numpy(), want.double().cpu().numpy(), torch.bfloat16,
                     f"no-alloc call {seed + 1}")


def test_no_alloc_rejects_problems_beyond_scratch(lib):
    w = Workload("big", L=65536, Hq=28, Hkv=4, d=128, dtype="bf16", chunk_size=8192,
                 local_window=1024, pretrain_window=16384)
    assert lib.dca_workspace_size(w.L, w.Hq, w.Hkv, w.d, w.chunk_size, w.local_window,
                                  w.pretrain_window, 0) > SCRATCH_BYTES
    p = 1 << 20  # never dereferenced: the size check comes first
    rc = lib.dca_prefill_noalloc(p, p, p, p, w.L, *_args(w), _stream())
    assert rc == N.DCA_ERR_WORKSPACE
