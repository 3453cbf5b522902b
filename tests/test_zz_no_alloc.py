"""dca_prefill_noalloc: the one-shot prefill for callers that cannot allocate
device memory (for example a serving process whose own pool took all free HBM
at start-up, or a plugin whose host framework owns every allocation).

Called through the C ABI after dca_noalloc_prepare, it must give exactly the
result of the workspace entry point dca_prefill (both run the same kernels on
the same inputs, so the outputs are compared for equality) on two calls in a
row, in bf16 and fp32 (the second call reuses the scratch the first one left
behind); refuse a problem larger than its fixed scratch, or a bad argument,
before touching the scratch; and report a bounded-wait timeout through
dca_noalloc_device_status, after which the next call is clean.  Collected
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
    L = N.lib()
    torch.cuda.set_device(DEV)
    assert L.dca_noalloc_prepare() == N.DCA_OK
    return L


def _stream():
    return torch.cuda.current_stream(DEV).cuda_stream


def _dt(w):
    return N.DCA_BF16 if w.dtype == "bf16" else N.DCA_F32


def _args(w):
    return (w.Hq, w.Hkv, w.d, w.chunk_size, w.local_window, w.pretrain_window, w.rope_base,
            w.yarn_scale, _dt(w))


def _with_workspace(lib, w, q, k, v):
    out = torch.empty_like(q)
    n = lib.dca_workspace_size(w.L, w.Hq, w.Hkv, w.d, w.chunk_size, w.local_window,
                               w.pretrain_window, _dt(w))
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    rc = lib.dca_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), w.L,
                         *_args(w), ws.data_ptr(), n, _stream())
    assert rc == N.DCA_OK, N.status_string(rc)
    assert lib.dca_device_status(ws.data_ptr(), _stream()) == N.DCA_OK
    return out


def _no_alloc(lib, w, q, k, v):
    out = torch.full_like(q, float("nan"))
    rc = lib.dca_prefill_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), w.L,
                                 *_args(w), _stream())
    assert rc == N.DCA_OK, N.status_string(rc)
    return out


CASES = [
    Workload("na1", L=3000, Hq=7, Hkv=1, d=128, dtype="bf16", chunk_size=1024,
             local_window=256, pretrain_window=1536, yarn_scale=2.0, scale_by_sqrt_d=False),
    Workload("na2", L=1337, Hq=4, Hkv=2, d=128, dtype="bf16", chunk_size=300,
             local_window=64, pretrain_window=400, yarn_scale=1.0, scale_by_sqrt_d=False),
    Workload("na3_f32", L=900, Hq=3, Hkv=1, d=128, dtype="f32", chunk_size=256,
             local_window=40, pretrain_window=384, yarn_scale=1.5, scale_by_sqrt_d=False),
]


def test_no_alloc_matches_workspace_entry_twice(lib):
    for seed, w in enumerate(CASES):  # calls in a row, different shapes, dtypes and contents
        q, k, v = generate(w, device=DEV, seed=seed)
        want = _with_workspace(lib, w, q, k, v)
        got = _no_alloc(lib, w, q, k, v)
        assert lib.dca_noalloc_device_status(_stream()) == N.DCA_OK
        assert torch.equal(got, want), f"no-alloc call {seed + 1} ({w.name}) differs"


def test_no_alloc_rejects_problems_beyond_scratch(lib):
    w = Workload("big", L=65536, Hq=28, Hkv=4, d=128, dtype="bf16", chunk_size=8192,
                 local_window=1024, pretrain_window=16384)
    assert lib.dca_workspace_size(w.L, w.Hq, w.Hkv, w.d, w.chunk_size, w.local_window,
                                  w.pretrain_window, 0) > SCRATCH_BYTES
    p = 1 << 20  # never dereferenced: the size check comes first
    rc = lib.dca_prefill_noalloc(p, p, p, p, w.L, *_args(w), _stream())
    assert rc == N.DCA_ERR_WORKSPACE


def test_no_alloc_timeout_is_reported_and_the_next_call_is_clean(lib):
    """Withhold one key-tile load: the bounded waits run out, the kernel
    returns, and the scratch's status word says so.  A call rejected for a bad
    argument in between must not clear that word; the next good call clears it
    and matches dca_prefill exactly."""
    w = CASES[1]
    q, k, v = generate(w, device=DEV, seed=11)
    want = _with_workspace(lib, w, q, k, v)
    lib.dca_set_wait_timeout_ns(20_000_000)
    try:
        lib.dca_set_debug_flags(1)
        out = torch.zeros_like(q)
        rc = lib.dca_prefill_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                     w.L, *_args(w), _stream())
        assert rc == N.DCA_OK
        torch.cuda.synchronize()
    finally:
        lib.dca_set_debug_flags(0)
        lib.dca_set_wait_timeout_ns(0)
    # misaligned output pointer: rejected on the host, before the scratch is touched
    rc = lib.dca_prefill_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr() + 2,
                                 w.L, *_args(w), _stream())
    assert rc == N.DCA_ERR_ARG
    assert lib.dca_noalloc_device_status(_stream()) == N.DCA_ERR_TIMEOUT
    assert lib.dca_noalloc_device_status(_stream()) == N.DCA_OK   # read clears the word
    got = _no_alloc(lib, w, q, k, v)
    assert lib.dca_noalloc_device_status(_stream()) == N.DCA_OK
    assert torch.equal(got, want)
    assert_close(got.double().cpu().numpy(), want.double().cpu().numpy(), torch.bfloat16)
