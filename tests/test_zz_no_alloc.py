"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Those callers (a host application that plans all device memory itself and gives
this library no allocator, or a latency-critical loop where cudaMalloc is not
allowed) call fa_bwd_noalloc, whose scratch lives in a fixed static array inside
the library. This test calls it through the C ABI twice in a row and checks each
result against fa_bwd (which takes a caller-provided workspace) and against the
fp64 oracle, with the gradient bounds the parity tests use, and that a problem
whose workspace does not fit the static array is rejected before anything runs.
The file is named so that pytest collects it after every other test file.
"""
import ctypes

import pytest
import torch

import io_aware_exact_19_b200 as fa
import oracle
from tests.gpu_inputs import Case, assert_grads

pytestmark = pytest.mark.gpu

G_TOL = 2e-2
SCRATCH_BYTES = 32 << 20  # FA_BWD_NOALLOC_SCRATCH_BYTES in include/fa.h


def _rel(a, b):
    a, b = a.double(), b.double()
    return float(torch.linalg.norm(a - b) / torch.clamp(torch.linalg.norm(b), min=1e-30))


@pytest.mark.parametrize("B,H,N,d,causal", [(2, 3, 1000, 64, True), (1, 2, 777, 128, False), (2, 4, 1024, 128, True)])
def test_noalloc_backward_matches_workspace_backward(B, H, N, d, causal):
    assert fa.fa_bwd_workspace_size(B, H, N, d) <= SCRATCH_BYTES
    c = Case(B, H, N, d, "bf16", seed=N + d + 1)
    q, k, v, do = (c.dev[n] for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=causal)
    ref = fa.attention_backward(q, k, v, o, lse, do, causal=causal)
    torch.cuda.synchronize()
    vals = [c.values(n) for n in ("q", "k", "v", "do")]
    exact = oracle.backward(*vals, c.scale, causal=causal)
    for _ in range(2):  # two calls in a row share the static scratch
        dq, dk, dv = (torch.full_like(t, float("nan")) for t in (q, k, v))
        fa.fa_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, causal=causal)
        torch.cuda.synchronize()
        assert fa.fa_device_status() == fa.FA_OK
        for got, exp in zip((dq, dk, dv), ref):
            assert torch.isfinite(got).all()
            assert _rel(got, exp) <= G_TOL
        assert_grads([(c.flat(g), G) for g, G in zip((dq, dk, dv), exact)])


def test_noalloc_rejects_problems_larger_than_its_scratch():
    B, H, N, d = 16, 64, 8192, 128
    assert fa.fa_bwd_workspace_size(B, H, N, d) > SCRATCH_BYTES
    lib = fa.load_library()
    p = ctypes.c_void_p(4096)  # never dereferenced: the size check comes first
    st = lib.fa_bwd_noalloc(fa.FA_BF16, p, p, p, p, p, p, p, p, p, B, H, N, d, 0.1, 1, None)
    assert st == fa.FA_ERR_UNSUPPORTED
