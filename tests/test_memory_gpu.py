"""Linear memory in N (the card's "实测摘要" row: memory linear in sequence length up
to 64K): the library allocates no device memory of its own, and the caller's
footprint (inputs, outputs, lse and the backward workspace) is affine in N.

Sweep N = 1K .. 64K at B=1, H=16, d=64, causal, bf16, forward + backward.
"""
import numpy as np
import pytest
import torch

import io_aware_exact_19_b200 as fa

pytestmark = pytest.mark.gpu

B, H, D = 1, 16, 64
NS = [1024, 2048, 4096, 8192, 16384, 32768, 65536]


def _run(N, on_peak=None):
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(N)
    q, k, v, do = (torch.empty(B, H, N, D, device=dev, dtype=torch.bfloat16).normal_(generator=g) for _ in range(4))
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, D), dtype=torch.uint8, device=dev)
    fa.fa_fwd(q, k, v, o, lse, causal=True)
    fa.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, causal=True)
    torch.cuda.synchronize()
    if on_peak is not None:
        on_peak()  # before any temporary below is allocated
    assert fa.fa_device_status() == fa.FA_OK
    assert torch.isfinite(dq.float()).all() and torch.isfinite(o.float()).all()
    return sum(t.numel() * t.element_size() for t in (q, k, v, do, o, lse, dq, dk, dv, ws))


def test_memory_is_linear_in_n_and_library_allocates_nothing():
    _run(1024)  # module load and first-launch setup happen here, outside the sweep
    torch.cuda.empty_cache()
    footprint, extra = [], []
    for N in NS:
        torch.cuda.empty_cache()
        free0, _ = torch.cuda.mem_get_info()
        reserved0 = torch.cuda.memory_reserved()
        torch.cuda.reset_peak_memory_stats()
        base = torch.cuda.memory_allocated()
        seen = {}

        def record():
            seen["peak"] = torch.cuda.max_memory_allocated() - base
            seen["free"] = torch.cuda.mem_get_info()[0]
            seen["reserved"] = torch.cuda.memory_reserved()

        caller = _run(N, record)
        peak, free1 = seen["peak"], seen["free"]
        footprint.append(peak)
        # Device memory taken outside PyTorch's caching allocator while the calls ran.
        extra.append((free0 - free1) - (seen["reserved"] - reserved0))
        assert peak == pytest.approx(caller, rel=0.02)
        print(f"N={N:6d}: caller-owned bytes {caller:>12d}  peak allocated {peak:>12d}")
    ns = np.array(NS, dtype=np.float64)
    fp = np.array(footprint, dtype=np.float64)
    # Affine fit a + b*N; the quadratic coefficient of a degree-2 fit is ~0.
    b, a = np.polyfit(ns, fp, 1)
    resid = np.abs(fp - (a + b * ns)) / fp
    assert resid.max() < 0.01, resid
    c2 = np.polyfit(ns, fp, 2)[0]
    assert abs(c2) * ns[-1] ** 2 < 0.01 * fp[-1]
    # bytes per token and head: 8 bf16 [.., d] tensors (q k v dO o dq dk dv), lse,
    # and the two fp32 vectors of the backward workspace
    assert b == pytest.approx(B * H * (8 * D * 2 + 4 + 8), rel=0.02)
    for e in extra:
        assert e < 64 << 20
