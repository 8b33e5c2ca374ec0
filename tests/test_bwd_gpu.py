"""Backward parity: dQ, dK, dV from the CUDA path (forward then backward, through
the C ABI) against the fp64 oracle. Tolerance: relative Frobenius error <= 2e-2
per gradient, also over every 128-row block of every head (sampled rows: every
row), and every element within 10% of (the gradient's RMS + its row's RMS) (see
``tests.gpu_inputs.grad_errors``); tile indexing bit-exact."""
import numpy as np
import pytest
import torch

import fa_synth as S
import io_aware_exact_19_b200 as fa
import oracle
from tests.gpu_inputs import Case, assert_grads

pytestmark = pytest.mark.gpu


def _run(c: Case, causal, mask=None):
    mdev = None if mask is None else torch.from_numpy(mask).cuda()
    q, k, v, do = (c.dev[n] for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=causal, block_mask=mdev)
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, causal=causal, block_mask=mdev)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    return dq, dk, dv


def _check_full(c: Case, causal, mask=None, heads=None):
    dq, dk, dv = _run(c, causal, mask)
    vals = [c.values(n, heads) for n in ("q", "k", "v", "do")]
    DQ, DK, DV = oracle.backward(*vals, c.scale, causal=causal, block_mask=mask)
    errs = assert_grads([(c.flat(g, heads), G) for g, G in ((dq, DQ), (dk, DK), (dv, DV))])
    for g in (dq, dk, dv):
        assert torch.isfinite(g).all()
    return errs


def test_tiny_fp16_exact_check():
    _check_full(Case(1, 1, 128, 64, "fp16"), causal=False)


@pytest.mark.parametrize("B,H,N,d,fmt,causal", [
    (2, 3, 1000, 64, "bf16", False), (2, 3, 1000, 64, "bf16", True),
    (1, 2, 1000, 128, "bf16", True), (1, 2, 777, 128, "fp16", False),
    (1, 1, 1, 64, "bf16", False), (1, 1, 1, 128, "fp16", True),
    (1, 2, 129, 64, "bf16", True), (2, 1, 256, 128, "bf16", False),
    (1, 1, 384, 64, "fp16", True), (1, 3, 640, 128, "bf16", True),
    (1, 1, 65, 128, "bf16", False),
    # head dimensions 32 and 96 (inside the 64 and 128 kernels, zero-filled columns)
    (2, 3, 1000, 32, "bf16", True), (1, 2, 777, 32, "fp16", False), (1, 1, 1, 32, "bf16", False),
    (2, 2, 1000, 96, "bf16", True), (1, 2, 129, 96, "fp16", False), (1, 1, 1, 96, "bf16", True),
])
def test_ragged_and_small(B, H, N, d, fmt, causal):
    _check_full(Case(B, H, N, d, fmt, seed=N + d), causal)


@pytest.mark.parametrize("causal", [False, True])
def test_gpt2_small_shape(causal):
    _check_full(Case(8, 12, 1024, 64, "bf16"), causal)


def test_long_context_d128_causal_heads():
    _check_full(Case(4, 16, 4096, 128, "bf16"), True, heads=[0, 21, 42, 63])


def _check_sampled(c: Case, causal, mask, nq, nk):
    dq, dk, dv = _run(c, causal, mask)
    N = c.shape[2]
    rows_q = S.sample_rows(N, nq, seed=1)
    rows_k = S.sample_rows(N, nk, seed=2)
    vals = [c.values(n) for n in ("q", "k", "v", "do")]
    ref = oracle.sampled_forward_backward(*vals, c.scale, causal, rows_q, rows_k, block_mask=mask)
    # Sampled rows are not contiguous: every row is its own block.
    assert_grads([(c.flat(dq)[:, rows_q], ref["dq"]), (c.flat(dk)[:, rows_k], ref["dk"]),
                  (c.flat(dv)[:, rows_k], ref["dv"])], tile=1, what="dQ/dK/dV (sampled rows)")


def test_linear_memory_stress_sampled_rows():
    _check_sampled(Case(1, 16, 65536, 64, "bf16"), True, None, 256, 256)


def test_block_sparse_workload_sampled_rows():
    _check_sampled(Case(2, 16, 8192, 64, "bf16"), False, S.block_mask_recipe(64), 256, 256)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [32, 64, 96, 128])
def test_block_sparse_full(causal, d):
    _check_full(Case(2, 2, 1024, d, "bf16", seed=9), causal, mask=S.block_mask_recipe(8, seed=4))


def test_block_sparse_empty_row_and_column():
    mask = np.ones((4, 4), dtype=np.uint8)
    mask[1, :] = 0   # query tile 1 sees no key: zero dQ there
    mask[:, 2] = 0   # key tile 2 is seen by no query: zero dK, dV there
    for d in (64, 128):
        c = Case(1, 2, 512, d, "bf16", seed=3)
        dq, dk, dv = _run(c, False, mask)
        assert torch.all(dq[:, :, 128:256] == 0)
        assert torch.all(dk[:, :, 256:384] == 0) and torch.all(dv[:, :, 256:384] == 0)
        _check_full(c, False, mask=mask)


def test_unused_key_tile_is_never_read():
    mask = S.block_mask_recipe(8, seed=5)
    mask[:, 5] = 0
    c = Case(1, 2, 1024, 64, "bf16", seed=11)
    g1 = _run(c, False, mask)
    k, v = c.dev["k"].clone(), c.dev["v"].clone()
    k[:, :, 640:768] = float("nan")
    v[:, :, 640:768] = float("nan")
    mdev = torch.from_numpy(mask).cuda()
    q, do = c.dev["q"], c.dev["do"]
    o, lse = fa.attention_forward(q, k, v, block_mask=mdev)
    g2 = fa.attention_backward(q, k, v, o, lse, do, block_mask=mdev)
    torch.cuda.synchronize()
    for a, b in zip(g1, g2):
        assert torch.isfinite(b).all()
        # Every accumulation runs in a fixed order (no atomics): bit-identical.
        assert torch.equal(a, b)


@pytest.mark.parametrize("N,causal,use_mask,d", [(1000, False, False, 64), (1000, True, False, 128),
                                                 (1024, False, True, 64), (1024, True, True, 128),
                                                 (1408, True, True, 64)])
def test_tile_trace_matches_oracle_enumeration(N, causal, use_mask, d):
    B, H = 1, 2
    c = Case(B, H, N, d, "bf16", seed=1)
    mask = S.block_mask_recipe(N // 128, seed=6) if use_mask else None
    mdev = torch.from_numpy(mask).cuda() if use_mask else None
    q, k, v, do = (c.dev[n] for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=causal, block_mask=mdev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    trace = torch.full((fa.fa_bwd_trace_size(B, H, N, d),), -1, dtype=torch.int32, device="cuda")
    fa.fa_debug_bwd_trace(q, k, v, o, lse, do, dq, dk, dv, ws, trace, causal=causal, block_mask=mdev)
    torch.cuda.synchronize()
    got = trace.cpu().numpy().astype(np.int64)
    br = fa.fa_bwd_row_tile(d)
    t = -(-N // 128)
    tq = -(-N // br)
    # key-stationary CTAs: the query tiles (br rows) that reach each key tile
    key_lists = oracle.backward_tile_lists(N, causal, mask, br=br, bc=128)
    key_part = got[:B * H * t * (tq + 1)].reshape(B * H, t, tq + 1)
    # query-stationary CTAs: the key tiles each 128-row query tile reaches
    query_lists = oracle.forward_tile_lists(N, causal, mask, br=128, bc=128)
    query_part = got[B * H * t * (tq + 1):].reshape(B * H, t, t + 1)
    for bh in range(B * H):
        for j, exp in enumerate(key_lists):
            assert key_part[bh, j, 0] == len(exp)
            assert list(key_part[bh, j, 1:1 + len(exp)]) == [i | (1 << 16) for i in exp], (bh, j)
        for i, exp in enumerate(query_lists):
            assert query_part[bh, i, 0] == len(exp)
            assert list(query_part[bh, i, 1:1 + len(exp)]) == [j | (1 << 16) for j in exp], (bh, i)


@pytest.mark.parametrize("d", [64, 128])
def test_backward_kernel_abort_path_reports_timeout_and_context_survives(d):
    # The production backward main kernel with producers that issue no load: both
    # CTA kinds' first waits run out (20 ms), every role leaves its loop, the MMA
    # issuers wait for what they issued, the CTAs exit. The status word reports
    # the time-out; the next, normal backward is still correct.
    c = Case(1, 3, 700, d, "bf16", seed=23)
    q, k, v, do = (c.dev[n] for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    dq, dk, dv = (torch.zeros_like(t) for t in (q, k, v))
    ws = torch.empty(fa.fa_bwd_workspace_size(1, 3, 700, d), dtype=torch.uint8, device="cuda")
    fa.fa_debug_bwd_withhold(q, k, v, o, lse, do, dq, dk, dv, ws, 20, causal=True)
    assert fa.fa_device_status() == fa.FA_ERR_TIMEOUT
    assert fa.fa_device_status() == fa.FA_OK
    assert all(torch.count_nonzero(g) == 0 for g in (dq, dk, dv))
    _check_full(c, True)
