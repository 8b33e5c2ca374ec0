"""Parity with N_q query rows and N_k key rows (fa_fwd_qk / fa_bwd_qk) against the
fp64 oracle. The causal mask is bottom-right aligned: query i sees key j iff
j <= i + N_k - N_q, so a query block of N_q rows is the last N_q positions of
the key sequence; rows with no key get O = 0, lse = -inf and no gradient.
Tolerances as for the square case: O max-abs <= 1e-2, lse max-abs <= 1e-3,
dQ/dK/dV relative Frobenius <= 2e-2 over each tensor and each 128-row block, and
every element within 10% of (the gradient's RMS + its row's RMS)."""
import numpy as np
import pytest
import torch

import io_aware_exact_19_b200 as fa
import oracle
from tests.gpu_inputs import Case, assert_grads, max_abs

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3


def _run_qk(B, H, Nq, Nk, d, fmt, causal, mask=None):
    cq = Case(B, H, Nq, d, fmt, seed=5)  # Q and dO
    ck = Case(B, H, Nk, d, fmt, seed=6)  # K and V
    q, do = cq.dev["q"], cq.dev["do"]
    k, v = ck.dev["k"], ck.dev["v"]
    mdev = None if mask is None else torch.from_numpy(mask).cuda()
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    fa.fa_fwd_qk(q, k, v, o, lse, causal=causal, block_mask=mdev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, Nq, d), dtype=torch.uint8, device=q.device)
    fa.fa_bwd_qk(q, k, v, o, lse, do, dq, dk, dv, ws, causal=causal, block_mask=mdev)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    Q, DO = cq.values("q"), cq.values("do")
    K, V = ck.values("k"), ck.values("v")
    O, LSE = oracle.forward(Q, K, V, cq.scale, causal=causal, block_mask=mask)
    DQ, DK, DV = oracle.backward(Q, K, V, DO, cq.scale, causal=causal, block_mask=mask)
    eo = max_abs(cq.flat(o), O)
    el = max_abs(lse.cpu().numpy().reshape(B * H, Nq), LSE)
    assert eo <= O_TOL and el <= LSE_TOL, f"O {eo:.3e} lse {el:.3e}"
    assert_grads([(cq.flat(dq), DQ), (ck.flat(dk), DK), (ck.flat(dv), DV)])
    for g in (o, dq, dk, dv):
        assert torch.isfinite(g).all()
    return o, lse, dq


@pytest.mark.parametrize("B,H,Nq,Nk,d,fmt,causal", [
    (1, 2, 128, 384, 64, "bf16", True),
    (1, 2, 1, 1000, 128, "bf16", True),      # one query row: sees every key
    (2, 1, 1000, 777, 64, "bf16", True),
    (1, 2, 777, 1000, 128, "fp16", False),
    (1, 2, 300, 129, 128, "bf16", True),
    (1, 2, 129, 300, 64, "bf16", False),
    (1, 1, 640, 1, 64, "bf16", True),        # one key: only the last query row sees it
    (1, 2, 300, 777, 96, "bf16", True),
    (2, 1, 500, 200, 32, "fp16", True),
])
def test_unequal_lengths(B, H, Nq, Nk, d, fmt, causal):
    _run_qk(B, H, Nq, Nk, d, fmt, causal)


def test_rows_without_keys():
    # N_q > N_k, causal: the first N_q - N_k rows see no key.
    B, H, Nq, Nk = 1, 2, 384, 128
    o, lse, dq = _run_qk(B, H, Nq, Nk, 128, "bf16", True)
    e = Nq - Nk
    assert torch.all(o[:, :, :e] == 0)
    assert torch.all(torch.isinf(lse[:, :, :e])) and torch.all(lse[:, :, :e] < 0)
    assert torch.all(dq[:, :, :e] == 0)


def test_block_sparse_unequal_lengths():
    rng = np.random.default_rng(4)
    mask = (rng.random((2, 4)) < 0.6).astype(np.uint8)
    mask[:, 0] = 1
    _run_qk(1, 2, 256, 512, 64, "bf16", True, mask)
    _run_qk(1, 2, 256, 512, 128, "bf16", False, mask)


def test_square_case_matches_fa_fwd_bitwise():
    c = Case(1, 2, 384, 64, "bf16", seed=7)
    q, k, v = (c.dev[n] for n in ("q", "k", "v"))
    o1, lse1 = fa.attention_forward(q, k, v, causal=True)
    o2 = torch.empty_like(q)
    lse2 = torch.empty_like(lse1)
    fa.fa_fwd_qk(q, k, v, o2, lse2, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(lse1, lse2)
