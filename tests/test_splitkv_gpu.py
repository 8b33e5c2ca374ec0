"""Split-KV forward (fa_fwd_splitkv) against the fp64 oracle.

The keys are cut into n_splits ranges of whole 128-key tiles; each range's
partial (O_s, lse_s) is checked against ``oracle.split_kv_forward`` on the same
ranges, and the merged (O, lse) against ``oracle.forward``. Tolerances as for
the forward: O max-abs <= 1e-2 (partials too, in fp32), lse max-abs <= 1e-3.
Decoding shapes (one or a few query rows against up to 64K keys; at most 4 rows
run on the CUDA-core kernel), ragged sizes, head dimensions 32/64/96/128/256,
causal (bottom-right) and block-sparse masks, and ranges in which a row has no
allowed key (lse_s = -inf, O_s = 0)."""
import numpy as np
import pytest
import torch

import io_aware_exact_19_b200 as fa
import oracle
from tests.gpu_inputs import Case, max_abs

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3


def _bounds(nk, n_splits):
    t = -(-nk // 128)
    return [min(nk, 128 * (s * t // n_splits)) for s in range(n_splits)] + [nk]


def _run(B, H, Nq, Nk, d, fmt, causal, n_splits=None, mask=None, seed=0):
    cq = Case(B, H, Nq, d, fmt, seed=seed + 1)
    ck = Case(B, H, Nk, d, fmt, seed=seed + 2)
    q, k, v = cq.dev["q"], ck.dev["k"], ck.dev["v"]
    if n_splits is None:
        n_splits = fa.fa_fwd_splitkv_splits(B, H, Nq, Nk)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    ws = torch.full((fa.fa_fwd_splitkv_workspace_size(B, H, Nq, d, n_splits),), 255, dtype=torch.uint8,
                    device="cuda")
    mdev = None if mask is None else torch.from_numpy(mask).cuda()
    fa.fa_fwd_splitkv(q, k, v, o, lse, n_splits, ws, causal=causal, block_mask=mdev)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    rows = B * H * Nq
    o_part = ws[:n_splits * rows * d * 4].view(torch.float32).reshape(n_splits, B * H, Nq, d).cpu().numpy()
    off = -(-(n_splits * rows * d * 4) // 256) * 256
    lse_part = ws[off:off + n_splits * rows * 4].view(torch.float32).reshape(n_splits, B * H, Nq).cpu().numpy()
    Q, K, V = cq.values("q"), ck.values("k"), ck.values("v")
    O, L = oracle.forward(Q, K, V, cq.scale, causal=causal, block_mask=mask)
    assert max_abs(cq.flat(o), O) <= O_TOL
    assert max_abs(lse.cpu().numpy().reshape(B * H, Nq), L) <= LSE_TOL
    bounds = _bounds(Nk, n_splits)
    for h in range(B * H):
        _, _, Os, lses = oracle.split_kv_forward(Q[h], K[h], V[h], cq.scale, bounds, causal=causal, block_mask=mask)
        for s in range(n_splits):
            assert max_abs(o_part[s, h], Os[s]) <= O_TOL, (h, s)
            assert max_abs(lse_part[s, h], lses[s]) <= LSE_TOL, (h, s)
            empty = np.isneginf(lses[s])
            assert np.array_equal(np.isneginf(lse_part[s, h]), empty), (h, s)
            assert np.all(o_part[s, h][empty] == 0), (h, s)
    return o, lse, n_splits


@pytest.mark.parametrize("B,H,Nq,Nk,d,fmt,causal,n_splits", [
    (1, 4, 1, 65536, 128, "bf16", True, None),    # decoding one token against a 64K cache
    (2, 2, 16, 4096, 64, "fp16", False, 8),
    (1, 2, 300, 1000, 96, "bf16", True, 3),       # ragged; early rows see no key of the last ranges
    (1, 1, 1024, 1024, 64, "bf16", True, 8),      # square causal: rows < 896 see nothing of range 7
    (1, 2, 5, 777, 128, "bf16", False, 7),        # one 128-key tile per range, ragged last tile
    (1, 1, 1, 1, 64, "bf16", False, 1),
    (1, 2, 3, 2000, 256, "bf16", True, 6),       # head dimension 256 (forward only)
    (2, 3, 7, 5000, 64, "fp16", True, 9),         # one query tile, odd range count: a CTA with one range
    (1, 2, 100, 1000, 128, "bf16", True, 8),      # causal: ranges past a row's reach are empty
    # at most 4 query rows: the CUDA-core decoding kernel
    (1, 16, 1, 65536, 64, "fp16", False, None),   # the decoding benchmark's shape
    (2, 2, 2, 3000, 96, "fp16", True, 5),         # padded head dimension, causal shift per row
    (1, 3, 4, 1029, 32, "bf16", True, 9),         # ragged last tile, d = 32
    (1, 1, 4, 4, 128, "bf16", True, 1),           # rows 0-2 see 1-3 keys
])
def test_splitkv_matches_oracle(B, H, Nq, Nk, d, fmt, causal, n_splits):
    _run(B, H, Nq, Nk, d, fmt, causal, n_splits)


def test_splitkv_block_sparse():
    mask = np.array([[1, 0, 0, 1, 1, 0, 0, 1], [0, 0, 0, 0, 1, 1, 1, 1]], dtype=np.uint8)
    _run(1, 2, 256, 1024, 64, "bf16", False, 4, mask=mask)
    _run(1, 2, 256, 1024, 128, "bf16", True, 4, mask=mask)


def test_splitkv_agrees_with_unsplit_forward():
    B, H, Nq, Nk, d = 2, 3, 64, 3000, 128
    o, lse, _ = _run(B, H, Nq, Nk, d, "bf16", True, 5, seed=4)
    cq = Case(B, H, Nq, d, "bf16", seed=5)
    ck = Case(B, H, Nk, d, "bf16", seed=6)
    o2 = torch.empty_like(o)
    lse2 = torch.empty_like(lse)
    fa.fa_fwd_qk(cq.dev["q"], ck.dev["k"], ck.dev["v"], o2, lse2, causal=True)
    torch.cuda.synchronize()
    assert (o.float() - o2.float()).abs().max().item() <= 1e-2
    assert (lse - lse2).abs().max().item() <= 1e-3


def test_suggested_splits_fill_the_gpu():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # At most 4 query rows (CUDA-core decoding): one range per CTA, two CTAs per SM.
    ns = fa.fa_fwd_splitkv_splits(1, 16, 1, 65536)
    assert 2 <= ns <= 512 and 16 * ns <= 2 * sms < 16 * (ns + 1)
    # One query tile of more rows: a CTA takes two consecutive ranges, B*H*ceil(n/2) CTAs.
    ns = fa.fa_fwd_splitkv_splits(1, 16, 64, 65536)
    ctas = 16 * ((ns + 1) // 2)
    assert 2 <= ns <= 512 and ctas <= sms and ctas + 16 > sms
    assert fa.fa_fwd_splitkv_splits(8, 64, 4096, 4096) == 1
    ns2 = fa.fa_fwd_splitkv_splits(1, 4, 256, 65536)  # two query tiles: a CTA per range
    assert 4 * ns2 <= sms < 4 * (ns2 + 1)
