"""Dropout fused into the attention kernels (fa_fwd_dropout / fa_bwd_dropout)
against the fp64 oracle (oracle.dropout).

Keep decisions are integer work: the draws the kernels generate, through both
device generator paths, must equal the oracle's bit for bit, and with V = I
the output's zeros are exactly the dropped (or masked) entries. Values: lse
max-abs <= 1e-3 and the gradient bounds of ``tests.gpu_inputs.assert_grads``, as
for the plain path; O within 1e-2 + 2^-7 |O| elementwise. The plain path's 1e-2
assumes |O| <= max |v|; dropout scales kept entries by 1/q, and a row that sees
one key has O = Z v exactly, so the 16-bit rounding of P o Z and of O (half a
unit, 2^-8 |x|, each) alone reaches 0.018 at |O| = 4.5. The gradients' element
bound is 0.25 (0.1 without dropout): the cancellation in dS = P o (dP o Z - D)
that D, formed from the 16-bit O, leaves in rows with few keys is larger when Z
zeroes some of them (measured 0.14 at B=2 H=3 N=1000 d=64 causal p=0.1, where
the norms are 0.003); the keep decisions themselves are checked bit-exactly."""
import numpy as np
import pytest
import torch

import io_aware_exact_19_b200 as fa
from oracle import dropout as Dr
from oracle.attention import allowed_mask
from tests.gpu_inputs import Case, assert_grads, max_abs

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3


@pytest.mark.parametrize("B,H,Nq,Nk,seed", [(1, 3, 300, 517, 0x0123456789ABCDEF), (2, 1, 128, 128, 7),
                                            (1, 2, 1, 1000, 2 ** 64 - 1), (1, 1, 1029, 255, 0)])
def test_device_draws_equal_the_oracle(B, H, Nq, Nk, seed):
    rm = torch.zeros((B * H, Nq, Nk), dtype=torch.uint8, device="cuda")
    cm = torch.zeros_like(rm)
    fa.fa_debug_dropout_draws(B, H, Nq, Nk, seed, rm, cm)
    torch.cuda.synchronize()
    for bh in range(B * H):
        exp = Dr.draws(Nq, Nk, bh, seed)
        assert np.array_equal(rm[bh].cpu().numpy(), exp), f"row-major draws, head {bh}"
        assert np.array_equal(cm[bh].cpu().numpy(), exp), f"column-major draws, head {bh}"


def _inputs(B, H, Nq, Nk, d, fmt, seed):
    cq = Case(B, H, Nq, d, fmt, seed=seed)
    ck = Case(B, H, Nk, d, fmt, seed=seed + 100)
    return cq, ck


def _run(B, H, Nq, Nk, d, fmt, causal, p, seed, mask=None):
    cq, ck = _inputs(B, H, Nq, Nk, d, fmt, seed=Nq + Nk + d)
    q, do = cq.dev["q"], cq.dev["do"]
    k, v = ck.dev["k"], ck.dev["v"]
    mdev = None if mask is None else torch.from_numpy(mask).cuda()
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    fa.fa_fwd_dropout(q, k, v, o, lse, p, seed, causal=causal, block_mask=mdev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, Nq, d), dtype=torch.uint8, device="cuda")
    fa.fa_bwd_dropout(q, k, v, o, lse, do, dq, dk, dv, ws, p, seed, causal=causal, block_mask=mdev)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    Q, DO, K, V = cq.values("q"), cq.values("do"), ck.values("k"), ck.values("v")
    O, L = Dr.forward_dropout(Q, K, V, cq.scale, p, seed, causal=causal, block_mask=mask)
    err = np.abs(cq.flat(o) - O) - (O_TOL + 2.0 ** -7 * np.abs(O))
    assert float(err.max()) <= 0.0, f"O error exceeds 1e-2 + 2^-7|O| by {float(err.max()):.3e}"
    assert max_abs(lse.cpu().numpy().reshape(B * H, Nq), L) <= LSE_TOL
    G = Dr.backward_dropout(Q, K, V, DO, cq.scale, p, seed, causal=causal, block_mask=mask)
    assert_grads([(cq.flat(dq), G[0]), (ck.flat(dk), G[1]), (ck.flat(dv), G[2])], elem_tol=0.25)
    return o, lse, (dq, dk, dv)


@pytest.mark.parametrize("B,H,Nq,Nk,d,fmt,causal,p", [
    (2, 3, 1000, 1000, 64, "bf16", True, 0.1),
    (1, 2, 777, 777, 128, "fp16", False, 0.5),
    (1, 2, 300, 517, 128, "bf16", True, 0.25),
    (2, 1, 640, 200, 64, "bf16", True, 0.2),
    (1, 2, 129, 129, 96, "bf16", False, 0.3),
])
def test_dropout_matches_oracle(B, H, Nq, Nk, d, fmt, causal, p):
    _run(B, H, Nq, Nk, d, fmt, causal, p, seed=0xFEEDFACECAFEBEEF)


def test_dropout_block_sparse():
    mask = np.array([[1, 0, 1, 1], [0, 1, 1, 0]], dtype=np.uint8)
    _run(1, 2, 256, 512, 64, "bf16", False, 0.4, seed=11, mask=mask)


@pytest.mark.parametrize("d,causal", [(64, True), (128, False)])
def test_identity_values_expose_the_keep_decisions(d, causal):
    # V = I (N = d): O = P o Z, so its zeros are exactly the dropped or masked entries.
    N, seed, p = d, 99, 0.3
    c = Case(1, 1, N, d, "bf16", seed=3)
    v = torch.eye(N, dtype=torch.bfloat16, device="cuda").reshape(1, 1, N, d).contiguous()
    o = torch.empty_like(c.dev["q"])
    lse = torch.empty((1, 1, N), dtype=torch.float32, device="cuda")
    fa.fa_fwd_dropout(c.dev["q"], c.dev["k"], v, o, lse, p, seed, causal=causal)
    torch.cuda.synchronize()
    kept = (Dr.keep_scale(N, N, 0, seed, p) > 0) & allowed_mask(N, N, causal)
    got = o[0, 0].float().cpu().numpy()
    assert np.array_equal(got != 0, kept)


def test_zero_probability_is_the_plain_kernel_and_seeds_matter():
    c = Case(1, 2, 384, 64, "bf16", seed=5)
    q, k, v = (c.dev[n] for n in ("q", "k", "v"))
    o1, l1 = fa.attention_forward(q, k, v, causal=True)
    o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
    fa.fa_fwd_dropout(q, k, v, o2, l2, 0.0, 123, causal=True)
    o3, l3, o4, l4 = torch.empty_like(o1), torch.empty_like(l1), torch.empty_like(o1), torch.empty_like(l1)
    fa.fa_fwd_dropout(q, k, v, o3, l3, 0.2, 5, causal=True)
    fa.fa_fwd_dropout(q, k, v, o4, l4, 0.2, 5, causal=True)
    o5, l5 = torch.empty_like(o1), torch.empty_like(l1)
    fa.fa_fwd_dropout(q, k, v, o5, l5, 0.2, 6, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(o3, o4) and torch.equal(l3, l4)
    assert not torch.equal(o3, o5) and torch.equal(l3, l5)


@pytest.mark.parametrize("d,p", [(128, 0.1), (128, 0.5), (64, 0.998), (64, 0.3)])
def test_keep_decisions_across_key_tiles(d, p):
    # Q = 0 makes P uniform (every exponential is 1, l = Nk); V[j] = 2^(j // d) e_(j % d)
    # sums the keep decisions of keys c, c + d, c + 2d, c + 3d of a row into one integer
    # O[i, c] * Nk / Z_kept, so every decision of four key groups is checked exactly,
    # at thresholds t = 26, 128, 255 and 77.
    B, H, Nq, Nk, seed = 1, 2, 256, 4 * d, 0x5EED0FD40F
    c = Case(B, H, Nk, d, "bf16", seed=21)
    q = torch.zeros((B, H, Nq, d), dtype=torch.bfloat16, device="cuda")
    j = np.arange(Nk)
    vals = np.zeros((Nk, d), dtype=np.float32)
    vals[j, j % d] = 2.0 ** (j // d)
    v = torch.from_numpy(vals).to(torch.bfloat16).cuda().expand(B, H, Nk, d).contiguous()
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    fa.fa_fwd_dropout(q, c.dev["k"], v, o, lse, p, seed)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    t = Dr.drop_threshold(p)
    z_kept = 256.0 / (256 - t)
    for bh in range(B * H):
        kept = (Dr.keep_scale(Nq, Nk, bh, seed, p) > 0).astype(np.int64)      # [Nq, Nk]
        expect = sum(kept[:, g * d:(g + 1) * d] << g for g in range(4))      # [Nq, d]
        got = o.reshape(B * H, Nq, d)[bh].float().cpu().numpy() * Nk / z_kept
        assert np.array_equal(np.rint(got).astype(np.int64), expect), f"head {bh}"
        assert float(np.abs(got - np.rint(got)).max()) < 0.05


def _one_hot_powers(n, d):
    """[n, d]: row r is 2^(r // d) at column r % d (n = 4d rows: four groups)."""
    r = np.arange(n)
    x = np.zeros((n, d), dtype=np.float32)
    x[r, r % d] = 2.0 ** (r // d)
    return x


@pytest.mark.parametrize("grad,d,p", [("dv", 128, 0.1), ("dv", 64, 0.998), ("dq", 128, 0.5), ("dq", 64, 0.3),
                                      ("dk", 128, 0.25), ("dk", 64, 0.7)])
def test_backward_keep_decisions_exact(grad, d, p):
    # S = Q K^T = 0 (Q = 0, or K = 0 for dK) makes P = 1/Nk exactly. Then, with one-hot
    # powers of two, each gradient element is an integer combination of the keep
    # decisions of four rows (or keys), decoded exactly:
    #   dv: dO[i] = 2^(i//d) e_(i%d)            -> dV[j, c] Nk / zq = sum_g M[gd+c, j] 2^g
    #   dq: K[j] likewise, V[j] = dO[i] = e_0    -> dS = (Z - D_i) / Nk,
    #       (dQ[i, c] Nk / scale + 15 D_i) / zq  = sum_g M[i, gd+c] 2^g
    #   dk: Q[i] likewise, K = 0, V = dO = e_0   -> (dK[j, c] Nk / scale + sum_g 2^g D_(gd+c)) / zq
    #                                             = sum_g M[gd+c, j] 2^g
    # with zq = 256 / (256 - t) and D_i = O[i, 0] (the 16-bit O the prep reads).
    B, H, seed = 1, 2, 0xD0D0CAFE
    Nq, Nk = (4 * d, 256) if grad in ("dv", "dk") else (256, 4 * d)
    dev = dict(dtype=torch.bfloat16, device="cuda")
    rnd = Case(B, H, max(Nq, Nk), d, "bf16", seed=31)
    e0 = torch.zeros(d, **dev)
    e0[0] = 1
    powers_q = torch.from_numpy(_one_hot_powers(Nq, d)).to(**dev).expand(B, H, Nq, d).contiguous()
    powers_k = torch.from_numpy(_one_hot_powers(Nk, d)).to(**dev).expand(B, H, Nk, d).contiguous()
    if grad == "dv":
        q = torch.zeros((B, H, Nq, d), **dev)
        k = rnd.dev["k"][:, :, :Nk].contiguous()
        v = rnd.dev["v"][:, :, :Nk].contiguous()
        do = powers_q
    elif grad == "dq":
        q = torch.zeros((B, H, Nq, d), **dev)
        k = powers_k
        v = e0.expand(B, H, Nk, d).contiguous()
        do = e0.expand(B, H, Nq, d).contiguous()
    else:
        q = powers_q
        k = torch.zeros((B, H, Nk, d), **dev)
        v = e0.expand(B, H, Nk, d).contiguous()
        do = e0.expand(B, H, Nq, d).contiguous()
    scale = 1.0 / np.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    fa.fa_fwd_dropout(q, k, v, o, lse, p, seed, scale=scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, Nq, d), dtype=torch.uint8, device="cuda")
    fa.fa_bwd_dropout(q, k, v, o, lse, do, dq, dk, dv, ws, p, seed, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    zq = 256.0 / (256 - Dr.drop_threshold(p))
    w = 2 ** np.arange(4)
    for bh in range(B * H):
        kept = (Dr.keep_scale(Nq, Nk, bh, seed, p) > 0).astype(np.int64)          # [Nq, Nk]
        D = o.reshape(B * H, Nq, d)[bh, :, 0].float().cpu().numpy().astype(np.float64)
        if grad == "dv":
            got = dv.reshape(B * H, Nk, d)[bh].double().cpu().numpy() * Nk / zq
            expect = sum(kept[g * d:(g + 1) * d, :].T << g for g in range(4))     # [Nk, d]
        elif grad == "dq":
            got = (dq.reshape(B * H, Nq, d)[bh].double().cpu().numpy() * Nk / scale + 15 * D[:, None]) / zq
            expect = sum(kept[:, g * d:(g + 1) * d] << g for g in range(4))      # [Nq, d]
        else:
            dsum = (D.reshape(4, d) * w[:, None]).sum(axis=0)                     # [d]
            got = (dk.reshape(B * H, Nk, d)[bh].double().cpu().numpy() * Nk / scale + dsum[None, :]) / zq
            expect = sum(kept[g * d:(g + 1) * d, :].T << g for g in range(4))     # [Nk, d]
        assert float(np.abs(got - np.rint(got)).max()) < 0.25, f"{grad} head {bh}: not near integers"
        assert np.array_equal(np.rint(got).astype(np.int64), expect), f"{grad} head {bh}"
