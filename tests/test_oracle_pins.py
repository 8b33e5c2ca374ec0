"""The fp64 oracle against closed forms, invariants, finite differences and brute force."""
import numpy as np
import pytest

import oracle
from oracle import attention as A
from tests import oracle_pins as pins


def test_closed_forms():
    pins.check_closed_forms(oracle.forward, oracle.backward)


@pytest.mark.parametrize("check", pins.ALL_FORWARD_CHECKS, ids=lambda f: f.__name__)
def test_forward_invariant(check):
    check(oracle.forward)


def test_online_recurrence_equals_two_pass():
    pins.check_online_equals_two_pass(oracle.forward, oracle.online_forward)


def test_finite_differences():
    pins.check_finite_differences(oracle.forward, oracle.backward)


def test_gradient_identities():
    pins.check_gradient_identities(oracle.forward, oracle.backward)


def test_split_kv_merge():
    pins.check_split_kv_merge(oracle.forward, oracle.split_kv_forward, oracle.merge_partials)


def test_blocksparse_reductions():
    pins.check_blocksparse_reductions(oracle.forward, oracle.backward)


def test_fully_masked_row_convention():
    # A mask that removes every key of query tile 1: O = 0, lse = -inf, zero gradients.
    r = np.random.default_rng(0)
    q, k, v, do = (r.standard_normal((8, 3)) for _ in range(4))
    mask = np.array([[1, 1], [0, 0]], dtype=np.uint8)
    O, lse = oracle.forward(q, k, v, 0.5, block_mask=mask, tile=4)
    assert np.all(O[4:] == 0) and np.all(np.isneginf(lse[4:]))
    dq, dk, dv = oracle.backward(q, k, v, do, 0.5, block_mask=mask, tile=4)
    assert np.all(dq[4:] == 0)
    assert np.all(np.isfinite(dk)) and np.all(np.isfinite(dv))


def test_sampled_mode_matches_full():
    r = np.random.default_rng(12)
    B, H, N, d = 1, 2, 384, 16
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    rows_q = np.array([0, 5, 127, 128, 200, 383])
    rows_k = np.array([0, 1, 130, 255, 256, 383])
    mask = np.array([[1, 0, 1], [1, 1, 0], [1, 0, 1]], dtype=np.uint8)
    for causal, bm in ((True, None), (False, None), (False, mask)):
        s = oracle.sampled_forward_backward(q, k, v, do, 0.25, causal, rows_q, rows_k,
                                            block_mask=bm, chunk=100, workers=2)
        O, lse = oracle.forward(q, k, v, 0.25, causal=causal, block_mask=bm)
        dq, dk, dv = oracle.backward(q, k, v, do, 0.25, causal=causal, block_mask=bm)
        np.testing.assert_allclose(s["o"], O[..., rows_q, :], rtol=0, atol=1e-12)
        np.testing.assert_allclose(s["lse"], lse[..., rows_q], rtol=0, atol=1e-12)
        np.testing.assert_allclose(s["dq"], dq[..., rows_q, :], rtol=0, atol=1e-12)
        np.testing.assert_allclose(s["dk"], dk[..., rows_k, :], rtol=0, atol=1e-12)
        np.testing.assert_allclose(s["dv"], dv[..., rows_k, :], rtol=0, atol=1e-12)


# ------------------------------------------------------------------ tile enumeration

def _tiles_with_allowed_pair(n, br, bc, causal, block_mask, nk=None):
    nk = n if nk is None else nk
    a = A.allowed_mask(n, nk, causal, block_mask)
    tr, tc = -(-n // br), -(-nk // bc)
    return {(i, j) for i in range(tr) for j in range(tc)
            if a[i * br:(i + 1) * br, j * bc:(j + 1) * bc].any()}


@pytest.mark.parametrize("n", [1, 64, 127, 128, 129, 300, 512, 1000])
@pytest.mark.parametrize("br,bc", [(128, 128), (64, 128)])
def test_causal_tile_set_is_exactly_the_tiles_with_an_unmasked_entry(n, br, bc):
    assert set(A.causal_tile_set(n, br, bc)) == _tiles_with_allowed_pair(n, br, bc, True, None)


@pytest.mark.parametrize("nq,nk", [(1, 1000), (128, 384), (384, 128), (300, 129), (129, 300), (1000, 777),
                                   (640, 1), (5, 7)])
def test_causal_tile_set_with_unequal_lengths(nq, nk):
    # Bottom-right alignment: still exactly the tiles holding an allowed pair, and
    # the transpose lists agree with the forward lists.
    assert set(A.causal_tile_set(nq, 128, 128, nk)) == _tiles_with_allowed_pair(nq, 128, 128, True, None, nk)
    fwd = A.forward_tile_lists(nq, True, nk=nk)
    bwd = A.backward_tile_lists(nq, True, nk=nk)
    assert {(i, j) for i, js in enumerate(fwd) for j in js} == {(i, j) for j, is_ in enumerate(bwd) for i in is_}
    assert len(fwd) == -(-nq // 128) and len(bwd) == -(-nk // 128)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("br", [128, 64])
def test_tile_lists_match_mask_and_transpose(causal, br):
    n = 1024
    from fa_synth import block_mask_recipe
    bm = block_mask_recipe(n // 128, seed=3)
    fwd = A.forward_tile_lists(n, causal, bm, br=br, bc=128)
    bwd = A.backward_tile_lists(n, causal, bm, br=br, bc=128)
    pairs_f = {(i, j) for i, js in enumerate(fwd) for j in js}
    pairs_b = {(i, j) for j, is_ in enumerate(bwd) for i in is_}
    assert pairs_f == pairs_b
    assert pairs_f == _tiles_with_allowed_pair(n, br, 128, causal, bm)


def test_forward_rows_matches_full():
    r = np.random.default_rng(13)
    q, k, v = (r.standard_normal((2, 300, 8)) for _ in range(3))
    rows = np.array([0, 1, 150, 255, 256, 299])
    mask = np.array([[1, 0, 1], [0, 1, 1], [1, 1, 0]], dtype=np.uint8)
    for causal, bm in ((False, None), (True, None), (False, mask), (True, mask)):
        O, lse = oracle.forward(q, k, v, 0.3, causal=causal, block_mask=bm)
        Or, lser = oracle.forward_rows(q, k, v, 0.3, rows, causal=causal, block_mask=bm)
        np.testing.assert_allclose(Or, O[:, rows], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lser, lse[:, rows], rtol=0, atol=1e-13)


def test_backward_rows_equals_full_backward_on_all_rows():
    r = np.random.default_rng(14)
    q, k, v, do = (r.standard_normal((40, 6)) for _ in range(4))
    for causal in (False, True):
        O, lse = oracle.forward(q, k, v, 0.4, causal=causal)
        dq, dk, dv = oracle.backward(q, k, v, do, 0.4, causal=causal)
        o2, l2, dq2, dk2, dv2 = oracle.backward_rows(q, k, v, do, 0.4, np.arange(40), causal=causal)
        for a, b in ((o2, O), (l2, lse), (dq2, dq), (dk2, dk), (dv2, dv)):
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_backward_rows_finite_differences():
    # L = sum over the chosen rows of <dO_i, O_i>; its gradient by central differences.
    r = np.random.default_rng(15)
    q, k, v, do = (r.standard_normal((9, 3)) for _ in range(4))
    rows = np.array([1, 4, 8])
    h = 1e-5
    for causal in (False, True):
        _, _, dq_r, dk, dv = oracle.backward_rows(q, k, v, do, 0.7, rows, causal=causal)
        dq = np.zeros_like(q)
        dq[rows] = dq_r

        def L(q_, k_, v_):
            O, _ = oracle.forward(q_, k_, v_, 0.7, causal=causal)
            return float(np.sum(do[rows] * O[rows]))

        for name, g in (("q", dq), ("k", dk), ("v", dv)):
            R = r.standard_normal(q.shape)
            args = {"q": q, "k": k, "v": v}
            plus = {n: a + h * R if n == name else a for n, a in args.items()}
            minus = {n: a - h * R if n == name else a for n, a in args.items()}
            fd = (L(plus["q"], plus["k"], plus["v"]) - L(minus["q"], minus["k"], minus["v"])) / (2 * h)
            an = float(np.sum(g * R))
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (name, causal, fd, an)


def test_row_routines_with_unequal_lengths():
    pins.check_rows_unequal_lengths(oracle.forward, oracle.forward_rows, oracle.backward_rows)


def test_dropout():
    from oracle import dropout as Dr
    pins.check_philox_against_numpy(Dr.philox4)
    pins.check_philox_vectorised(Dr.philox4, Dr.philox4x32_arrays)
    pins.check_dropout_layout(Dr.draws, Dr.philox4)
    pins.check_dropout_statistics(Dr.draws, Dr.keep_scale)
    pins.check_dropout_reductions(oracle.forward, oracle.backward, Dr.forward_dropout, Dr.backward_dropout)
    pins.check_dropout_finite_differences(Dr.forward_dropout, Dr.backward_dropout)
