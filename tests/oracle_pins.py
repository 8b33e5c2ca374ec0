"""Checks that pin the fp64 oracle to facts fixed by the pages and by mathematics.

Each ``check_*`` takes the oracle functions it exercises and raises
AssertionError on a mismatch, so the same checks run against the real oracle
(``test_oracle_pins.py``) and against copies of it with planted mistakes
(``test_oracle_mutants.py``), where at least one check must fail.

What pins what:
  * closed forms worked out by hand (tests/golden/closed_forms.json);
  * rows of P sum to 1; equal keys give the mean of the values; one key gives
    that key's value; causal row 0 returns V_0; a constant value column passes
    through; shifting every key by one vector leaves O unchanged;
  * the two-pass softmax equals the online-softmax recurrence of the
    interview explainer (section 三.2) for any split of the keys;
  * central finite differences of L = <dO, O> confirm dQ, dK, dV;
  * gradient identities: D = rowsum(dO∘O) = rowsum(P∘dP), Σ_j dK_j = 0,
    Σ_j dV_j = Σ_i dO_i;
  * block-sparse with an all-ones mask equals dense, and a block-diagonal mask
    equals independent attention on each block;
  * pure-Python loops on tiny inputs (a second, loop-level reading of the
    definition).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol, what):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    err = np.where(both_inf, 0.0, np.abs(a - b))
    m = float(np.max(err)) if err.size else 0.0
    assert m <= tol, f"{what}: max abs err {m:.3e} > {tol:.1e}"


# ----------------------------------------------------------------------------- closed forms

def check_closed_forms(forward, backward):
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q, k, v, do = (np.array(c[n], dtype=np.float64) for n in ("q", "k", "v", "do"))
        O, lse = forward(q, k, v, c["scale"], causal=c["causal"])
        _close(O, c["o"], 1e-12, c["name"] + " O")
        _close(lse, c["lse"], 1e-12, c["name"] + " lse")
        if q.shape[0] == k.shape[0]:
            dq, dk, dv = backward(q, k, v, do, c["scale"], causal=c["causal"])
            _close(dq, c["dq"], 1e-12, c["name"] + " dQ")
            _close(dk, c["dk"], 1e-12, c["name"] + " dK")
            _close(dv, c["dv"], 1e-12, c["name"] + " dV")


# ----------------------------------------------------------------------------- invariants

def check_rows_sum_to_one(forward):
    r = _rng(1)
    for causal, mask in ((False, None), (True, None), (False, np.array([[1, 0], [1, 1]]))):
        q, k, v = (r.standard_normal((2, 8, 3)) for _ in range(3))
        _, _, P = forward(q, k, v, 0.5, causal=causal, block_mask=mask, tile=4, return_p=True)
        _close(P.sum(-1), np.ones((2, 8)), 1e-12, "rows of P sum to 1")
        assert np.all(P >= 0), "P has a negative entry"


def check_equal_keys(forward):
    r = _rng(2)
    n, d, scale = 7, 5, 0.37
    q = r.standard_normal((n, d))
    krow = r.standard_normal(d)
    k = np.tile(krow, (n, 1))
    v = r.standard_normal((n, d))
    O, lse = forward(q, k, v, scale)
    _close(O, np.tile(v.mean(0), (n, 1)), 1e-12, "equal keys: O = mean of V")
    _close(lse, scale * q @ krow + math.log(n), 1e-12, "equal keys: lse")
    O, lse = forward(q, k, v, scale, causal=True)
    exp_o = np.stack([v[: i + 1].mean(0) for i in range(n)])
    _close(O, exp_o, 1e-12, "equal keys causal: O = running mean of V")
    _close(lse, scale * q @ krow + np.log(np.arange(1, n + 1)), 1e-12, "equal keys causal: lse")


def check_single_key(forward):
    r = _rng(3)
    q, k, v = (r.standard_normal((1, 4)) for _ in range(3))
    O, lse = forward(q, k, v, 0.8)
    _close(O, v, 1e-15, "N=1: O = V")
    _close(lse, 0.8 * q @ k.T[:, 0], 1e-15, "N=1: lse = scale q.k")


def check_causal_first_row(forward):
    r = _rng(4)
    q, k, v = (r.standard_normal((6, 3)) for _ in range(3))
    O, lse = forward(q, k, v, 1.3, causal=True)
    _close(O[0], v[0], 1e-15, "causal row 0: O_0 = V_0")
    _close(lse[0], 1.3 * q[0] @ k[0], 1e-14, "causal row 0: lse_0 = S_00")


def check_constant_value_column(forward):
    r = _rng(5)
    q, k, v = (r.standard_normal((9, 4)) for _ in range(3))
    v[:, 2] = -1.75
    for causal in (False, True):
        O, _ = forward(q, k, v, 0.5, causal=causal)
        _close(O[:, 2], np.full(9, -1.75), 1e-14, "constant V column passes through")


def check_key_shift(forward):
    r = _rng(6)
    q, k, v = (r.standard_normal((8, 3)) for _ in range(3))
    u = r.standard_normal(3)
    for causal in (False, True):
        O1, lse1 = forward(q, k, v, 0.7, causal=causal)
        O2, lse2 = forward(q, k + u, v, 0.7, causal=causal)
        _close(O1, O2, 1e-12, "key shift leaves O unchanged")
        _close(lse2 - lse1, 0.7 * q @ u, 1e-12, "key shift moves lse by scale q.u")


def check_online_equals_two_pass(forward, online_forward):
    r = _rng(7)
    n, d = 13, 4
    q, k, v = (r.standard_normal((n, d)) for _ in range(3))
    q *= 3.0  # spread the scores so the running maximum moves
    mask = np.array([[1, 0, 1, 0], [0, 1, 1, 0], [1, 1, 1, 0], [0, 0, 1, 1]])
    splits = [list(range(n + 1)), [0, n], [0, 5, n], [0, 1, 2, 7, 12, n]]
    for _ in range(4):
        cuts = sorted(r.choice(np.arange(1, n), size=r.integers(1, 6), replace=False).tolist())
        splits.append([0] + cuts + [n])
    for causal in (False, True):
        for bm in (None, mask):
            O, lse = forward(q, k, v, 0.6, causal=causal, block_mask=bm, tile=4)
            for b in splits:
                O2, lse2 = online_forward(q, k, v, 0.6, b, causal=causal, block_mask=bm, tile=4)
                _close(O2, O, 1e-12, f"online recurrence vs two-pass, split {b}")
                _close(lse2, lse, 1e-12, f"online lse vs two-pass, split {b}")


# ----------------------------------------------------------------------------- gradients

def check_finite_differences(forward, backward):
    r = _rng(8)
    n, d, h = 6, 3, 1e-5
    mask = np.array([[1, 0, 1], [1, 1, 0], [0, 1, 1]])
    for causal, bm in ((False, None), (True, None), (False, mask), (True, mask)):
        q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
        dq, dk, dv = backward(q, k, v, do, 0.45, causal=causal, block_mask=bm, tile=2)

        def L(q_, k_, v_):
            O, _ = forward(q_, k_, v_, 0.45, causal=causal, block_mask=bm, tile=2)
            return float(np.sum(do * O))

        for _ in range(3):
            for which, grad in (("q", dq), ("k", dk), ("v", dv)):
                R = r.standard_normal((n, d))
                args_p = {"q_": q, "k_": k, "v_": v}
                args_m = dict(args_p)
                args_p[which + "_"] = args_p[which + "_"] + h * R
                args_m[which + "_"] = args_m[which + "_"] - h * R
                fd = (L(**args_p) - L(**args_m)) / (2 * h)
                an = float(np.sum(grad * R))
                rel = abs(fd - an) / max(1e-12, abs(an), abs(fd))
                assert rel <= 1e-7, f"finite differences d{which} (causal={causal}, mask={bm is not None}): rel {rel:.2e}"


def check_gradient_identities(forward, backward):
    r = _rng(9)
    n, d = 10, 4
    mask = np.array([[1, 0, 0], [1, 1, 0], [0, 1, 1]])
    for causal, bm in ((False, None), (True, None), (False, mask)):
        q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
        O, _ = forward(q, k, v, 0.5, causal=causal, block_mask=bm, tile=4)
        dq, dk, dv, D = backward(q, k, v, do, 0.5, causal=causal, block_mask=bm, tile=4, return_d=True)
        _close(D, (do * O).sum(1), 1e-12, "D = rowsum(dO∘O) = rowsum(P∘dP)")
        _close(dk.sum(0), np.zeros(d), 1e-12, "Σ_j dK_j = 0")
        _close(dv.sum(0), do.sum(0), 1e-12, "Σ_j dV_j = Σ_i dO_i")


# ----------------------------------------------------------------------------- block-sparse

def check_blocksparse_reductions(forward, backward):
    r = _rng(10)
    n, d, t = 12, 3, 4
    q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
    ones = np.ones((3, 3), dtype=np.uint8)
    for causal in (False, True):
        a = forward(q, k, v, 0.6, causal=causal)
        b = forward(q, k, v, 0.6, causal=causal, block_mask=ones, tile=t)
        _close(a[0], b[0], 0, "all-ones mask = dense (O)")
        _close(a[1], b[1], 0, "all-ones mask = dense (lse)")
        ga = backward(q, k, v, do, 0.6, causal=causal)
        gb = backward(q, k, v, do, 0.6, causal=causal, block_mask=ones, tile=t)
        for x, y in zip(ga, gb):
            _close(x, y, 0, "all-ones mask = dense (grads)")
    # An asymmetric mask fixes its orientation: row I of the mask selects the key
    # tiles J seen by query tile I, so query tile I equals dense attention over
    # the keys of those tiles only.
    asym = np.array([[1, 0, 0], [1, 0, 1], [0, 1, 0]], dtype=np.uint8)
    O, lse = forward(q, k, v, 0.6, block_mask=asym, tile=t)
    for I in range(3):
        rows = slice(I * t, (I + 1) * t)
        keys = np.concatenate([np.arange(J * t, (J + 1) * t) for J in range(3) if asym[I, J]])
        Oi, lsei = forward(q[rows], k[keys], v[keys], 0.6)
        _close(O[rows], Oi, 1e-12, "mask row I selects the key tiles of query tile I (O)")
        _close(lse[rows], lsei, 1e-12, "mask row I selects the key tiles of query tile I (lse)")
    diag = np.eye(3, dtype=np.uint8)
    O, lse = forward(q, k, v, 0.6, block_mask=diag, tile=t)
    g = backward(q, k, v, do, 0.6, block_mask=diag, tile=t)
    for c in range(3):
        s = slice(c * t, (c + 1) * t)
        Oc, lsec = forward(q[s], k[s], v[s], 0.6)
        gc = backward(q[s], k[s], v[s], do[s], 0.6)
        _close(O[s], Oc, 1e-12, "block-diagonal = independent blocks (O)")
        _close(lse[s], lsec, 1e-12, "block-diagonal = independent blocks (lse)")
        for x, y in zip(g, gc):
            _close(x[s], y, 1e-12, "block-diagonal = independent blocks (grads)")


# ----------------------------------------------------------------------------- brute force

def brute_forward(q, k, v, scale, causal):
    """Loop-level reading of the definition, for tiny inputs. With len(q) = n_q
    queries and len(k) = n_k keys, the causal rule lets query i see key j when
    j <= i + n_k - n_q (the queries are the last n_q positions); a query with no
    key gets O = 0 and lse = -inf."""
    n, d = len(q), len(q[0])
    nk = len(k)
    dv = len(v[0])
    O = [[0.0] * dv for _ in range(n)]
    lse = [0.0] * n
    for i in range(n):
        keys = [j for j in range(nk) if (not causal or j <= i + nk - n)]
        if not keys:
            lse[i] = -math.inf
            continue
        s = {j: scale * sum(q[i][t] * k[j][t] for t in range(d)) for j in keys}
        mx = max(s.values())
        e = {j: math.exp(s[j] - mx) for j in keys}
        z = sum(e.values())
        for c in range(dv):
            O[i][c] = sum(e[j] * v[j][c] for j in keys) / z
        lse[i] = mx + math.log(z)
    return O, lse


def check_bruteforce(forward):
    r = _rng(11)
    for n, nk, d, causal in ((1, 1, 1, False), (3, 3, 2, False), (5, 5, 3, True), (6, 6, 4, False), (4, 4, 4, True),
                             (2, 5, 3, True), (5, 2, 3, True), (1, 6, 2, True), (3, 7, 2, False)):
        q = r.standard_normal((n, d))
        k = r.standard_normal((nk, d))
        v2 = r.standard_normal((nk, d + 1))
        Ob, lseb = brute_forward(q.tolist(), k.tolist(), v2.tolist(), 0.9, causal)
        O, lse = forward(q, k, v2, 0.9, causal=causal)
        _close(O, Ob, 1e-13, f"brute force O n={n} nk={nk} d={d}")
        _close(lse, lseb, 1e-13, f"brute force lse n={n} nk={nk} d={d}")


def check_causal_suffix_alignment(forward):
    """N_q < N_k: causal attention of the queries against all keys equals the
    last N_q rows of square causal attention over the key positions (queries
    are the suffix of the sequence). N_q > N_k: the first N_q - N_k rows see no
    key (O = 0, lse = -inf) and the rest equal square causal attention of the
    last N_k queries."""
    r = _rng(12)
    for nq, nk in ((1, 5), (3, 7), (4, 4), (7, 3), (6, 1)):
        d = 3
        q = r.standard_normal((nq, d))
        k = r.standard_normal((nk, d))
        v = r.standard_normal((nk, d))
        O, lse = forward(q, k, v, 0.7, causal=True)
        if nq <= nk:
            qfull = np.concatenate([r.standard_normal((nk - nq, d)), q])
            Of, lsef = forward(qfull, k, v, 0.7, causal=True)
            _close(O, Of[nk - nq:], 1e-13, f"suffix alignment O nq={nq} nk={nk}")
            _close(lse, lsef[nk - nq:], 1e-13, f"suffix alignment lse nq={nq} nk={nk}")
        else:
            e = nq - nk
            assert np.all(O[:e] == 0.0) and np.all(lse[:e] == -np.inf), f"rows without keys nq={nq} nk={nk}"
            Of, lsef = forward(q[e:], k, v, 0.7, causal=True)
            _close(O[e:], Of, 1e-13, f"short keys O nq={nq} nk={nk}")
            _close(lse[e:], lsef, 1e-13, f"short keys lse nq={nq} nk={nk}")


def check_split_kv_merge(forward, split_kv_forward, merge_partials):
    """Split-KV: merging per-split partials equals the one-pass forward for any
    split (sizes down to one key), with causal and block masks and N_q != N_k; a
    split without allowed keys carries lse = -inf and changes nothing."""
    r = _rng(13)
    for nq, nk, causal, mask in ((1, 9, False, None), (1, 9, True, None), (4, 11, True, None),
                                 (7, 5, True, None), (6, 8, False, np.array([[1, 0], [1, 1]], np.uint8))):
        d = 3
        q = r.standard_normal((nq, d))
        k = r.standard_normal((nk, d))
        v = r.standard_normal((nk, d + 1))
        O, lse = forward(q, k, v, 0.8, causal=causal, block_mask=mask, tile=4)
        cuts = sorted(set(r.choice(np.arange(1, nk), size=min(3, nk - 1), replace=False).tolist())) if nk > 1 else []
        for bounds in ([0, nk], [0] + cuts + [nk], list(range(nk + 1))):
            Om, lsem, Os, lses = split_kv_forward(q, k, v, 0.8, bounds, causal=causal, block_mask=mask, tile=4)
            _close(Om, O, 1e-13, f"split-KV O nq={nq} nk={nk} bounds={bounds}")
            _close(lsem, lse, 1e-13, f"split-KV lse nq={nq} nk={nk} bounds={bounds}")
    # An empty split (every key masked for every row) has lse = -inf and no effect;
    # the merge is associative.
    q = r.standard_normal((3, 2))
    k = r.standard_normal((6, 2))
    v = r.standard_normal((6, 2))
    mask = np.array([[1, 0, 1], [1, 0, 1]], np.uint8)  # key block 1 (keys 2, 3) removed for all rows
    O, lse, Os, lses = split_kv_forward(q, k, v, 1.1, [0, 2, 4, 6], block_mask=mask, tile=2)
    assert np.all(lses[1] == -np.inf) and np.all(Os[1] == 0.0), "empty split"
    _merge = merge_partials
    O2, lse2 = _merge([Os[0], Os[2]], [lses[0], lses[2]])
    _close(O2, O, 1e-15, "empty split dropped")
    Oa, lsea = _merge([Os[0], Os[1]], [lses[0], lses[1]])
    O3, lse3 = _merge([Oa, Os[2]], [lsea, lses[2]])
    _close(O3, O, 1e-14, "merge associativity O")
    _close(lse3, lse, 1e-14, "merge associativity lse")


ALL_FORWARD_CHECKS = (
    check_rows_sum_to_one, check_equal_keys, check_single_key, check_causal_first_row,
    check_constant_value_column, check_key_shift, check_bruteforce, check_causal_suffix_alignment,
)


def check_rows_unequal_lengths(forward, forward_rows, backward_rows):
    """The row-restricted routines with N_q != N_k (bottom-right causal diagonal):
    forward_rows equals the rows of the whole forward (itself pinned by brute force
    and suffix alignment), and backward_rows' gradients of
    L = sum over the chosen rows of <dO_i, O_i> match central finite differences
    of that loss computed through the forward."""
    r = _rng(14)
    mask = np.array([[1, 0, 1], [0, 1, 1]], dtype=np.uint8)
    for nq, nk, causal, bm in ((3, 9, True, None), (9, 4, True, None), (5, 7, False, None), (7, 12, True, mask),
                               (8, 5, False, mask[:, :2])):
        d = 3
        q = r.standard_normal((nq, d))
        k = r.standard_normal((nk, d))
        v = r.standard_normal((nk, d))
        do = r.standard_normal((nq, d))
        rows = np.array(sorted(set([0, nq // 2, nq - 1])))
        O, lse = forward(q, k, v, 0.6, causal=causal, block_mask=bm, tile=4)
        Or, lser = forward_rows(q, k, v, 0.6, rows, causal=causal, block_mask=bm, tile=4)
        _close(Or, O[rows], 1e-13, f"forward_rows O nq={nq} nk={nk} causal={causal}")
        _close(lser, lse[rows], 1e-13, f"forward_rows lse nq={nq} nk={nk} causal={causal}")
        o2, l2, dq_r, dk, dv = backward_rows(q, k, v, do, 0.6, rows, causal=causal, block_mask=bm, tile=4)
        _close(o2, O[rows], 1e-13, f"backward_rows O nq={nq} nk={nk}")
        _close(l2, lse[rows], 1e-13, f"backward_rows lse nq={nq} nk={nk}")
        dq = np.zeros_like(q)
        dq[rows] = dq_r

        def L(q_, k_, v_):
            Ox, _ = forward(q_, k_, v_, 0.6, causal=causal, block_mask=bm, tile=4)
            return float(np.sum(do[rows] * Ox[rows]))

        h = 1e-5
        for which, grad in (("q", dq), ("k", dk), ("v", dv)):
            base = {"q": q, "k": k, "v": v}
            R = r.standard_normal(base[which].shape)
            plus = {n: a + h * R if n == which else a for n, a in base.items()}
            minus = {n: a - h * R if n == which else a for n, a in base.items()}
            fd = (L(plus["q"], plus["k"], plus["v"]) - L(minus["q"], minus["k"], minus["v"])) / (2 * h)
            an = float(np.sum(grad * R))
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), \
                f"backward_rows finite differences d{which} nq={nq} nk={nk} causal={causal}: {fd} vs {an}"


# ----------------------------------------------------------------------------- dropout

def check_philox_against_numpy(philox4):
    """The Philox round function and key schedule, through the 4x64 instance,
    against numpy's Philox bit generator (numpy increments its 256-bit counter
    before each block, so its block for counter c is Philox(c + 1))."""
    r = _rng(20)
    for _ in range(20):
        c = [int(x) for x in r.integers(0, 2 ** 63, size=4, dtype=np.uint64)]
        key = [int(x) for x in r.integers(0, 2 ** 63, size=2, dtype=np.uint64)]
        bg = np.random.Philox(key=np.array(key, dtype=np.uint64), counter=np.array(c, dtype=np.uint64))
        got = [int(x) for x in bg.random_raw(4)]
        exp = philox4([c[0] + 1] + c[1:], key, 64)
        assert got == list(exp), "Philox4x64-10 differs from numpy's Philox"


def check_philox_vectorised(philox4, philox4x32_arrays):
    """The numpy-vectorised 4x32 rounds equal the integer rounds, word for word."""
    r = _rng(21)
    c = r.integers(0, 2 ** 32, size=(4, 64), dtype=np.uint64)
    k0, k1 = (int(x) for x in r.integers(0, 2 ** 32, size=2))
    words = philox4x32_arrays(c[0], c[1], c[2], c[3], k0, k1)
    for n in range(64):
        exp = philox4([int(c[w, n]) for w in range(4)], [k0, k1], 32)
        assert [int(words[w][n]) for w in range(4)] == list(exp), "vectorised Philox4x32 differs"


def check_dropout_layout(draws, philox4):
    """Element (i, j) of head bh draws byte (j & 3) of output word (i & 3) of the
    Philox4x32-10 block with counter (j >> 2, i >> 2, bh, 0) and key (seed low, high)."""
    seed = 0x1234_5678_9ABC_DEF0
    for bh in (0, 5):
        u = draws(11, 13, bh, seed)
        for i in range(11):
            for j in range(13):
                w = philox4([j >> 2, i >> 2, bh, 0], [seed & 0xFFFFFFFF, seed >> 32], 32)[i & 3]
                assert u[i, j] == (w >> (8 * (j & 3))) & 0xFF, f"draw layout at ({i}, {j}, {bh})"


def check_dropout_statistics(draws, keep_scale):
    """Draws are uniform bytes; kept entries are scaled so that E[Z] = 1."""
    u = np.concatenate([draws(256, 256, bh, 77 + bh).ravel() for bh in range(4)]).astype(np.float64)
    n = u.size
    counts = np.bincount(u.astype(np.int64), minlength=256)
    mean, sd = n / 256, np.sqrt(n / 256 * (1 - 1 / 256))
    assert np.all(np.abs(counts - mean) <= 6 * sd), "byte draws are not uniform"
    for p in (0.1, 0.5, 0.9):
        Z = np.concatenate([keep_scale(256, 256, bh, 99, p).ravel() for bh in range(4)])
        t = int(np.floor(256 * p + 0.5))
        q = 1 - t / 256
        kept = np.mean(Z > 0)
        assert abs(kept - q) <= 5 * np.sqrt(q * (1 - q) / Z.size), f"keep rate at p={p}"
        assert abs(Z.mean() - 1.0) <= 5 * np.sqrt((1 - q) / q / Z.size), f"E[Z] != 1 at p={p}"


def check_dropout_reductions(forward, backward, forward_dropout, backward_dropout):
    """p = 0 keeps every element with Z = 1: the plain attention."""
    r = _rng(22)
    q, k, v, do = (r.standard_normal((2, 9, 4)) for _ in range(4))
    for causal in (False, True):
        O, lse = forward(q, k, v, 0.5, causal=causal)
        Od, lsed = forward_dropout(q, k, v, 0.5, 0.0, 123, causal=causal)
        _close(Od, O, 1e-13, "dropout p=0 O")
        _close(lsed, lse, 1e-13, "dropout p=0 lse")
        for a, b in zip(backward(q, k, v, do, 0.5, causal=causal), backward_dropout(q, k, v, do, 0.5, 0.0, 123,
                                                                                      causal=causal)):
            _close(b, a, 1e-12, "dropout p=0 gradients")


def check_dropout_finite_differences(forward_dropout, backward_dropout):
    """For a fixed seed the mask is fixed: central differences of L = <dO, O>."""
    r = _rng(23)
    n, nk, d, h = 6, 9, 3, 1e-5
    mask = np.array([[1, 0, 1], [1, 1, 0]], dtype=np.uint8)
    for causal, bm, p in ((False, None, 0.3), (True, None, 0.5), (False, mask, 0.2)):
        q, do = r.standard_normal((n, d)), r.standard_normal((n, d))
        k, v = r.standard_normal((nk, d)), r.standard_normal((nk, d))
        dq, dk, dv, D = backward_dropout(q, k, v, do, 0.45, p, 2024, causal=causal, block_mask=bm, tile=3,
                                         return_d=True)
        O, _ = forward_dropout(q, k, v, 0.45, p, 2024, causal=causal, block_mask=bm, tile=3)
        _close(D, (do * O).sum(axis=1), 1e-12, "dropout: rowsum(P∘dP) = rowsum(dO∘O)")

        def L(q_, k_, v_):
            Ox, _ = forward_dropout(q_, k_, v_, 0.45, p, 2024, causal=causal, block_mask=bm, tile=3)
            return float(np.sum(do * Ox))

        for which, grad in (("q", dq), ("k", dk), ("v", dv)):
            base = {"q": q, "k": k, "v": v}
            R = r.standard_normal(base[which].shape)
            plus = {x: a + h * R if x == which else a for x, a in base.items()}
            minus = {x: a - h * R if x == which else a for x, a in base.items()}
            fd = (L(plus["q"], plus["k"], plus["v"]) - L(minus["q"], minus["k"], minus["v"])) / (2 * h)
            an = float(np.sum(grad * R))
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), f"dropout finite differences d{which}: {fd} vs {an}"
