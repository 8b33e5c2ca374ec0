"""Plant plausible mistakes in a copy of the oracle and require that a pin catches each.

The copy is made from the oracle's source text with one substitution, executed
as a fresh module on the CPU; the real oracle is never modified.
"""
import importlib.util
import os
import types

import pytest

from tests import oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "attention.py")

MUTANTS = {
    "scale dropped from S": ("S = scale * (q @ k.T)                       #", "S = (q @ k.T)                       #"),
    "P transposed in PV": ("O = P @ v ", "O = P.T @ v "),
    "sign flipped in dS": ("dS = P * (dP - D)", "dS = P * (dP + D)"),
    "D term dropped from dS": ("dS = P * (dP - D)", "dS = P * dP"),
    "causal mask off by one": ("<= np.arange(nq)[:, None]", "< np.arange(nq)[:, None]"),
    "scale dropped from dQ": ("dQ = scale * (dS @ k)", "dQ = (dS @ k)"),
    "dS not transposed in dK": ("dK = scale * (dS.T @ q)", "dK = scale * (dS @ q.T).T"),
    "max dropped from lse": ("lse[pos] = m_safe[..., 0][pos] + np.log(l1[pos])", "lse[pos] = np.log(l1[pos])"),
    "P not transposed in dV": ("dV = P.T @ do", "dV = P @ do"),
    "dP operands swapped": ("dP = do @ v.T", "dP = v @ do.T"),
    "block mask transposed": ("a &= bm[np.arange(nq)[:, None] // tile, np.arange(nk)[None, :] // tile]",
                              "a &= bm.T[np.arange(nq)[:, None] // tile, np.arange(nk)[None, :] // tile]"),
    "online rescale of l dropped": ("l = a_old * l + a_new * l_t", "l = l + a_new * l_t"),
    "online rescale of O dropped": ("O = a_old[:, None] * O + a_new[:, None] * O_t", "O = O + a_new[:, None] * O_t"),
    "causal diagonal not shifted for N_q != N_k": ("<= np.arange(nq)[:, None] + (nk - nq)", "<= np.arange(nq)[:, None]"),
    "split-KV merge without the lse weights": ("w = np.exp(lses - m_safe)", "w = np.ones_like(lses)"),
    "split-KV merged lse without the max": ("lse[pos] = m_safe[pos] + np.log(z[pos])", "lse[pos] = np.log(z[pos])"),
    "row routines' causal diagonal not shifted for N_q != N_k": ("a &= cols[None, :] <= rows[:, None] + offset",
                                                                 "a &= cols[None, :] <= rows[:, None]"),
}


def _mutant(old, new):
    with open(SRC) as f:
        text = f.read()
    assert text.count(old) >= 1, f"mutation site not found: {old!r}"
    text = text.replace(old, new)
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = SRC
    exec(compile(text, SRC + " (mutant)", "exec"), mod.__dict__)
    return mod


def _run_all(mod):
    failures = []
    checks = [
        lambda: pins.check_closed_forms(mod.forward, mod.backward),
        lambda: pins.check_online_equals_two_pass(mod.forward, mod.online_forward),
        lambda: pins.check_finite_differences(mod.forward, mod.backward),
        lambda: pins.check_gradient_identities(mod.forward, mod.backward),
        lambda: pins.check_blocksparse_reductions(mod.forward, mod.backward),
        lambda: pins.check_split_kv_merge(mod.forward, mod.split_kv_forward, mod.merge_partials),
        lambda: pins.check_rows_unequal_lengths(mod.forward, mod.forward_rows, mod.backward_rows),
    ] + [lambda c=c: c(mod.forward) for c in pins.ALL_FORWARD_CHECKS]
    for c in checks:
        try:
            c()
        except AssertionError as e:
            failures.append(str(e))
        except Exception as e:  # a crash also counts as caught
            failures.append(repr(e))
    return failures


DROPOUT_SRC = os.path.join(os.path.dirname(SRC), "dropout.py")

DROPOUT_MUTANTS = {
    "dropout scale 1/q dropped": ("256.0 / (256 - t), 0.0)", "1.0, 0.0)"),
    "dropout mask missing from dP": ("dP = (do[idx] @ v[idx].T) * Z", "dP = (do[idx] @ v[idx].T)"),
    "dropout counter rows and columns swapped": ("philox4x32_arrays(j >> np.uint64(2), i >> np.uint64(2),",
                                                 "philox4x32_arrays(i >> np.uint64(2), j >> np.uint64(2),"),
    "dropout word picked by column": ("sel = (i & np.uint64(3))", "sel = (j & np.uint64(3))"),
    "Philox key bump missing": ("kk0, kk1 = (kk0 + w0) & 0xFFFFFFFF, (kk1 + w1) & 0xFFFFFFFF",
                                "kk0, kk1 = kk0, kk1"),
    "Philox high and low halves swapped": ("x0, x1, x2, x3 = (p1 >> width) ^ x1 ^ k0, p1 & mask,",
                                           "x0, x1, x2, x3 = (p1 & mask) ^ x1 ^ k0, p1 >> width,"),
    "dropout keeps draws below the threshold": ("np.where(draws(nq, nk, bh, seed) >= t,",
                                                "np.where(draws(nq, nk, bh, seed) < t,"),
}


def _dropout_mutant(old, new):
    import oracle
    with open(DROPOUT_SRC) as f:
        text = f.read()
    assert text.count(old) >= 1, f"mutation site not found: {old!r}"
    text = text.replace(old, new).replace("from .attention import", "from oracle.attention import")
    mod = types.ModuleType("oracle_dropout_mutant")
    mod.__file__ = DROPOUT_SRC
    exec(compile(text, DROPOUT_SRC + " (mutant)", "exec"), mod.__dict__)
    return oracle, mod


def _run_dropout(oracle, mod):
    failures = []
    checks = [
        lambda: pins.check_philox_against_numpy(mod.philox4),
        lambda: pins.check_philox_vectorised(mod.philox4, mod.philox4x32_arrays),
        lambda: pins.check_dropout_layout(mod.draws, mod.philox4),
        lambda: pins.check_dropout_statistics(mod.draws, mod.keep_scale),
        lambda: pins.check_dropout_reductions(oracle.forward, oracle.backward, mod.forward_dropout,
                                              mod.backward_dropout),
        lambda: pins.check_dropout_finite_differences(mod.forward_dropout, mod.backward_dropout),
    ]
    for c in checks:
        try:
            c()
        except AssertionError as e:
            failures.append(str(e))
        except Exception as e:  # a crash also counts as caught
            failures.append(repr(e))
    return failures


def test_unmutated_dropout_copy_passes():
    assert _run_dropout(*_dropout_mutant("import numpy as np", "import numpy as np")) == []


@pytest.mark.parametrize("name", sorted(DROPOUT_MUTANTS))
def test_dropout_mutant_is_caught(name):
    old, new = DROPOUT_MUTANTS[name]
    assert _run_dropout(*_dropout_mutant(old, new)), f"no pin caught the planted mistake: {name}"


def test_unmutated_copy_passes():
    with open(SRC) as f:
        text = f.read()
    mod = types.ModuleType("oracle_copy")
    exec(compile(text, SRC, "exec"), mod.__dict__)
    assert _run_all(mod) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    assert _run_all(_mutant(old, new)), f"no pin caught the planted mistake: {name}"
