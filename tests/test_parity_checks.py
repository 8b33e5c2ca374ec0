"""The gradient comparison the GPU parity tests use (tests.gpu_inputs.grad_errors)
must catch the mistakes a whole-tensor norm hides: one wrong row, one wrong
ragged tail tile, one wrong element. Checked here on the CPU with planted errors."""
import numpy as np

from tests.gpu_inputs import G_ELEM_TOL, G_TOL, grad_errors


def _noisy(shape, rel, seed):
    r = np.random.default_rng(seed)
    G = r.standard_normal(shape)
    return G, G * (1 + rel * r.standard_normal(shape))


def _passes(e):
    return e["fro"] <= G_TOL and e["tile"] <= G_TOL and e["elem"] <= G_ELEM_TOL


def test_accurate_gradient_passes():
    G, g = _noisy((6, 1000, 64), 3e-3, 0)
    assert _passes(grad_errors(g, G))


def test_one_wrong_row_fails_although_the_norm_passes():
    G, g = _noisy((6, 1000, 64), 3e-3, 1)
    g[3, 517] = np.random.default_rng(2).standard_normal(64)  # a completely wrong row
    e = grad_errors(g, G)
    assert e["fro"] <= G_TOL            # the whole-tensor norm alone misses it
    assert not _passes(e)


def test_wrong_ragged_tail_tile_fails():
    G, g = _noisy((2, 1000, 64), 3e-3, 3)
    g[1, 896:] *= 1.05                   # 104 tail rows 5% off
    e = grad_errors(g, G)
    assert e["fro"] <= G_TOL and e["tile"] > G_TOL


def test_one_wrong_element_fails():
    G, g = _noisy((4, 512, 128), 3e-3, 4)
    g[2, 100, 7] += 0.5 * np.sqrt(np.mean(G * G)) * 2
    assert not _passes(grad_errors(g, G))


def test_exactly_zero_gradient_uses_the_absolute_floor():
    G = np.zeros((1, 1, 64))
    assert _passes(grad_errors(np.full_like(G, 1e-6), G))
    assert not _passes(grad_errors(np.full_like(G, 1e-3), G))
