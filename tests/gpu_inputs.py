"""Seeded inputs on the GPU: the same 16-bit words the oracle decodes to float64."""
import numpy as np
import torch

import fa_synth as S

TORCH_DT = {"bf16": torch.bfloat16, "fp16": torch.float16}


def to_device(bits: np.ndarray, fmt: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(TORCH_DT[fmt]).cuda()


class Case:
    """Q, K, V, dO of one workload as device tensors and as exact float64 values."""

    def __init__(self, B, H, N, d, fmt, seed=0):
        self.shape = (B, H, N, d)
        self.fmt = fmt
        self.scale = 1.0 / np.sqrt(d)
        bits = S.attention_input_bits(B, H, N, d, fmt, seed)
        self.bits = bits
        self.dev = {k: to_device(v, fmt) for k, v in bits.items()}

    def values(self, name, heads=None):
        """Exact float64 values, flattened to [B*H, N, d] (optionally a subset of heads)."""
        x = self.bits[name]
        x = x.reshape((-1,) + x.shape[2:])
        if heads is not None:
            x = x[list(heads)]
        return S.bits_to_values(x, self.fmt)

    def flat(self, t: torch.Tensor, heads=None):
        """Device result -> float64 numpy, optionally restricted to flat (b*H+h) heads."""
        a = t.float().cpu().numpy().astype(np.float64)
        a = a.reshape((-1,) + a.shape[2:])
        return a if heads is None else a[list(heads)]


def max_abs(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    return float(np.max(np.where(both_inf, 0.0, np.abs(a - b)))) if a.size else 0.0


def rel_fro(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def grad_errors(g, G, tile=128, floor=1e-4):
    """Errors of a gradient g against the oracle's G, both [heads, rows, d]:

    * ``fro``: relative Frobenius error over the whole tensor (the stated metric);
    * ``tile``: the worst relative Frobenius error of one block of ``tile``
      consecutive rows of one head, its denominator floored at the norm such a
      block would have at the tensor's RMS, so one wrong row or ragged tail tile
      cannot hide inside a large tensor;
    * ``elem``: the largest element error relative to (the tensor's RMS + the
      RMS of that element's row): the 16-bit rounding of P and dS errs in
      proportion to a row's magnitude, and rows that see few keys are tens of
      times the tensor's RMS.

    The RMS has an absolute floor (``floor``) so a gradient that is exactly zero in
    exact arithmetic (a single key: P = 1, dS = 0) is compared against that scale.
    """
    g = np.asarray(g, np.float64)
    G = np.asarray(G, np.float64)
    assert g.shape == G.shape, (g.shape, G.shape)
    err = g - G
    rms = max(float(np.sqrt(np.mean(G * G))) if G.size else 0.0, floor)
    fro = float(np.linalg.norm(err) / max(np.linalg.norm(G), rms * np.sqrt(max(G.size, 1))))
    worst = 0.0
    rows = G.shape[-2]
    E = err.reshape((-1,) + G.shape[-2:])
    R = G.reshape((-1,) + G.shape[-2:])
    for r0 in range(0, rows, tile):
        e_blk = E[:, r0:r0 + tile]
        g_blk = R[:, r0:r0 + tile]
        num = np.sqrt((e_blk * e_blk).sum(axis=(1, 2)))
        den = np.maximum(np.sqrt((g_blk * g_blk).sum(axis=(1, 2))), rms * np.sqrt(e_blk[0].size))
        worst = max(worst, float(np.max(num / den)))
    row_rms = np.sqrt(np.mean(G * G, axis=-1, keepdims=True))
    elem = float(np.max(np.abs(err) / (rms + row_rms))) if err.size else 0.0
    return {"fro": fro, "tile": worst, "elem": elem}


# Gradient bounds: relative Frobenius <= 2e-2 over the tensor and over every block
# of rows; every element within 10% of (RMS + its row's RMS), so a single wrong
# element of typical size fails. The element bound is looser than the norms
# because D = rowsum(dO o O) is formed from the 16-bit O: in a row with few keys
# and one dominant P, dS = P o (dP - D) is a small difference and errs by a few
# per cent of the row (measured: up to 5.5% at B=8 H=12 N=1024 d=64 causal).
G_TOL = 2e-2
G_ELEM_TOL = 0.1


def assert_grads(pairs, tile=128, what="dQ/dK/dV", elem_tol=G_ELEM_TOL):
    """Assert the gradient bounds for a sequence of (g, G) pairs; returns their errors."""
    errs = [grad_errors(g, G, tile) for g, G in pairs]
    bad = [e for e in errs if e["fro"] > G_TOL or e["tile"] > G_TOL or e["elem"] > elem_tol]
    assert not bad, f"{what} errors {errs}"
    return errs
