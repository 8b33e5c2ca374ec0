"""fp64 oracle for attention with dropout on P (test infrastructure).

Only ``tests/`` and the CPU legs of ``bench.py`` use this module; it shares no
code with the CUDA library. Page keys are defined in ``oracle/__init__.py``.

[card] 算法要点, "Kernel fusion": the fused kernel runs QKᵀ → softmax (+ mask /
dropout) → PV without writing the intermediate to HBM. The pages name dropout
as part of that fusion but fix neither its generator nor its formula. Readings
taken here:
  * dropout acts on the normalised probabilities: with keep decisions M and
    keep probability q, Z = M / q and O = (P∘Z)·V, P = softmax(S) as without
    dropout; the saved lse is that of the undropped softmax;
  * the keep decisions are not stored: they come from a counter-based generator,
    Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
    as 1, 2, 3", SC'11), from the seed and the element's position, so the
    backward draws them again ([card] 反向：重算而非存储 applied to the mask);
  * one generator call covers a 4×4 block of (query row i, key column j): counter
    words (j >> 2, i >> 2, b·H + h, 0), key words (seed mod 2³², seed >> 32); the
    call's output word (i & 3) holds row i's four draws, byte (j & 3) of it
    (least significant first) is element (i, j)'s draw u ∈ {0, …, 255};
  * the drop probability is rounded to t/256 with t = ⌊256·p + ½⌋ (halves round
    up): the element is kept iff u ≥ t, so q = 1 − t/256 and kept entries of Z
    are 256/(256 − t).

Backward, by the chain rule through O = (P∘Z)V: dV = (P∘Z)ᵀ dO, dP = (dO Vᵀ)∘Z,
D = rowsum(P∘dP) (which equals rowsum(dO∘O)), dS = P∘(dP − D), dQ = scale·dS K,
dK = scale·dSᵀ Q.
"""
from __future__ import annotations

import numpy as np

from .attention import _softmax_rows, allowed_mask, TILE

# Philox constants (Salmon et al., SC'11): round multipliers and Weyl key increments.
PHILOX = {
    32: {"mult": (0xD2511F53, 0xCD9E8D57), "weyl": (0x9E3779B9, 0xBB67AE85)},
    64: {"mult": (0xD2E7470EE14C6C93, 0xCA5A826395121157), "weyl": (0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B)},
}


def philox4(counter, key, width: int, rounds: int = 10):
    """Philox4xW-R on Python integers: four counter words, two key words, W = 32 or 64.

    Each round multiplies counter words 0 and 2 by the two round multipliers
    (double-width products split into high and low halves), then
        (x0, x1, x2, x3) ← (hi(M1·x2) ⊕ x1 ⊕ k0, lo(M1·x2), hi(M0·x0) ⊕ x3 ⊕ k1, lo(M0·x0)),
    and the key is bumped by the Weyl constants between rounds.
    """
    mask = (1 << width) - 1
    m0, m1 = PHILOX[width]["mult"]
    w0, w1 = PHILOX[width]["weyl"]
    x0, x1, x2, x3 = (int(c) & mask for c in counter)
    k0, k1 = (int(k) & mask for k in key)
    for r in range(rounds):
        if r:
            k0, k1 = (k0 + w0) & mask, (k1 + w1) & mask
        p0, p1 = m0 * x0, m1 * x2
        x0, x1, x2, x3 = (p1 >> width) ^ x1 ^ k0, p1 & mask, (p0 >> width) ^ x3 ^ k1, p0 & mask
    return x0, x1, x2, x3


def philox4x32_arrays(c0, c1, c2, c3, k0: int, k1: int, rounds: int = 10):
    """The same Philox4x32 rounds on numpy arrays of counter words (vectorised;
    the 32 x 32-bit products are exact in uint64)."""
    lo32 = np.uint64(0xFFFFFFFF)
    m0, m1 = (np.uint64(m) for m in PHILOX[32]["mult"])
    w0, w1 = PHILOX[32]["weyl"]
    x = [np.asarray(c, dtype=np.uint64) & lo32 for c in (c0, c1, c2, c3)]
    x0, x1, x2, x3 = np.broadcast_arrays(*x)
    kk0, kk1 = k0 & 0xFFFFFFFF, k1 & 0xFFFFFFFF
    for r in range(rounds):
        if r:
            kk0, kk1 = (kk0 + w0) & 0xFFFFFFFF, (kk1 + w1) & 0xFFFFFFFF
        p0, p1 = m0 * x0, m1 * x2
        x0, x1, x2, x3 = ((p1 >> np.uint64(32)) ^ x1 ^ np.uint64(kk0), p1 & lo32,
                          (p0 >> np.uint64(32)) ^ x3 ^ np.uint64(kk1), p0 & lo32)
    return x0, x1, x2, x3


def drop_threshold(p_drop: float) -> int:
    """t with drop probability t/256 (the reading above); 0 <= p < 1."""
    if not 0.0 <= p_drop < 1.0:
        raise ValueError("dropout probability must be in [0, 1)")
    return min(255, int(np.floor(256.0 * p_drop + 0.5)))


def draws(nq: int, nk: int, bh: int, seed: int) -> np.ndarray:
    """uint8 [nq, nk]: the draw u of every element (i, j) of head bh."""
    i = np.arange(nq, dtype=np.uint64)[:, None]
    j = np.arange(nk, dtype=np.uint64)[None, :]
    words = philox4x32_arrays(j >> np.uint64(2), i >> np.uint64(2), np.uint64(bh), np.uint64(0),
                              seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    sel = (i & np.uint64(3)).astype(np.int64)           # output word of row i
    w = np.choose(np.broadcast_to(sel, (nq, nk)), [np.broadcast_to(x, (nq, nk)) for x in words])
    return ((w >> ((j & np.uint64(3)) * np.uint64(8))) & np.uint64(0xFF)).astype(np.uint8)


def keep_scale(nq: int, nk: int, bh: int, seed: int, p_drop: float) -> np.ndarray:
    """Z [nq, nk]: 256/(256 - t) where the element is kept, 0 where it is dropped."""
    t = drop_threshold(p_drop)
    return np.where(draws(nq, nk, bh, seed) >= t, 256.0 / (256 - t), 0.0)


def _heads(q):
    lead = q.shape[:-2]
    return lead, list(np.ndindex(*lead))


def forward_dropout(q, k, v, scale: float, p_drop: float, seed: int, causal: bool = False, block_mask=None,
                    tile: int = TILE):
    """O = (P∘Z)·V and lse of the undropped softmax, for inputs [..., N, d]; the
    flat index of the leading dimensions is the head index b·H + h of the counter."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    lead, heads = _heads(q)
    nq, nk = q.shape[-2], k.shape[-2]
    allowed = allowed_mask(nq, nk, causal, block_mask, tile)
    O = np.empty(lead + (nq, v.shape[-1]))
    lse = np.empty(lead + (nq,))
    for bh, idx in enumerate(heads):
        S = np.where(allowed, scale * (q[idx] @ k[idx].T), -np.inf)
        P, lse[idx] = _softmax_rows(S)
        O[idx] = (P * keep_scale(nq, nk, bh, seed, p_drop)) @ v[idx]
    return O, lse


def backward_dropout(q, k, v, do, scale: float, p_drop: float, seed: int, causal: bool = False, block_mask=None,
                     tile: int = TILE, return_d: bool = False):
    """dQ, dK, dV of a loss with ∂L/∂O = dO through O = (P∘Z)·V (chain rule)."""
    q, k, v, do = (np.asarray(t, dtype=np.float64) for t in (q, k, v, do))
    lead, heads = _heads(q)
    nq, nk = q.shape[-2], k.shape[-2]
    allowed = allowed_mask(nq, nk, causal, block_mask, tile)
    dQ, dK, dV = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    D = np.empty(lead + (nq,))
    for bh, idx in enumerate(heads):
        S = np.where(allowed, scale * (q[idx] @ k[idx].T), -np.inf)
        P, _ = _softmax_rows(S)
        Z = keep_scale(nq, nk, bh, seed, p_drop)
        dV[idx] = (P * Z).T @ do[idx]                    # dV = (P∘Z)ᵀ dO
        dP = (do[idx] @ v[idx].T) * Z                    # dP = (dO Vᵀ)∘Z
        Di = (P * dP).sum(axis=1, keepdims=True)         # D = rowsum(P∘dP)
        dS = P * (dP - Di)                               # softmax Jacobian
        dQ[idx] = scale * (dS @ k[idx])
        dK[idx] = scale * (dS.T @ q[idx])
        D[idx] = Di[:, 0]
    return (dQ, dK, dV, D) if return_d else (dQ, dK, dV)
