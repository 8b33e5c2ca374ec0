"""Seeded synthetic inputs for the attention workloads.

This module is shared by the fp64 oracle, the tests and ``bench.py``. It holds
none of the attention arithmetic: only random draws, rounding of those draws to
the 16-bit storage formats, conversions between stored bits and exact values,
and the recipe that draws the fixed block mask of the block-sparse workload.

Recipe (the pages use GPT-2 attention at sequence length 1K, long contexts up to
64K and block-sparse masks; no dataset is needed because attention inputs are
plain tensors):
  * one ``numpy.random.default_rng(seed)`` (PCG64) stream per workload;
  * Q, K, V, dO drawn in that order, each ``standard_normal`` of shape
    [B, H, N, d] in C order (float64);
  * each value rounded to fp16 or bf16 by round-to-nearest, ties-to-even, done
    directly from float64 (no double rounding through float32);
  * both the CUDA path (as 16-bit words) and the oracle (as exact float64
    values) receive the same rounded numbers.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "FORMATS",
    "round_to_format",
    "values_to_bits",
    "bits_to_values",
    "draw_tensor_bits",
    "attention_input_bits",
    "attention_inputs",
    "block_mask_recipe",
    "sample_rows",
    "fp8_attention_input_bits",
]

# (mantissa bits, minimum normal exponent, maximum finite value)
FORMATS = {
    "fp16": (10, -14, 65504.0),
    "bf16": (7, -126, 3.3895313892515355e38),
    "e4m3": (3, -6, 448.0),  # 8-bit float: 4 exponent bits (bias 7), 3 mantissa bits, no infinities
}


def round_to_format(x, fmt: str) -> np.ndarray:
    """Round float64 values to the nearest ``fmt`` value (ties to even).

    Returns float64 values that are exactly representable in ``fmt``. Subnormals
    of the format are handled by clamping the exponent at the minimum normal
    exponent, which gives the subnormal spacing 2**(emin - mantissa).
    """
    mant, emin, fmax = FORMATS[fmt]
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)  # x = f * 2**e with 0.5 <= |f| < 1, so floor(log2|x|) = e - 1
    e = np.maximum(e.astype(np.int64) - 1, emin)
    ulp_exp = (e - mant).astype(np.int64)
    q = np.rint(np.ldexp(x, -ulp_exp))  # exact scaling by a power of two; rint = ties to even
    out = np.ldexp(q, ulp_exp)
    if np.any(np.abs(out) > fmax):
        raise OverflowError(f"value outside the finite range of {fmt}")
    return out


def values_to_bits(vals: np.ndarray, fmt: str) -> np.ndarray:
    """Encode exactly representable float64 values as 16-bit storage words."""
    vals = np.asarray(vals, dtype=np.float64)
    if fmt == "fp16":
        h = vals.astype(np.float16)
        return h.view(np.uint16)
    if fmt == "bf16":
        f = vals.astype(np.float32)  # exact: bf16 is a subset of float32
        return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    if fmt == "e4m3":
        # sign | 4-bit biased exponent | 3-bit mantissa; exponent field 0 holds the
        # subnormals (spacing 2**-9).
        sign = (np.signbit(vals)).astype(np.uint8) << np.uint8(7)
        a = np.abs(vals)
        _, e = np.frexp(a)
        e = np.maximum(e.astype(np.int64) - 1, -6)
        normal = a >= 2.0 ** -6
        mant = np.where(normal, np.rint(np.ldexp(a, -e) * 8) - 8, np.rint(np.ldexp(a, 9)))
        field = np.where(normal, e + 7, 0)
        return (sign | (field.astype(np.uint8) << np.uint8(3)) | mant.astype(np.uint8)).astype(np.uint8)
    raise ValueError(fmt)


def bits_to_values(bits: np.ndarray, fmt: str) -> np.ndarray:
    """Decode 16-bit (or, for e4m3, 8-bit) storage words to exact float64 values."""
    if fmt != "e4m3":
        bits = np.asarray(bits, dtype=np.uint16)
    if fmt == "fp16":
        return bits.view(np.float16).astype(np.float64)
    if fmt == "bf16":
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if fmt == "e4m3":
        b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
        field, mant = (b >> 3) & 15, b & 7
        mag = np.where(field == 0, np.ldexp(mant.astype(np.float64), -9),
                       np.ldexp(1.0 + mant / 8.0, field - 7))
        return np.where(b & 128, -mag, mag)
    raise ValueError(fmt)


def draw_tensor_bits(rng: np.random.Generator, shape, fmt: str, chunk_rows: int = 1 << 22) -> np.ndarray:
    """Draw standard normals of ``shape`` (C order) and return their rounded 16-bit words.

    The draw is made in consecutive chunks of the flattened array; a Generator
    continues its stream across calls, so the result equals one single draw.
    """
    total = int(np.prod(shape))
    out = np.empty(total, dtype=np.uint16)
    pos = 0
    while pos < total:
        n = min(chunk_rows, total - pos)
        out[pos:pos + n] = values_to_bits(round_to_format(rng.standard_normal(n), fmt), fmt)
        pos += n
    return out.reshape(shape)


def attention_input_bits(B: int, H: int, N: int, d: int, fmt: str, seed: int = 0,
                         names=("q", "k", "v", "do")) -> dict:
    """Q, K, V, dO of shape [B, H, N, d] as 16-bit words, drawn in that order."""
    rng = np.random.default_rng(seed)
    out = {}
    for name in ("q", "k", "v", "do"):
        bits = draw_tensor_bits(rng, (B, H, N, d), fmt)
        if name in names:
            out[name] = bits
    return out


def attention_inputs(B: int, H: int, N: int, d: int, fmt: str, seed: int = 0) -> dict:
    """Same draws as :func:`attention_input_bits`, decoded to exact float64 values."""
    bits = attention_input_bits(B, H, N, d, fmt, seed)
    return {k: bits_to_values(v, fmt) for k, v in bits.items()}


def block_mask_recipe(n_tiles: int, density: float = 0.2, seed: int = 0) -> np.ndarray:
    """Fixed tile mask: block diagonal, first block column, and seeded random tiles.

    Of the tiles that are neither diagonal nor in the first column, exactly
    ``round(density * count)`` are switched on, chosen without replacement by a
    seeded permutation. Returns uint8 [n_tiles, n_tiles], row-major.
    """
    m = np.zeros((n_tiles, n_tiles), dtype=np.uint8)
    idx = np.arange(n_tiles)
    m[idx, idx] = 1
    m[:, 0] = 1
    rest = np.flatnonzero(m.reshape(-1) == 0)
    k = int(round(density * rest.size))
    rng = np.random.default_rng(seed)
    chosen = rest[rng.permutation(rest.size)[:k]]
    m.reshape(-1)[chosen] = 1
    return m


def sample_rows(n: int, count: int, seed: int) -> np.ndarray:
    """``count`` distinct row indices in [0, n), drawn without replacement, sorted."""
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(n, size=min(count, n), replace=False))


def fp8_attention_input_bits(B: int, H: int, Nq: int, Nk: int, d: int, seed: int = 0):
    """Q [B, H, Nq, d], K and V [B, H, Nk, d] for the 8-bit forward: standard
    normals drawn in that order from ``default_rng(seed)``, each tensor divided by
    its per-tensor scale s = max|x| / 448 and rounded to e4m3 (nearest, ties to
    even). Returns ({name: uint8 words}, {name: s}); the tensor the attention
    sees is s times the decoded words."""
    rng = np.random.default_rng(seed)
    bits, scales = {}, {}
    for name, n in (("q", Nq), ("k", Nk), ("v", Nk)):
        x = rng.standard_normal((B, H, n, d))
        s = float(np.max(np.abs(x))) / 448.0
        bits[name] = values_to_bits(round_to_format(x / s, "e4m3"), "e4m3")
        scales[name] = s
    return bits, scales
