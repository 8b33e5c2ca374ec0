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
