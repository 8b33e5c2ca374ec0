"""8-bit forward (fa_fwd_fp8) against the fp64 oracle.

Inputs: e4m3 Q, K, V with per-tensor scales (``fa_synth.fp8_attention_input_bits``);
the oracle runs the plain definition on the tensors they stand for (scale times
the decoded e4m3 values). S is formed from the exact stored values with fp32
accumulation and P V runs in bf16, as in the 16-bit path, so the tolerances are
those of the forward: O max-abs <= 1e-2, lse max-abs <= 1e-3."""
import numpy as np
import pytest
import torch

import fa_synth as S
import io_aware_exact_19_b200 as fa
import oracle
from tests.gpu_inputs import max_abs

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3


def _run(B, H, Nq, Nk, causal, mask=None, seed=0, heads=None):
    d = 128
    bits, sc = S.fp8_attention_input_bits(B, H, Nq, Nk, d, seed=seed)
    dev = {n: torch.from_numpy(b).cuda() for n, b in bits.items()}
    o = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    mdev = None if mask is None else torch.from_numpy(mask).cuda()
    fa.fa_fwd_fp8(dev["q"], dev["k"], dev["v"], sc["q"], sc["k"], sc["v"], o, lse, causal=causal, block_mask=mdev)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK

    def vals(n):
        x = bits[n].reshape((-1,) + bits[n].shape[2:])
        if heads is not None:
            x = x[list(heads)]
        return sc[n] * S.bits_to_values(x, "e4m3")

    O, L = oracle.forward(vals("q"), vals("k"), vals("v"), 1.0 / np.sqrt(d), causal=causal, block_mask=mask)
    got_o = o.float().cpu().numpy().reshape(B * H, Nq, d)
    got_l = lse.cpu().numpy().reshape(B * H, Nq)
    if heads is not None:
        got_o, got_l = got_o[list(heads)], got_l[list(heads)]
    eo, el = max_abs(got_o, O), max_abs(got_l, L)
    assert eo <= O_TOL and el <= LSE_TOL, f"O {eo:.3e} lse {el:.3e}"
    return eo, el


@pytest.mark.parametrize("B,H,Nq,Nk,causal", [
    (1, 2, 1000, 1000, True), (2, 2, 384, 777, False), (1, 1, 1, 300, True), (1, 2, 129, 129, False),
    (1, 3, 640, 1280, True),
])
def test_fp8_forward_matches_oracle(B, H, Nq, Nk, causal):
    _run(B, H, Nq, Nk, causal, seed=Nq + Nk)


def test_fp8_forward_block_sparse():
    mask = np.array([[1, 0, 1, 1], [0, 1, 0, 1]], dtype=np.uint8)
    _run(1, 2, 256, 512, False, mask=mask, seed=5)


def test_fp8_long_context_causal_heads():
    # The long-context causal workload's shape, in 8 bits; four heads checked.
    _run(4, 16, 4096, 4096, True, heads=[0, 21, 42, 63])
