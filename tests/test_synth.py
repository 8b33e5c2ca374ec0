"""The seeded input module: rounding, encodings, stream continuity and the block-mask recipe."""
import numpy as np
import pytest
import torch

import fa_synth as S


@pytest.mark.parametrize("fmt,tdtype", [("bf16", torch.bfloat16), ("fp16", torch.float16)])
def test_rounding_matches_torch_on_float32_inputs(fmt, tdtype):
    # float32 inputs round once to the 16-bit format, so torch's RNE conversion is a reference.
    r = np.random.default_rng(0)
    x = np.concatenate([r.standard_normal(200000), r.standard_normal(1000) * 1e-6,
                        r.standard_normal(1000) * 1e3]).astype(np.float32)
    ours = S.round_to_format(x.astype(np.float64), fmt)
    ref = torch.from_numpy(x).to(tdtype).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


def test_ties_go_to_even():
    # bf16 spacing at 1.0 is 2**-7: 1 + 2**-8 is a tie between 1 and 1 + 2**-7 -> 1 (even).
    assert S.round_to_format(np.array([1 + 2 ** -8]), "bf16")[0] == 1.0
    # 1 + 3*2**-8 is a tie between 1 + 2**-7 (odd) and 1 + 2**-6 (even) -> 1 + 2**-6.
    assert S.round_to_format(np.array([1 + 3 * 2 ** -8]), "bf16")[0] == 1 + 2 ** -6
    # fp16 subnormal spacing is 2**-24: 2**-25 ties to 0, 3*2**-25 ties to 2*2**-24.
    assert S.round_to_format(np.array([2.0 ** -25]), "fp16")[0] == 0.0
    assert S.round_to_format(np.array([3 * 2.0 ** -25]), "fp16")[0] == 2 * 2.0 ** -24


def test_direct_rounding_from_float64():
    # A float64 just above a bf16 tie must round up; rounding through float32 would tie to even.
    x = 1 + 2 ** -8 + 2 ** -40
    assert S.round_to_format(np.array([x]), "bf16")[0] == 1 + 2 ** -7


@pytest.mark.parametrize("fmt", ["bf16", "fp16"])
def test_bits_roundtrip(fmt):
    r = np.random.default_rng(1)
    v = S.round_to_format(r.standard_normal(10000), fmt)
    bits = S.values_to_bits(v, fmt)
    assert bits.dtype == np.uint16
    assert np.array_equal(S.bits_to_values(bits, fmt), v)


def test_chunked_draw_equals_single_draw():
    a = S.draw_tensor_bits(np.random.default_rng(5), (3, 1000), "bf16", chunk_rows=77)
    b = S.values_to_bits(S.round_to_format(np.random.default_rng(5).standard_normal((3, 1000)), "bf16"), "bf16")
    assert np.array_equal(a, b)


def test_inputs_drawn_in_order():
    bits = S.attention_input_bits(1, 2, 16, 8, "fp16", seed=0)
    r = np.random.default_rng(0)
    for name in ("q", "k", "v", "do"):
        exp = S.values_to_bits(S.round_to_format(r.standard_normal((1, 2, 16, 8)), "fp16"), "fp16")
        assert np.array_equal(bits[name], exp), name


def test_block_mask_recipe_counts():
    m = S.block_mask_recipe(64)
    assert m.shape == (64, 64) and m.dtype == np.uint8
    assert np.all(np.diag(m) == 1) and np.all(m[:, 0] == 1)
    rest = 64 * 64 - 64 - 63
    assert int(m.sum()) == 64 + 63 + round(0.2 * rest) == 921
    assert np.array_equal(m, S.block_mask_recipe(64))


def test_e4m3_rounding_and_encoding_match_torch():
    # Round to nearest (ties to even) onto the e4m3 grid, and the 8-bit encoding,
    # against torch's float8_e4m3fn conversion (a library routine).
    import torch
    r = np.random.default_rng(0)
    x = np.concatenate([r.standard_normal(50000) * 100, r.standard_normal(5000) * 0.01,
                        np.array([0.0, -0.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -6, 3 * 2.0 ** -9, 17.0, 19.0])])
    x = np.clip(x, -448.0, 448.0)
    ours = S.round_to_format(x, "e4m3")
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(ours, ref.to(torch.float64).numpy())
    bits = S.values_to_bits(ours, "e4m3")
    assert np.array_equal(bits, ref.view(torch.uint8).numpy())
    assert np.array_equal(S.bits_to_values(bits, "e4m3"), ours)


def test_fp8_inputs_use_the_e4m3_range():
    bits, scales = S.fp8_attention_input_bits(1, 2, 100, 300, 64, seed=3)
    assert bits["q"].shape == (1, 2, 100, 64) and bits["k"].shape == (1, 2, 300, 64)
    for name in ("q", "k", "v"):
        vals = S.bits_to_values(bits[name], "e4m3")
        assert np.max(np.abs(vals)) == 448.0  # the per-tensor scale maps max|x| to the largest e4m3 value
        assert scales[name] > 0
