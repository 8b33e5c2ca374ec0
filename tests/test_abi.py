"""The C-ABI library: it builds, loads, exports every symbol include/fa.h declares,
and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

import io_aware_exact_19_b200 as fa
from io_aware_exact_19_b200 import build as fa_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("fa_fwd", "fa_bwd", "fa_blocksparse_fwd", "fa_blocksparse_bwd", "fa_bwd_workspace_size"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(_declared_functions()) == set(fa.EXPORTED)


def test_status_strings(lib):
    for code, name in enumerate(["FA_OK", "FA_ERR_INVALID_ARG", "FA_ERR_UNSUPPORTED", "FA_ERR_CUDA", "FA_ERR_TIMEOUT"]):
        assert lib.fa_status_string(code).decode() == name


def test_workspace_is_linear_in_n(lib):
    sizes = [lib.fa_bwd_workspace_size(1, 16, n, 64) for n in (1024, 2048, 4096, 8192, 16384, 32768, 65536)]
    diffs = [b - a for a, b in zip(sizes, sizes[1:])]
    # doubling N doubles the increment: no N^2 term
    for a, b in zip(diffs, diffs[1:]):
        assert b == 2 * a
    assert lib.fa_bwd_workspace_size(1, 16, 65536, 64) == 1 * 16 * 65536 * 8
    assert lib.fa_bwd_workspace_size(1, 1, 100, 80) == 0
    assert lib.fa_bwd_workspace_size(1, 1, 100, 96) == lib.fa_bwd_workspace_size(1, 1, 100, 64)


def _fake(addr=4096):
    return ctypes.c_void_p(addr)


def test_host_argument_errors_return_before_launch(lib):
    p = _fake()
    # unsupported head dimension (32, 64, 96 and 128 are supported)
    for d in (16, 48, 80, 160, 512):
        assert lib.fa_fwd(1, p, p, p, p, p, 1, 1, 128, d, 0.1, 0, None) == fa.FA_ERR_UNSUPPORTED
    # non-positive sizes, bad dtype
    assert lib.fa_fwd(1, p, p, p, p, p, 0, 1, 128, 64, 0.1, 0, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd(1, p, p, p, p, p, 1, 1, 0, 64, 0.1, 0, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd(7, p, p, p, p, p, 1, 1, 128, 64, 0.1, 0, None) == fa.FA_ERR_INVALID_ARG
    # null and misaligned pointers
    assert lib.fa_fwd(1, None, p, p, p, p, 1, 1, 128, 64, 0.1, 0, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd(1, _fake(4100), p, p, p, p, 1, 1, 128, 64, 0.1, 0, None) == fa.FA_ERR_INVALID_ARG
    # block-sparse needs N % 128 == 0 and a mask
    assert lib.fa_blocksparse_fwd(1, p, p, p, p, p, 1, 1, 1000, 64, 0.1, 0, p, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_blocksparse_fwd(1, p, p, p, p, p, 1, 1, 1024, 64, 0.1, 0, None, None) == fa.FA_ERR_INVALID_ARG
    # backward: workspace must be 256-byte aligned
    assert lib.fa_bwd(1, p, p, p, p, p, p, p, p, p, _fake(4096 + 16), 1, 1, 128, 64, 0.1, 0, None) \
        == fa.FA_ERR_INVALID_ARG
    assert lib.fa_debug_timeout_probe(0, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_debug_fwd_withhold(1, p, p, p, p, p, 1, 1, 128, 64, 0.1, 0, 0, None) == fa.FA_ERR_INVALID_ARG
    # d = 256 is forward-only
    assert lib.fa_bwd(1, p, p, p, p, p, p, p, p, p, p, 1, 1, 128, 256, 0.1, 0, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_bwd_workspace_size(1, 1, 128, 256) == 0
    assert lib.fa_bwd_noalloc(1, p, p, p, p, p, p, p, p, p, 1, 1, 128, 256, 0.1, 0, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_fwd_dropout(1, p, p, p, p, p, 1, 1, 128, 128, 256, 0.1, 0, None, 0.5, 1, None) \
        == fa.FA_ERR_UNSUPPORTED
    # 8-bit forward: d = 128 only, positive finite scales
    assert lib.fa_fwd_fp8(p, p, p, 1.0, 1.0, 1.0, p, p, 1, 1, 128, 128, 64, 0.1, 0, None, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_fwd_fp8(p, p, p, 0.0, 1.0, 1.0, p, p, 1, 1, 128, 128, 128, 0.1, 0, None, None) \
        == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_fp8(p, p, p, 1.0, float("inf"), 1.0, p, p, 1, 1, 128, 128, 128, 0.1, 0, None, None) \
        == fa.FA_ERR_INVALID_ARG
    # dropout: probability in [0, 1)
    for pd in (-0.1, 1.0, float("nan")):
        assert lib.fa_fwd_dropout(1, p, p, p, p, p, 1, 1, 128, 128, 64, 0.1, 0, None, pd, 1, None) \
            == fa.FA_ERR_INVALID_ARG
        assert lib.fa_bwd_dropout(1, p, p, p, p, p, p, p, p, p, p, 1, 1, 128, 128, 64, 0.1, 0, None, pd, 1, None) \
            == fa.FA_ERR_INVALID_ARG
    assert lib.fa_debug_dropout_draws(1, 1, 0, 5, 1, p, p, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_debug_bwd_withhold(1, p, p, p, p, p, p, p, p, p, p, 1, 1, 128, 64, 0.1, 0, 9999, None) \
        == fa.FA_ERR_INVALID_ARG
    # split-KV: range count within 1..ceil(Nk/128), aligned workspace, sizes
    assert lib.fa_fwd_splitkv(1, p, p, p, p, p, 1, 1, 1, 1000, 64, 0.1, 1, None, 0, p, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_splitkv(1, p, p, p, p, p, 1, 1, 1, 1000, 64, 0.1, 1, None, 9, p, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_splitkv(1, p, p, p, p, p, 1, 1, 1, 1000, 64, 0.1, 1, None, 4, _fake(4096 + 16), None) \
        == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_splitkv(1, p, p, p, p, p, 1, 1, 1, 1000, 80, 0.1, 1, None, 4, p, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_fwd_splitkv(1, p, p, p, p, p, 1, 1, 1, 1000, 64, 0.1, 1, p, 4, p, None) == fa.FA_ERR_UNSUPPORTED
    # N_q != N_k entry points: sizes, head dimension, block-mask shape rules
    assert lib.fa_fwd_qk(1, p, p, p, p, p, 1, 1, 0, 128, 64, 0.1, 1, None, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_qk(1, p, p, p, p, p, 1, 1, 128, 0, 64, 0.1, 1, None, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_qk(1, p, p, p, p, p, 1, 1, 128, 256, 80, 0.1, 1, None, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_fwd_qk(1, p, p, p, p, p, 1, 1, 128, 200, 64, 0.1, 0, p, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_fwd_qk(1, None, p, p, p, p, 1, 1, 128, 256, 64, 0.1, 0, None, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_qk(1, p, p, p, p, p, p, p, p, p, _fake(4096 + 16), 1, 1, 128, 256, 64, 0.1, 0, None, None) \
        == fa.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_qk(1, p, p, p, p, p, p, p, p, p, p, 1, 1, 256, 100, 64, 0.1, 1, p, None) \
        == fa.FA_ERR_UNSUPPORTED


def test_trace_sizes(lib):
    assert lib.fa_fwd_trace_size(2, 3, 1000) == 2 * 3 * 4 * (8 + 1)
    assert lib.fa_bwd_row_tile(64) == 128 and lib.fa_bwd_row_tile(128) == 128
    assert lib.fa_bwd_trace_size(2, 3, 1000, 128) == 2 * 3 * 8 * ((8 + 1) + (8 + 1))


def test_splitkv_workspace_layout(lib):
    # partial O fp32 [n][B*H][Nq][d], then partial lse fp32 [n][B*H][Nq] at a 256-byte boundary
    n, B, H, Nq, d = 5, 2, 3, 7, 64
    o_bytes = n * B * H * Nq * d * 4
    lse_off = -(-o_bytes // 256) * 256
    assert lib.fa_fwd_splitkv_workspace_size(B, H, Nq, d, n) == lse_off + -(-(n * B * H * Nq * 4) // 256) * 256
    assert lib.fa_fwd_splitkv_workspace_size(B, H, Nq, 80, n) == 0
    assert lib.fa_fwd_splitkv_workspace_size(B, H, Nq, d, 0) == 0
