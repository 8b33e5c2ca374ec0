"""Python binding of libfa.so, the B200 (sm_100a) exact fused attention library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/fa.h``. PyTorch supplies device
memory and streams. There is no fallback: if ``libfa.so`` is missing or no CUDA
device is present, the calls raise.

Functions keep the C names: :func:`fa_fwd`, :func:`fa_bwd`,
:func:`fa_blocksparse_fwd`, :func:`fa_blocksparse_bwd`, :func:`fa_fwd_qk`,
:func:`fa_bwd_qk` (N_q query rows, N_k key rows), :func:`fa_bwd_workspace_size`,
plus debug entry points for tile traces and the device status word.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(5)
FA_FP16, FA_BF16 = 0, 1

EXPORTED = (
    "fa_status_string", "fa_fwd", "fa_bwd", "fa_blocksparse_fwd", "fa_blocksparse_bwd",
    "fa_bwd_workspace_size", "fa_fwd_trace_size", "fa_bwd_trace_size", "fa_bwd_row_tile",
    "fa_debug_fwd_trace", "fa_debug_bwd_trace", "fa_debug_bwd_phase", "fa_device_status",
    "fa_debug_timeout_probe", "fa_bwd_noalloc", "fa_fwd_qk", "fa_bwd_qk", "fa_debug_fwd_withhold",
    "fa_fwd_splitkv", "fa_fwd_splitkv_workspace_size", "fa_fwd_splitkv_splits", "fa_debug_bwd_withhold",
    "fa_fwd_dropout", "fa_bwd_dropout", "fa_debug_dropout_draws", "fa_fwd_fp8",
)


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfa.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FileNotFoundError(f"{path} is not built; run `python -m io_aware_exact_19_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    fwd_args = [i, vp, vp, vp, vp, vp, i, i, i, i, f, i]
    bwd_args = [i, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i]
    sigs = {
        "fa_status_string": ([i], ctypes.c_char_p),
        "fa_fwd": (fwd_args + [vp], i),
        "fa_blocksparse_fwd": (fwd_args + [vp, vp], i),
        "fa_debug_fwd_trace": (fwd_args + [vp, vp, vp], i),
        "fa_bwd": (bwd_args + [vp], i),
        "fa_blocksparse_bwd": (bwd_args + [vp, vp], i),
        "fa_debug_bwd_trace": (bwd_args + [vp, vp, vp], i),
        "fa_debug_bwd_phase": ([i] + bwd_args + [vp, vp], i),
        "fa_bwd_workspace_size": ([i, i, i, i], sz),
        "fa_fwd_trace_size": ([i, i, i], sz),
        "fa_bwd_trace_size": ([i, i, i, i], sz),
        "fa_bwd_row_tile": ([i], i),
        "fa_device_status": ([vp], i),
        "fa_debug_timeout_probe": ([i, vp], i),
        "fa_debug_fwd_withhold": (fwd_args + [i, vp], i),
        "fa_debug_bwd_withhold": (bwd_args + [i, vp], i),
        "fa_bwd_noalloc": (bwd_args[:10] + bwd_args[11:] + [vp], i),
        # N_q, N_k in place of N
        "fa_fwd_qk": (fwd_args[:8] + [i] + fwd_args[8:] + [vp, vp], i),
        "fa_bwd_qk": (bwd_args[:13] + [i] + bwd_args[13:] + [vp, vp], i),
        "fa_fwd_splitkv": (fwd_args[:8] + [i] + fwd_args[8:] + [vp, i, vp, vp], i),
        "fa_fwd_splitkv_workspace_size": ([i, i, i, i, i], sz),
        "fa_fwd_splitkv_splits": ([i, i, i, i], i),
        "fa_fwd_dropout": (fwd_args[:8] + [i] + fwd_args[8:] + [vp, f, ctypes.c_ulonglong, vp], i),
        "fa_bwd_dropout": (bwd_args[:13] + [i] + bwd_args[13:] + [vp, f, ctypes.c_ulonglong, vp], i),
        "fa_debug_dropout_draws": ([i, i, i, i, ctypes.c_ulonglong, vp, vp, vp], i),
        "fa_fwd_fp8": ([vp, vp, vp, f, f, f, vp, vp, i, i, i, i, i, f, i, vp, vp], i),
    }
    for name, (argtypes, restype) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = argtypes
        fn.restype = restype
    _lib = lib
    return lib


def status_string(status: int) -> str:
    try:
        return load_library().fa_status_string(int(status)).decode()
    except FileNotFoundError:
        return f"status {status}"


def _check(status: int, where: str) -> None:
    if status != FA_OK:
        raise FAError(status, where)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float16:
        return FA_FP16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float16 or bfloat16")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _shape(q):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(int(x) for x in q.shape)


def _check_tensors(ref, *ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")


def _scale(scale, d):
    return float(scale) if scale is not None else 1.0 / (d ** 0.5)


def fa_fwd(q, k, v, o, lse, causal: bool = False, scale: float | None = None, stream=None) -> None:
    """Forward: writes ``o`` [B,H,N,d] and ``lse`` [B,H,N] fp32 (see include/fa.h)."""
    B, H, N, d = _shape(q)
    _check_tensors(q, k, v, o, lse)
    st = load_library().fa_fwd(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                               _scale(scale, d), int(bool(causal)), _stream(stream))
    _check(st, "fa_fwd")


def fa_blocksparse_fwd(q, k, v, o, lse, block_mask, causal: bool = False, scale: float | None = None,
                       stream=None) -> None:
    """Block-sparse forward; ``block_mask`` is a uint8 CUDA tensor [N/128, N/128]."""
    B, H, N, d = _shape(q)
    _check_tensors(q, k, v, o, lse, block_mask)
    st = load_library().fa_blocksparse_fwd(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H,
                                           N, d, _scale(scale, d), int(bool(causal)), _ptr(block_mask),
                                           _stream(stream))
    _check(st, "fa_blocksparse_fwd")


def fa_bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().fa_bwd_workspace_size(B, H, N, d))


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, causal: bool = False, scale: float | None = None,
           stream=None) -> None:
    """Backward: writes ``dq``, ``dk``, ``dv``; ``workspace`` is a CUDA uint8 tensor of
    at least :func:`fa_bwd_workspace_size` bytes."""
    B, H, N, d = _shape(q)
    _check_tensors(q, k, v, o, lse, dout, dq, dk, dv, workspace)
    st = load_library().fa_bwd(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                               _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), B, H, N, d, _scale(scale, d),
                               int(bool(causal)), _stream(stream))
    _check(st, "fa_bwd")


def fa_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, causal: bool = False, scale: float | None = None,
                   stream=None) -> None:
    """Backward without a workspace argument, for callers that cannot allocate device
    memory: the scratch lives in a fixed static device array inside the library (see
    include/fa.h for the size limit and the rule that overlapping calls race)."""
    B, H, N, d = _shape(q)
    _check_tensors(q, k, v, o, lse, dout, dq, dk, dv)
    st = load_library().fa_bwd_noalloc(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                       _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, _scale(scale, d),
                                       int(bool(causal)), _stream(stream))
    _check(st, "fa_bwd_noalloc")


def fa_blocksparse_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, block_mask, causal: bool = False,
                       scale: float | None = None, stream=None) -> None:
    B, H, N, d = _shape(q)
    _check_tensors(q, k, v, o, lse, dout, dq, dk, dv, workspace, block_mask)
    st = load_library().fa_blocksparse_bwd(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                           _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), B, H, N, d,
                                           _scale(scale, d), int(bool(causal)), _ptr(block_mask),
                                           _stream(stream))
    _check(st, "fa_blocksparse_bwd")


def fa_fwd_trace_size(B: int, H: int, N: int) -> int:
    return int(load_library().fa_fwd_trace_size(B, H, N))


def fa_bwd_trace_size(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().fa_bwd_trace_size(B, H, N, d))


def fa_bwd_row_tile(d: int) -> int:
    return int(load_library().fa_bwd_row_tile(d))


def fa_debug_fwd_trace(q, k, v, o, lse, trace, causal: bool = False, block_mask=None, scale=None,
                       stream=None) -> None:
    B, H, N, d = _shape(q)
    st = load_library().fa_debug_fwd_trace(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H,
                                           N, d, _scale(scale, d), int(bool(causal)), _ptr(block_mask),
                                           _ptr(trace), _stream(stream))
    _check(st, "fa_debug_fwd_trace")


def fa_debug_bwd_trace(q, k, v, o, lse, dout, dq, dk, dv, workspace, trace, causal: bool = False,
                       block_mask=None, scale=None, stream=None) -> None:
    B, H, N, d = _shape(q)
    st = load_library().fa_debug_bwd_trace(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                           _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), B, H, N, d,
                                           _scale(scale, d), int(bool(causal)), _ptr(block_mask), _ptr(trace),
                                           _stream(stream))
    _check(st, "fa_debug_bwd_trace")


def fa_debug_bwd_phase(phase: int, q, k, v, o, lse, dout, dq, dk, dv, workspace, causal: bool = False,
                       block_mask=None, scale=None, stream=None) -> None:
    """One of the backward's two launches (0 prep, 1 main); see include/fa.h."""
    B, H, N, d = _shape(q)
    st = load_library().fa_debug_bwd_phase(int(phase), _dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                           _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                           B, H, N, d, _scale(scale, d), int(bool(causal)), _ptr(block_mask),
                                           _stream(stream))
    _check(st, "fa_debug_bwd_phase")


def fa_device_status(stream=None) -> int:
    """Synchronise the stream, return and clear the device status word."""
    return int(load_library().fa_device_status(_stream(stream)))


def fa_debug_fwd_withhold(q, k, v, o, lse, timeout_ms: int, causal: bool = False, scale=None, stream=None) -> None:
    """The forward kernel with a producer that issues no load: its waits run out after
    ``timeout_ms`` and record FA_ERR_TIMEOUT (see include/fa.h)."""
    B, H, N, d = _shape(q)
    st = load_library().fa_debug_fwd_withhold(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H,
                                              N, d, _scale(scale, d), int(bool(causal)), int(timeout_ms),
                                              _stream(stream))
    _check(st, "fa_debug_fwd_withhold")


def fa_debug_bwd_withhold(q, k, v, o, lse, dout, dq, dk, dv, workspace, timeout_ms: int, causal: bool = False,
                          scale=None, stream=None) -> None:
    """The backward with main-kernel producers that issue no load: the waits run out
    after ``timeout_ms`` and record FA_ERR_TIMEOUT (see include/fa.h)."""
    B, H, N, d = _shape(q)
    st = load_library().fa_debug_bwd_withhold(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                              _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), B, H, N, d,
                                              _scale(scale, d), int(bool(causal)), int(timeout_ms), _stream(stream))
    _check(st, "fa_debug_bwd_withhold")


def fa_debug_timeout_probe(timeout_ms: int, stream=None) -> None:
    _check(load_library().fa_debug_timeout_probe(int(timeout_ms), _stream(stream)), "fa_debug_timeout_probe")


# ----------------------------------------------------------------------------- conveniences

def fa_fwd_qk(q, k, v, o, lse, causal: bool = False, block_mask=None, scale: float | None = None,
              stream=None) -> None:
    """Forward with q, o [B, H, N_q, d] and k, v [B, H, N_k, d]; the causal mask is
    bottom-right aligned (query i sees key j <= i + N_k - N_q)."""
    B, H, Nq, d = _shape(q)
    Nk = _shape(k)[2]
    _check_tensors(q, k, v, o, lse, block_mask)
    st = load_library().fa_fwd_qk(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, d,
                                  _scale(scale, d), int(bool(causal)),
                                  _ptr(block_mask) if block_mask is not None else None, _stream(stream))
    _check(st, "fa_fwd_qk")


def fa_bwd_qk(q, k, v, o, lse, dout, dq, dk, dv, workspace, causal: bool = False, block_mask=None,
              scale: float | None = None, stream=None) -> None:
    """Backward of :func:`fa_fwd_qk`; ``workspace`` holds at least
    ``fa_bwd_workspace_size(B, H, N_q, d)`` bytes."""
    B, H, Nq, d = _shape(q)
    Nk = _shape(k)[2]
    _check_tensors(q, k, v, o, lse, dout, dq, dk, dv, workspace, block_mask)
    st = load_library().fa_bwd_qk(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                  _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), B, H, Nq, Nk, d,
                                  _scale(scale, d), int(bool(causal)),
                                  _ptr(block_mask) if block_mask is not None else None, _stream(stream))
    _check(st, "fa_bwd_qk")


def fa_fwd_splitkv_workspace_size(B: int, H: int, Nq: int, d: int, n_splits: int) -> int:
    return int(load_library().fa_fwd_splitkv_workspace_size(B, H, Nq, d, n_splits))


def fa_fwd_splitkv_splits(B: int, H: int, Nq: int, Nk: int) -> int:
    return int(load_library().fa_fwd_splitkv_splits(B, H, Nq, Nk))


def fa_fwd_splitkv(q, k, v, o, lse, n_splits: int, workspace, causal: bool = False, block_mask=None,
                   scale: float | None = None, stream=None) -> None:
    """Split-KV forward: ``n_splits`` key ranges computed apart, then merged; the
    partials stay in ``workspace`` (see include/fa.h for its layout)."""
    B, H, Nq, d = _shape(q)
    Nk = _shape(k)[2]
    _check_tensors(q, k, v, o, lse, workspace, block_mask)
    st = load_library().fa_fwd_splitkv(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk,
                                       d, _scale(scale, d), int(bool(causal)),
                                       _ptr(block_mask) if block_mask is not None else None, int(n_splits),
                                       _ptr(workspace), _stream(stream))
    _check(st, "fa_fwd_splitkv")


def fa_fwd_dropout(q, k, v, o, lse, p_drop: float, seed: int, causal: bool = False, block_mask=None,
                   scale: float | None = None, stream=None) -> None:
    """Forward with dropout on P (keep decisions from Philox4x32-10; see include/fa.h)."""
    B, H, Nq, d = _shape(q)
    Nk = _shape(k)[2]
    _check_tensors(q, k, v, o, lse, block_mask)
    st = load_library().fa_fwd_dropout(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk,
                                       d, _scale(scale, d), int(bool(causal)),
                                       _ptr(block_mask) if block_mask is not None else None, float(p_drop),
                                       ctypes.c_ulonglong(int(seed)), _stream(stream))
    _check(st, "fa_fwd_dropout")


def fa_bwd_dropout(q, k, v, o, lse, dout, dq, dk, dv, workspace, p_drop: float, seed: int, causal: bool = False,
                   block_mask=None, scale: float | None = None, stream=None) -> None:
    """Backward of :func:`fa_fwd_dropout` (same p_drop and seed)."""
    B, H, Nq, d = _shape(q)
    Nk = _shape(k)[2]
    _check_tensors(q, k, v, o, lse, dout, dq, dk, dv, workspace, block_mask)
    st = load_library().fa_bwd_dropout(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                       _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), B, H, Nq, Nk, d,
                                       _scale(scale, d), int(bool(causal)),
                                       _ptr(block_mask) if block_mask is not None else None, float(p_drop),
                                       ctypes.c_ulonglong(int(seed)), _stream(stream))
    _check(st, "fa_bwd_dropout")


def fa_fwd_fp8(q8, k8, v8, q_scale: float, k_scale: float, v_scale: float, o, lse, causal: bool = False,
               block_mask=None, scale: float | None = None, stream=None) -> None:
    """8-bit forward: ``q8``, ``k8``, ``v8`` are uint8 CUDA tensors of e4m3 values
    [B, H, N, 128] with per-tensor scales; ``o`` is bf16 (see include/fa.h)."""
    B, H, Nq, d = _shape(q8)
    Nk = _shape(k8)[2]
    _check_tensors(q8, k8, v8, o, lse, block_mask)
    st = load_library().fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), float(q_scale), float(k_scale), float(v_scale),
                                   _ptr(o), _ptr(lse), B, H, Nq, Nk, d, _scale(scale, d), int(bool(causal)),
                                   _ptr(block_mask) if block_mask is not None else None, _stream(stream))
    _check(st, "fa_fwd_fp8")


def fa_debug_dropout_draws(B: int, H: int, Nq: int, Nk: int, seed: int, row_major, col_major, stream=None) -> None:
    """The dropout draws through both device generator paths (uint8 [B*H, Nq, Nk] each)."""
    st = load_library().fa_debug_dropout_draws(B, H, Nq, Nk, ctypes.c_ulonglong(int(seed)), _ptr(row_major),
                                               _ptr(col_major), _stream(stream))
    _check(st, "fa_debug_dropout_draws")


def attention_forward(q, k, v, causal: bool = False, block_mask=None, scale=None, stream=None):
    """Allocate O and lse with torch and run the forward; returns (o, lse)."""
    import torch
    B, H, N, d = _shape(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if block_mask is None:
        fa_fwd(q, k, v, o, lse, causal, scale, stream)
    else:
        fa_blocksparse_fwd(q, k, v, o, lse, block_mask, causal, scale, stream)
    return o, lse


def attention_backward(q, k, v, o, lse, dout, causal: bool = False, block_mask=None, scale=None,
                       workspace=None, stream=None):
    """Allocate dQ, dK, dV (and the workspace if none is given) and run the backward."""
    import torch
    B, H, N, d = _shape(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if workspace is None:
        workspace = torch.empty(fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=q.device)
    if block_mask is None:
        fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, causal, scale, stream)
    else:
        fa_blocksparse_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, block_mask, causal, scale, stream)
    return dq, dk, dv
