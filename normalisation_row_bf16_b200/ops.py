"""Thin Python binding over the C ABI in include/mxnorm.h (libmxnorm_b200.so).

Argument marshalling only: torch allocates device memory and supplies the
stream; every step of the computation runs in the library's CUDA kernels.
There is no CPU path: calling an op without the built library, or with CPU
tensors, raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

from . import build as _build

RNE, SR = 0, 1
SCALES_ROWMAJOR, SCALES_MMA = 0, 1
ELEM = {"e4m3": 0, "e2m1": 1, "nvfp4": 2}
STAT = {"absmax": 0, "scale_exp": 1}
MXN_OK, MXN_ERR_ARG, MXN_ERR_UNSUPPORTED, MXN_ERR_CUDA, MXN_ERR_TIMEOUT = 0, -1, -2, -3, -4

# Every symbol include/mxnorm.h declares, with its ctypes signature.
_P, _I64, _U64, _F32, _I32, _SZ = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float,
                                   ctypes.c_int, ctypes.c_size_t)
SIGNATURES = {
    "mxnorm_scales_bytes": (_SZ, [_I64, _I64, _I32]),
    "mxnorm_codes_bytes": (_SZ, [_I64, _I64, _I32]),
    "mxnorm_fwd": (_I32, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _F32, _I32, _U64, _I32, _P]),
    "mxnorm_fwd_ex": (_I32, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _F32, _I32, _U64, _I32, _I32, _I32,
                             _P]),
    "mxfp8_cast": (_I32, [_P, _P, _P, _I64, _I64, _I64, _I32, _U64, _I32, _P]),
    "mx_cast_ex": (_I32, [_P, _P, _P, _P, _I64, _I64, _I64, _I32, _U64, _I32, _I32, _P]),
    "mxnorm_fold_weight": (_I32, [_P, _P, _P, _P, _I64, _I64, _I64, _I32, _I32, _P]),
    "rmsnorm_bf16": (_I32, [_P, _P, _P, _I64, _I64, _I64, _F32, _P]),
    "rmsnorm_then_mxcast": (_I32, [_P, _P, _F32, _P, _P, _P, _I64, _I64, _I64, _I32, _P]),
    "mxnorm_bwd": (_I32, [_P, _P, _P, _P, _P, _P, _I64, _I64, _P, _SZ, _P]),
    "mxnorm_bwd_workspace_size": (_SZ, [_I64, _I64]),
    "mxnorm_bwd_noalloc": (_I32, [_P, _P, _P, _P, _P, _P, _I64, _I64, _P]),
    "mxfp8_gemm": (_I32, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "mxnorm_last_error": (ctypes.c_char_p, []),
    "mxnorm_device_status": (_I32, [_P]),
    "mxnorm_set_tuning": (_I32, [_I32, _I32, _I32]),
    "mxnorm_set_gemm_tiles": (_I32, [_I32]),
    "mxnorm_debug_fail_next": (None, [_I32]),
    "mxnorm_debug_wait_timeout": (_I32, [_U64, _P, _P]),
}

_lib = None


class MXNormError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"status {status}: {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_build.LIB):
            raise RuntimeError(f"{_build.LIB} is missing: run `python -m normalisation_row_bf16_b200.build` "
                               "(there is no CPU fallback)")
        L = ctypes.CDLL(_build.LIB)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(rc: int):
    if rc != MXN_OK:
        raise MXNormError(rc, lib().mxnorm_last_error().decode())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _rows_ld(x: torch.Tensor):
    if x.dim() != 2 or x.dtype != torch.bfloat16 or not x.is_cuda:
        raise ValueError("x must be a 2-D bf16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("x rows must be contiguous")
    return x.shape[0], x.shape[1], x.stride(0)


def _bf16_vec(g, D):
    if g is None:
        return None
    if g.dtype != torch.bfloat16 or not g.is_cuda or g.numel() != D or not g.is_contiguous():
        raise ValueError("gamma must be a contiguous bf16 CUDA tensor of D elements")
    return g


def scales_bytes(T: int, D: int, layout: int = SCALES_ROWMAJOR) -> int:
    return int(lib().mxnorm_scales_bytes(T, D, layout))


def _check_buffer(t, name, nbytes, dtype, device):
    """A caller-provided output must hold the bytes the library will write
    (the C ABI takes raw pointers and cannot check)."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor")
    if t.numel() * t.element_size() < nbytes:
        raise ValueError(f"{name} holds {t.numel() * t.element_size()} bytes, {nbytes} needed")


def _alloc_outputs(x, T, D, layout, q, scales, elem: str = "e4m3"):
    q_bytes = T * (D if elem == "e4m3" else D // 2)
    s_bytes = T * (D // 16) if elem == "nvfp4" else scales_bytes(T, D, layout)
    _check_buffer(q, "q", q_bytes, torch.uint8, x.device)
    _check_buffer(scales, "scales", s_bytes, torch.uint8, x.device)
    if q is None:
        q = torch.empty(T, D if elem == "e4m3" else D // 2, dtype=torch.uint8, device=x.device)
    if scales is None and elem == "nvfp4":
        scales = torch.empty(T, D // 16, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = (torch.empty(T, D // 32, dtype=torch.uint8, device=x.device) if layout == SCALES_ROWMAJOR
                  else torch.zeros(max(s_bytes, 1), dtype=torch.uint8, device=x.device))
    return q, scales


def mxnorm_fwd(x, gamma=None, p: float = 2.0, rounding: int = RNE, seed: int = 0,
               scale_layout: int = SCALES_ROWMAJOR, q=None, scales=None, G=None, stream=None):
    """MXNorm forward: returns (q uint8 [T, D] E4M3 codes, scales uint8 E8M0, G fp32 [T])."""
    T, D, ld = _rows_ld(x)
    gamma = _bf16_vec(gamma, D)
    q, scales = _alloc_outputs(x, T, D, scale_layout, q, scales)
    _check_buffer(G, "G", 4 * T, torch.float32, x.device)
    if G is None:
        G = torch.empty(T, dtype=torch.float32, device=x.device)
    _check(lib().mxnorm_fwd(_ptr(x), _ptr(gamma), _ptr(q), _ptr(scales), _ptr(G), T, D, ld,
                            float(p), int(rounding), ctypes.c_uint64(seed & (2**64 - 1)),
                            int(scale_layout), _stream(stream)))
    return q, scales, G


def mxfp8_cast(x, rounding: int = RNE, seed: int = 0, scale_layout: int = SCALES_ROWMAJOR,
               q=None, scales=None, stream=None):
    """MX quantisation of x itself: (q uint8 [T, D], scales uint8)."""
    T, D, ld = _rows_ld(x)
    q, scales = _alloc_outputs(x, T, D, scale_layout, q, scales)
    _check(lib().mxfp8_cast(_ptr(x), _ptr(q), _ptr(scales), T, D, ld, int(rounding),
                            ctypes.c_uint64(seed & (2**64 - 1)), int(scale_layout), _stream(stream)))
    return q, scales


def mxnorm_fwd_ex(x, gamma=None, p: float = 2.0, rounding: int = RNE, seed: int = 0,
                  scale_layout: int = SCALES_ROWMAJOR, elem: str = "e4m3", stat: str = "absmax",
                  q=None, scales=None, G=None, stream=None):
    """MXNorm forward with an element format ("e4m3", or "e2m1": q uint8 [T, D/2],
    two codes per byte) and a block statistic ("absmax", or "scale_exp")."""
    T, D, ld = _rows_ld(x)
    gamma = _bf16_vec(gamma, D)
    q, scales = _alloc_outputs(x, T, D, scale_layout, q, scales, elem)
    _check_buffer(G, "G", 4 * T, torch.float32, x.device)
    if G is None:
        G = torch.empty(T, dtype=torch.float32, device=x.device)
    _check(lib().mxnorm_fwd_ex(_ptr(x), _ptr(gamma), _ptr(q), _ptr(scales), _ptr(G), T, D, ld,
                               float(p), int(rounding), ctypes.c_uint64(seed & (2**64 - 1)),
                               int(scale_layout), ELEM[elem], STAT[stat], _stream(stream)))
    return q, scales, G


def mx_cast(x, gain=None, rounding: int = RNE, seed: int = 0, scale_layout: int = SCALES_ROWMAJOR,
            elem: str = "e4m3", q=None, scales=None, stream=None):
    """MX quantisation of x, or of x * gain along each row: (q, scales)."""
    T, D, ld = _rows_ld(x)
    gain = _bf16_vec(gain, D)
    q, scales = _alloc_outputs(x, T, D, scale_layout, q, scales, elem)
    _check(lib().mx_cast_ex(_ptr(x), _ptr(gain), _ptr(q), _ptr(scales), T, D, ld, int(rounding),
                            ctypes.c_uint64(seed & (2**64 - 1)), int(scale_layout), ELEM[elem],
                            _stream(stream)))
    return q, scales


def fold_weight(w, gamma, elem: str = "e4m3", scale_layout: int = SCALES_MMA, q=None, scales=None,
                stream=None):
    """MXNormLinear folding: MX codes and scales of w[n, k] * gamma[k], w [N, K]
    one output feature per row (the GEMM's B operand)."""
    N, K, ld = _rows_ld(w)
    gamma = _bf16_vec(gamma, K)
    q, scales = _alloc_outputs(w, N, K, scale_layout, q, scales, elem)
    _check(lib().mxnorm_fold_weight(_ptr(w), _ptr(gamma), _ptr(q), _ptr(scales), N, K, ld,
                                    ELEM[elem], int(scale_layout), _stream(stream)))
    return q, scales


def rmsnorm_bf16(x, gamma=None, eps: float = 1e-5, y=None, stream=None):
    T, D, ld = _rows_ld(x)
    gamma = _bf16_vec(gamma, D)
    _check_buffer(y, "y", 2 * T * D, torch.bfloat16, x.device)
    if y is None:
        y = torch.empty(T, D, dtype=torch.bfloat16, device=x.device)
    _check(lib().rmsnorm_bf16(_ptr(x), _ptr(gamma), _ptr(y), T, D, ld, float(eps), _stream(stream)))
    return y


def rmsnorm_then_mxcast(x, gamma=None, eps: float = 1e-5, scale_layout: int = SCALES_ROWMAJOR,
                        y_tmp=None, q=None, scales=None, stream=None):
    """Two-pass comparator: (q, scales, y_tmp)."""
    T, D, ld = _rows_ld(x)
    gamma = _bf16_vec(gamma, D)
    q, scales = _alloc_outputs(x, T, D, scale_layout, q, scales)
    _check_buffer(y_tmp, "y_tmp", 2 * T * D, torch.bfloat16, x.device)
    if y_tmp is None:
        y_tmp = torch.empty(T, D, dtype=torch.bfloat16, device=x.device)
    _check(lib().rmsnorm_then_mxcast(_ptr(x), _ptr(gamma), float(eps), _ptr(y_tmp), _ptr(q),
                                     _ptr(scales), T, D, ld, int(scale_layout), _stream(stream)))
    return q, scales, y_tmp


def bwd_workspace_bytes(T: int, D: int) -> int:
    return int(lib().mxnorm_bwd_workspace_size(T, D))


def mxnorm_bwd(x, dy, gamma, G, dx=None, dgamma=None, workspace=None, want_dgamma: bool = True,
               stream=None):
    """STE backward: returns (dx bf16 [T, D], dgamma bf16 [D] or None)."""
    T, D, ld = _rows_ld(x)
    if ld != D or dy.shape != x.shape or not dy.is_contiguous() or dy.dtype != torch.bfloat16:
        raise ValueError("x and dy must be dense bf16 [T, D]")
    gamma = _bf16_vec(gamma, D)
    _check_buffer(G, "G", 4 * T, torch.float32, x.device)
    _check_buffer(dx, "dx", 2 * T * D, torch.bfloat16, x.device)
    _check_buffer(dgamma, "dgamma", 2 * D, torch.bfloat16, x.device)
    if dx is None:
        dx = torch.empty_like(x)
    if gamma is not None and want_dgamma and dgamma is None:
        dgamma = torch.empty(D, dtype=torch.bfloat16, device=x.device)
    nbytes = 0
    if dgamma is not None:
        nbytes = bwd_workspace_bytes(T, D)
        if workspace is None:
            workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
        _check_buffer(workspace, "workspace", 0, workspace.dtype, x.device)
        nbytes = workspace.numel() * workspace.element_size()
    _check(lib().mxnorm_bwd(_ptr(x), _ptr(dy), _ptr(gamma), _ptr(G), _ptr(dx), _ptr(dgamma), T, D,
                            _ptr(workspace), nbytes, _stream(stream)))
    return dx, dgamma


def mxnorm_bwd_noalloc(x, dy, gamma, G, dx=None, dgamma=None, want_dgamma: bool = True,
                       stream=None):
    """The backward through the entry point that allocates no device memory
    (its dgamma partials live in the library's own scratch array; calls that
    overlap on the GPU race).  Outputs are allocated here only when not given."""
    T, D, ld = _rows_ld(x)
    if ld != D or dy.shape != x.shape or not dy.is_contiguous() or dy.dtype != torch.bfloat16:
        raise ValueError("x and dy must be dense bf16 [T, D]")
    gamma = _bf16_vec(gamma, D)
    _check_buffer(G, "G", 4 * T, torch.float32, x.device)
    _check_buffer(dx, "dx", 2 * T * D, torch.bfloat16, x.device)
    _check_buffer(dgamma, "dgamma", 2 * D, torch.bfloat16, x.device)
    if dx is None:
        dx = torch.empty_like(x)
    if gamma is not None and want_dgamma and dgamma is None:
        dgamma = torch.empty(D, dtype=torch.bfloat16, device=x.device)
    _check(lib().mxnorm_bwd_noalloc(_ptr(x), _ptr(dy), _ptr(gamma), _ptr(G), _ptr(dx), _ptr(dgamma),
                                    T, D, _stream(stream)))
    return dx, dgamma


def mxfp8_gemm(a_q, a_s, b_q, b_s, M: int, N: int, K: int, c=None, stream=None):
    """C bf16 [M, N] = dequant(A) @ dequant(B)^T; scales in the MMA layout."""
    for t in (a_q, a_s, b_q, b_s):
        if not t.is_cuda or t.dtype != torch.uint8:
            raise ValueError("GEMM operands must be uint8 CUDA tensors")
    if a_q.numel() != M * K or b_q.numel() != N * K:
        raise ValueError("code tensors do not match M, N, K")
    _check_buffer(a_s, "a_s", scales_bytes(M, K, SCALES_MMA), torch.uint8, a_q.device)
    _check_buffer(b_s, "b_s", scales_bytes(N, K, SCALES_MMA), torch.uint8, a_q.device)
    _check_buffer(c, "c", 2 * M * N, torch.bfloat16, a_q.device)
    if c is None:
        c = torch.empty(M, N, dtype=torch.bfloat16, device=a_q.device)
    _check(lib().mxfp8_gemm(_ptr(a_q), _ptr(a_s), _ptr(b_q), _ptr(b_s), _ptr(c), M, N, K, _stream(stream)))
    return c


def device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status."""
    return int(lib().mxnorm_device_status(_stream(stream)))


def set_tuning(consumer_threads: int = 0, stages: int = 0, ctas_per_sm: int = 0):
    _check(lib().mxnorm_set_tuning(consumer_threads, stages, ctas_per_sm))


def set_gemm_tiles(mode: int = 0):
    """0 (default): single-CTA 256 x 192 GEMM tiles where M % 256 == 0 and N % 384 == 0, else 128 x 256;
    1: CTA-pair 256 x 256 tiles where M % 256 == 0; 2: single-CTA 128 x 256 tiles."""
    _check(lib().mxnorm_set_gemm_tiles(int(mode)))


def debug_fail_next(count: int):
    lib().mxnorm_debug_fail_next(int(count))


def algorithmic_bytes_fwd(T: int, D: int, gamma: bool = True, G_out: bool = True) -> int:
    """Bytes MXNorm forward must move: read x (2 B/elem), write codes (1 B/elem)
    and scales (1 B per 32), plus gamma (2 B per column) and G (4 B per row)."""
    return T * D * 2 + T * D + T * (D // 32) + (2 * D if gamma else 0) + (4 * T if G_out else 0)


__all__ = [n for n in dir() if not n.startswith("_") and n not in ("ctypes", "math", "os", "torch")]
