"""CPU oracle for MXNorm -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  It shares no
code with the CUDA library ``normalisation_row_bf16_b200`` and never imports it.

The arithmetic lives in ``mxnorm_oracle.c`` (plain C, fp64 / long-double
statistics, exact E4M3 / E2M1 / E8M0 rounding); this module compiles it with gcc on
first use and marshals numpy arrays.  Every function names the passage it
follows in the C source.

Pins: every function here is checked by ``tests/test_oracle_pins.py`` against
something other than itself (a brute-force grid search, torch's float8 casts,
closed forms, scipy's power mean, quadrature of Theorem 1, Philox known-answer
values, finite differences).  Nothing is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mxnorm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmxnorm_oracle.so")
_CFLAGS = ["-O2", "-std=gnu11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-fexcess-precision=standard", "-Wall"]
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile mxnorm_oracle.c into libmxnorm_oracle.so (gcc)."""
    with _lock:
        stale = (not os.path.exists(_LIB_PATH)
                 or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
        if force or stale:
            tmp = _LIB_PATH + f".tmp{os.getpid()}"
            subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
            os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i64, f64, f32, i32, u64 = (ctypes.c_int64, ctypes.c_double, ctypes.c_float,
                                   ctypes.c_int, ctypes.c_uint64)
        lib.oracle_e4m3_rne_many.argtypes = [P, i64, P]
        lib.oracle_e4m3_sr_many.argtypes = [P, P, i64, P]
        lib.oracle_e8m0_exponent_many.argtypes = [P, i64, P]
        lib.oracle_e2m1_rne_many.argtypes = [P, i64, P]
        lib.oracle_e2m1_sr_many.argtypes = [P, P, i64, P]
        lib.oracle_mx_exponent_many.argtypes = [P, i64, f64, P]
        lib.oracle_nvfp4_scale_code_many.argtypes = [P, i64, P]
        lib.oracle_e2m1_value.argtypes = [i32]
        lib.oracle_e2m1_value.restype = f64
        lib.oracle_sr_words.argtypes = [u64, P, i64, P]
        lib.oracle_philox4x32_10.argtypes = [P, P, P]
        lib.oracle_pmean.argtypes = [P, i64, f64]
        lib.oracle_pmean.restype = f64
        lib.oracle_e4m3_value.argtypes = [i32]
        lib.oracle_e4m3_value.restype = f64
        lib.oracle_mxnorm_fwd.argtypes = [P, i64, P, i64, P, i64, f64, P, P, P, P, i32, u64, i32]
        lib.oracle_mxfp8_cast.argtypes = [P, i64, i64, P, i64, P, P, i32, u64, i32]
        lib.oracle_mxnorm_fwd_ex.argtypes = [P, i64, P, i64, P, i64, f64, P, P, P, P, i32, u64,
                                             i32, i32, i32]
        lib.oracle_mx_cast_ex.argtypes = [P, i64, P, i64, P, i64, P, P, i32, u64, i32, i32]
        lib.oracle_rmsnorm.argtypes = [P, i64, P, i64, P, i64, f32, P, i32]
        lib.oracle_mxnorm_bwd.argtypes = [P, P, P, P, i64, P, i64, i32, P, P]
        lib.oracle_mxfp8_gemm_entries.argtypes = [P, P, P, P, i64, i64, i64, i64, P, P, P, i32]
        for name in ("oracle_mxnorm_fwd", "oracle_mxfp8_cast", "oracle_rmsnorm",
                     "oracle_mxnorm_fwd_ex", "oracle_mx_cast_ex",
                     "oracle_mxnorm_bwd", "oracle_mxfp8_gemm_entries"):
            getattr(lib, name).restype = i32
        lib.oracle_num_threads.restype = i32
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(x):
    """bf16 data (torch bfloat16 tensor on the CPU, or uint16 numpy) -> uint16 numpy."""
    if x is None:
        return None
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        x = x.detach().cpu().contiguous().view(dtype=__import__("torch").int16).numpy()
    return np.ascontiguousarray(np.asarray(x).view(np.uint16))


def _u8(x):
    if hasattr(x, "detach"):
        x = x.detach().cpu().contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x).view(np.uint8))


def _rows(rows, T):
    if rows is None:
        return None, T
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    if r.size and (r.min() < 0 or r.max() >= T):
        raise IndexError("row index out of range")
    return r, int(r.size)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


# ------------------------------------------------------------------ elements

def e4m3_rne(v) -> np.ndarray:
    """fp32 -> E4M3 code, nearest-even, saturating finite (FP8 formats paper)."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32))
    out = np.empty(v.shape, np.uint8)
    _load().oracle_e4m3_rne_many(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_sr(v, r32) -> np.ndarray:
    """fp32 -> E4M3 code by stochastic rounding with the given 32-bit words."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32))
    r = np.ascontiguousarray(np.asarray(r32, dtype=np.uint32))
    assert r.shape == v.shape
    out = np.empty(v.shape, np.uint8)
    _load().oracle_e4m3_sr_many(_ptr(v), _ptr(r), v.size, _ptr(out))
    return out


def e4m3_value(code: int) -> float:
    return float(_load().oracle_e4m3_value(int(code)))


def e8m0_exponent(a) -> np.ndarray:
    """Smallest e in [-127, 127] with |a| <= 448 * 2^e (128 for NaN / inf)."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    out = np.empty(a.shape, np.int32)
    _load().oracle_e8m0_exponent_many(_ptr(a), a.size, _ptr(out))
    return out


def e2m1_rne(v) -> np.ndarray:
    """fp32 -> E2M1 4-bit code (sign in bit 3), nearest-even, saturating to 6."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32))
    out = np.empty(v.shape, np.uint8)
    _load().oracle_e2m1_rne_many(_ptr(v), v.size, _ptr(out))
    return out


def e2m1_sr(v, r32) -> np.ndarray:
    """fp32 -> E2M1 code by stochastic rounding with the given 32-bit words."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32))
    r = np.ascontiguousarray(np.asarray(r32, dtype=np.uint32))
    assert r.shape == v.shape
    out = np.empty(v.shape, np.uint8)
    _load().oracle_e2m1_sr_many(_ptr(v), _ptr(r), v.size, _ptr(out))
    return out


def e2m1_value(code: int) -> float:
    return float(_load().oracle_e2m1_value(int(code)))


def mx_exponent(a, elem_max: float) -> np.ndarray:
    """Smallest e in [-127, 127] with |a| <= elem_max * 2^e (128 for NaN / inf)."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    out = np.empty(a.shape, np.int32)
    _load().oracle_mx_exponent_many(_ptr(a), a.size, float(elem_max), _ptr(out))
    return out


FMT = {"e4m3": 0, "e2m1": 1, "nvfp4": 2}
BLOCK = {"e4m3": 32, "e2m1": 32, "nvfp4": 16}


def nvfp4_scale_code(a) -> np.ndarray:
    """E4M3 code of the smallest E4M3 value s with |a| <= 6 s (NVFP4 block scale)."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    out = np.empty(a.shape, np.int32)
    _load().oracle_nvfp4_scale_code_many(_ptr(a), a.size, _ptr(out))
    return out
STAT = {"absmax": 0, "scale_exp": 1}


def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32).reshape(4))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32).reshape(2))
    out = np.empty(4, np.uint32)
    _load().oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def sr_words(seed: int, idx) -> np.ndarray:
    """The 32-bit word element idx (= row * D + col) draws under this seed."""
    i = np.ascontiguousarray(np.asarray(idx, dtype=np.uint64))
    out = np.empty(i.shape, np.uint32)
    _load().oracle_sr_words(ctypes.c_uint64(seed), _ptr(i), i.size, _ptr(out))
    return out


def pmean(m, p: float) -> float:
    """((1/K) sum m_k^p)^(1/p) in long double; p = inf gives the max."""
    m = np.ascontiguousarray(np.asarray(m, dtype=np.float64))
    return float(_load().oracle_pmean(_ptr(m), m.size, float(p)))


# ------------------------------------------------------------------- rows

def mxnorm_fwd(x, gamma=None, p: float = 2.0, rows=None, G_in=None, rounding: int = 0,
               seed: int = 0, nthreads: int = 0):
    """MXNorm forward on the selected rows of x [T, D] (bf16).

    Returns (q uint8 [n, D], scales uint8 [n, D/32], G float32 [n]).  When G_in
    is given, the codes and scales are derived from those G values (the
    returned G is still the oracle's own)."""
    xu = _u16(x)
    T, D = xu.shape
    g = _u16(gamma)
    r, n = _rows(rows, T)
    Gi = None if G_in is None else np.ascontiguousarray(np.asarray(G_in, np.float32).reshape(n))
    q = np.empty((n, D), np.uint8)
    s = np.empty((n, D // 32), np.uint8)
    G = np.empty(n, np.float32)
    rc = _load().oracle_mxnorm_fwd(_ptr(xu), D, _ptr(g), n, _ptr(r), D, float(p), _ptr(Gi),
                                   _ptr(q), _ptr(s), _ptr(G), int(rounding),
                                   ctypes.c_uint64(seed), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_mxnorm_fwd: bad arguments")
    return q, s, G


def mxnorm_fwd_ex(x, gamma=None, p: float = 2.0, rows=None, G_in=None, rounding: int = 0,
                  seed: int = 0, stat: str = "absmax", fmt: str = "e4m3", nthreads: int = 0):
    """MXNorm forward with a choice of block statistic ("absmax", or "scale_exp":
    the block's scale) and element format ("e4m3"; "e2m1" with two codes per
    byte, q uint8 [n, D/2]; "nvfp4": E2M1 codes with one E4M3 scale per 16,
    scales uint8 [n, D/16]).  Returns (q, scales, G)."""
    xu = _u16(x)
    T, D = xu.shape
    g = _u16(gamma)
    r, n = _rows(rows, T)
    Gi = None if G_in is None else np.ascontiguousarray(np.asarray(G_in, np.float32).reshape(n))
    q = np.empty((n, D if fmt == "e4m3" else D // 2), np.uint8)
    s = np.empty((n, D // BLOCK[fmt]), np.uint8)
    G = np.empty(n, np.float32)
    rc = _load().oracle_mxnorm_fwd_ex(_ptr(xu), D, _ptr(g), n, _ptr(r), D, float(p), _ptr(Gi),
                                      _ptr(q), _ptr(s), _ptr(G), int(rounding),
                                      ctypes.c_uint64(seed), STAT[stat], FMT[fmt], int(nthreads))
    if rc != 0:
        raise ValueError("oracle_mxnorm_fwd_ex: bad arguments")
    return q, s, G


def mx_cast(x, gamma=None, rows=None, rounding: int = 0, seed: int = 0, fmt: str = "e4m3",
            nthreads: int = 0):
    """MX quantisation of x, or of fl32(x * gamma) along each row (the folded
    MXNormLinear weight): (q uint8 [n, D] or [n, D/2], scales uint8 [n, D/32])."""
    xu = _u16(x)
    T, D = xu.shape
    g = _u16(gamma)
    r, n = _rows(rows, T)
    q = np.empty((n, D if fmt == "e4m3" else D // 2), np.uint8)
    s = np.empty((n, D // BLOCK[fmt]), np.uint8)
    rc = _load().oracle_mx_cast_ex(_ptr(xu), D, _ptr(g), n, _ptr(r), D, _ptr(q), _ptr(s),
                                   int(rounding), ctypes.c_uint64(seed), FMT[fmt], int(nthreads))
    if rc != 0:
        raise ValueError("oracle_mx_cast_ex: bad arguments")
    return q, s


def mxfp8_cast(x, rows=None, rounding: int = 0, seed: int = 0, nthreads: int = 0):
    """MX quantisation of x itself: (q uint8 [n, D], scales uint8 [n, D/32])."""
    xu = _u16(x)
    T, D = xu.shape
    r, n = _rows(rows, T)
    q = np.empty((n, D), np.uint8)
    s = np.empty((n, D // 32), np.uint8)
    rc = _load().oracle_mxfp8_cast(_ptr(xu), D, n, _ptr(r), D, _ptr(q), _ptr(s), int(rounding),
                                   ctypes.c_uint64(seed), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_mxfp8_cast: bad arguments")
    return q, s


def rmsnorm(x, gamma=None, eps: float = 1e-5, rows=None, nthreads: int = 0) -> np.ndarray:
    """bf16 RMSNorm (double math, one rounding): uint16 bf16 bits [n, D]."""
    xu = _u16(x)
    T, D = xu.shape
    g = _u16(gamma)
    r, n = _rows(rows, T)
    y = np.empty((n, D), np.uint16)
    rc = _load().oracle_rmsnorm(_ptr(xu), D, _ptr(g), n, _ptr(r), D, float(eps), _ptr(y),
                                int(nthreads))
    if rc != 0:
        raise ValueError("oracle_rmsnorm: bad arguments")
    return y


def mxnorm_bwd(x, dy, gamma, G, rows=None, true_rms: bool = False):
    """STE backward: (dx float64 [n, D], dgamma float64 [D] over the selected rows)."""
    xu, du, g = _u16(x), _u16(dy), _u16(gamma)
    T, D = xu.shape
    r, n = _rows(rows, T)
    Gv = np.ascontiguousarray(np.asarray(G, np.float32).reshape(n))
    dx = np.empty((n, D), np.float64)
    dg = np.empty(D, np.float64)
    rc = _load().oracle_mxnorm_bwd(_ptr(xu), _ptr(du), _ptr(g), _ptr(Gv), n, _ptr(r), D,
                                   int(bool(true_rms)), _ptr(dx), _ptr(dg))
    if rc != 0:
        raise ValueError("oracle_mxnorm_bwd: bad arguments")
    return dx, dg


def mxfp8_gemm_entries(aq, a_s, bq, b_s, ii, jj, nthreads: int = 0) -> np.ndarray:
    """Entries C[ii[t], jj[t]] of dequant(A) @ dequant(B)^T in double."""
    aq, a_s, bq, b_s = _u8(aq), _u8(a_s), _u8(bq), _u8(b_s)
    M, K = aq.shape
    N = bq.shape[0]
    i = np.ascontiguousarray(np.asarray(ii, np.int64))
    j = np.ascontiguousarray(np.asarray(jj, np.int64))
    c = np.empty(i.shape, np.float64)
    rc = _load().oracle_mxfp8_gemm_entries(_ptr(aq), _ptr(a_s), _ptr(bq), _ptr(b_s), M, N, K,
                                           i.size, _ptr(i), _ptr(j), _ptr(c), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_mxfp8_gemm_entries: bad arguments")
    return c
