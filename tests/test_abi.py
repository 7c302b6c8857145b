"""The C-ABI library loads, exports every symbol include/mxnorm.h declares, and
rejects bad arguments with the documented status before touching the GPU.

No test here launches a kernel: invalid calls return during validation, and
the fault-injection hook fails a call on the host before any CUDA call.
"""
import ctypes
import os
import re

import pytest

from normalisation_row_bf16_b200 import build as nbuild
from normalisation_row_bf16_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    nbuild.build()
    return ops.lib()


def _declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, re.M):
            if m.group(1) not in ("defined",):
                names.append(m.group(1))
    return sorted(set(names))


def test_library_exports_every_declared_symbol(L):
    names = _declared_functions()
    assert "mxnorm_fwd" in names and "mxnorm_bwd" in names and len(names) >= 10
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
        assert n in ops.SIGNATURES, f"{n} has no binding"


def test_scales_bytes(L):
    assert ops.scales_bytes(8192, 4096, ops.SCALES_ROWMAJOR) == 8192 * 128
    assert ops.scales_bytes(100, 4128, ops.SCALES_MMA) == 128 * 132
    assert ops.scales_bytes(0, 64, ops.SCALES_ROWMAJOR) == 0
    assert ops.scales_bytes(4, 33, ops.SCALES_ROWMAJOR) == 0
    assert ops.scales_bytes(4, 64, 7) == 0


FAKE = ctypes.c_void_p(0x10000)          # aligned, never dereferenced on these paths
MISALIGNED = ctypes.c_void_p(0x10008)


def _fwd(L, x=FAKE, q=FAKE, s=FAKE, T=4, D=64, ld=64, p=2.0, rnd=0, layout=0, gamma=None, G=None):
    return L.mxnorm_fwd(x, gamma, q, s, G, T, D, ld, p, rnd, 0, layout, None)


@pytest.mark.parametrize("kw,code", [
    (dict(D=33), ops.MXN_ERR_ARG),
    (dict(D=0), ops.MXN_ERR_ARG),
    (dict(T=-1), ops.MXN_ERR_ARG),
    (dict(ld=60), ops.MXN_ERR_ARG),
    (dict(ld=68), ops.MXN_ERR_ARG),
    (dict(x=None), ops.MXN_ERR_ARG),
    (dict(q=None), ops.MXN_ERR_ARG),
    (dict(s=None), ops.MXN_ERR_ARG),
    (dict(x=MISALIGNED), ops.MXN_ERR_ARG),
    (dict(gamma=MISALIGNED), ops.MXN_ERR_ARG),
    (dict(p=0.0), ops.MXN_ERR_ARG),
    (dict(p=-1.0), ops.MXN_ERR_ARG),
    (dict(p=float("nan")), ops.MXN_ERR_ARG),
    (dict(rnd=2), ops.MXN_ERR_ARG),
    (dict(layout=2), ops.MXN_ERR_ARG),
    (dict(D=32768 + 32, ld=32768 + 32), ops.MXN_ERR_UNSUPPORTED),
])
def test_fwd_argument_errors(L, kw, code):
    assert _fwd(L, **kw) == code
    assert L.mxnorm_last_error().decode() != ""


def test_empty_input_is_a_noop(L):
    assert _fwd(L, T=0) == ops.MXN_OK
    assert L.mxfp8_cast(FAKE, FAKE, FAKE, 0, 64, 64, 0, 0, 0, None) == ops.MXN_OK
    assert L.rmsnorm_bf16(FAKE, None, FAKE, 0, 64, 64, 1e-5, None) == ops.MXN_OK
    assert L.mxnorm_bwd(FAKE, FAKE, None, FAKE, FAKE, None, 0, 64, None, 0, None) == ops.MXN_OK


def test_other_entry_points_validate(L):
    assert L.mxfp8_cast(FAKE, FAKE, FAKE, 4, 48, 48, 0, 0, 0, None) == ops.MXN_ERR_ARG
    assert L.rmsnorm_bf16(FAKE, None, None, 4, 64, 64, 1e-5, None) == ops.MXN_ERR_ARG
    assert L.rmsnorm_bf16(FAKE, None, FAKE, 4, 64, 64, -1.0, None) == ops.MXN_ERR_ARG
    assert L.rmsnorm_then_mxcast(FAKE, None, 1e-5, FAKE, FAKE, FAKE, 4, 64, 64, 5, None) == ops.MXN_ERR_ARG
    # dgamma without gamma, and a row length beyond the backward's limit
    assert L.mxnorm_bwd(FAKE, FAKE, None, FAKE, FAKE, FAKE, 4, 64, FAKE, 1 << 20, None) == ops.MXN_ERR_ARG
    assert L.mxnorm_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, None, 4, 32768, None, 0, None) == ops.MXN_ERR_UNSUPPORTED
    assert L.mxnorm_bwd(FAKE, FAKE, None, MISALIGNED, FAKE, None, 4, 64, None, 0, None) == ops.MXN_ERR_ARG
    assert L.mxnorm_bwd_workspace_size(4, 33) == 0


def test_tuning_validation(L):
    assert L.mxnorm_set_tuning(100, 0, 0) == ops.MXN_ERR_ARG
    assert L.mxnorm_set_tuning(1024, 0, 0) == ops.MXN_ERR_ARG
    assert L.mxnorm_set_tuning(0, 17, 0) == ops.MXN_ERR_ARG
    assert L.mxnorm_set_tuning(0, 0, 9) == ops.MXN_ERR_ARG
    assert L.mxnorm_set_tuning(256, 4, 2) == ops.MXN_OK
    assert L.mxnorm_set_tuning(0, 0, 0) == ops.MXN_OK
    assert L.mxnorm_set_gemm_tiles(3) == ops.MXN_ERR_ARG
    assert L.mxnorm_set_gemm_tiles(2) == ops.MXN_OK
    assert L.mxnorm_set_gemm_tiles(-1) == ops.MXN_ERR_ARG
    assert L.mxnorm_set_gemm_tiles(1) == ops.MXN_OK
    assert L.mxnorm_set_gemm_tiles(0) == ops.MXN_OK


def test_host_fault_injection(L):
    """The hook makes the next calls fail on the host with MXN_ERR_CUDA, after
    argument checks and before any CUDA call; then calls behave again."""
    L.mxnorm_debug_fail_next(2)
    assert _fwd(L) == ops.MXN_ERR_CUDA
    assert "injected" in L.mxnorm_last_error().decode()
    assert L.mxfp8_cast(FAKE, FAKE, FAKE, 4, 64, 64, 0, 0, 0, None) == ops.MXN_ERR_CUDA
    # invalid arguments are still reported as such while injection is armed
    L.mxnorm_debug_fail_next(1)
    assert _fwd(L, D=33) == ops.MXN_ERR_ARG
    L.mxnorm_debug_fail_next(0)
    assert _fwd(L, T=0) == ops.MXN_OK


def test_python_binding_refuses_cpu_tensors(L):
    import torch
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.mxnorm_fwd(x)


def test_gemm_argument_checks(L):
    f = L.mxfp8_gemm
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 256, 128, None) == ops.MXN_OK        # empty
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, -1, 256, 128, None) == ops.MXN_ERR_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 0, None) == ops.MXN_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 100, 256, 128, None) == ops.MXN_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 200, 128, None) == ops.MXN_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 96, None) == ops.MXN_ERR_UNSUPPORTED
    assert f(None, FAKE, FAKE, FAKE, FAKE, 128, 256, 128, None) == ops.MXN_ERR_ARG
    assert f(FAKE, FAKE, MISALIGNED, FAKE, FAKE, 128, 256, 128, None) == ops.MXN_ERR_ARG
    L.mxnorm_debug_fail_next(1)
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 128, None) == ops.MXN_ERR_CUDA


def test_codes_bytes(L):
    assert L.mxnorm_codes_bytes(8192, 4096, 0) == 8192 * 4096
    assert L.mxnorm_codes_bytes(8192, 4096, 1) == 8192 * 2048
    assert L.mxnorm_codes_bytes(3, 96, 1) == 3 * 48
    assert L.mxnorm_codes_bytes(4, 33, 0) == 0
    assert L.mxnorm_codes_bytes(4, 64, 2) == 4 * 32        # NVFP4
    assert L.mxnorm_codes_bytes(4, 64, 3) == 0
    assert L.mxnorm_codes_bytes(-1, 64, 0) == 0


def test_variant_entry_points_validate(L):
    st = None
    fx = L.mxnorm_fwd_ex
    # element format and statistic out of range
    assert fx(FAKE, None, FAKE, FAKE, None, 4, 64, 64, 2.0, 0, 0, 0, 3, 0, st) == ops.MXN_ERR_ARG
    # NVFP4 scales exist only row-major
    assert fx(FAKE, None, FAKE, FAKE, None, 4, 64, 64, 2.0, 0, 0, 1, 2, 0, st) == ops.MXN_ERR_UNSUPPORTED
    assert fx(FAKE, None, FAKE, FAKE, None, 4, 64, 64, 2.0, 0, 0, 0, 0, 3, st) == ops.MXN_ERR_ARG
    # the shared checks still apply
    assert fx(FAKE, None, FAKE, FAKE, None, 4, 33, 64, 2.0, 0, 0, 0, 1, 0, st) == ops.MXN_ERR_ARG
    assert fx(FAKE, None, FAKE, FAKE, None, 4, 64, 64, 0.0, 0, 0, 0, 1, 1, st) == ops.MXN_ERR_ARG
    assert fx(FAKE, None, FAKE, FAKE, None, 0, 64, 64, 2.0, 0, 0, 0, 1, 1, st) == ops.MXN_OK   # empty
    cx = L.mx_cast_ex
    assert cx(FAKE, MISALIGNED, FAKE, FAKE, 4, 64, 64, 0, 0, 0, 0, st) == ops.MXN_ERR_ARG
    assert cx(FAKE, None, FAKE, FAKE, 4, 64, 64, 0, 0, 0, 5, st) == ops.MXN_ERR_ARG
    assert cx(FAKE, None, None, FAKE, 4, 64, 64, 0, 0, 0, 1, st) == ops.MXN_ERR_ARG
    fw = L.mxnorm_fold_weight
    assert fw(FAKE, None, FAKE, FAKE, 4, 64, 64, 0, 1, st) == ops.MXN_ERR_ARG          # nothing to fold
    assert fw(FAKE, FAKE, FAKE, FAKE, 4, 64, 64, 9, 1, st) == ops.MXN_ERR_ARG
    assert fw(FAKE, FAKE, FAKE, FAKE, 4, 64, 64, 0, 3, st) == ops.MXN_ERR_ARG
    assert fw(FAKE, FAKE, FAKE, FAKE, 0, 64, 64, 0, 1, st) == ops.MXN_OK               # empty


def test_python_variant_bindings_refuse_cpu_tensors(L):
    import torch
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.mxnorm_fwd_ex(x, elem="e2m1")
    with pytest.raises(ValueError):
        ops.mx_cast(x)
    with pytest.raises(ValueError):
        ops.fold_weight(x, x[0])


def test_binding_checks_output_buffers(L):
    """Caller-provided outputs must be CUDA tensors of the right type and size
    on the input's device (the C ABI writes through raw pointers)."""
    import torch
    from normalisation_row_bf16_b200.ops import _check_buffer
    cuda0 = torch.device("cuda", 0)
    with pytest.raises(ValueError):
        _check_buffer(torch.empty(10, dtype=torch.uint8), "q", 8, torch.uint8, cuda0)   # a CPU tensor
    with pytest.raises(ValueError):
        _check_buffer([0] * 10, "q", 8, torch.uint8, cuda0)                            # not a tensor
    _check_buffer(None, "q", 8, torch.uint8, cuda0)                                     # allocated by the binding


def test_binding_raises_when_the_library_is_missing(monkeypatch, tmp_path):
    """No fallback: with the library file absent every op raises before doing work."""
    import torch
    monkeypatch.setattr(ops, "_lib", None)
    monkeypatch.setattr(ops._build, "LIB", str(tmp_path / "libmxnorm_b200.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        ops.lib()
    with pytest.raises((RuntimeError, ValueError)):      # refused, never computed on the host
        ops.mxnorm_fwd(torch.zeros(2, 64, dtype=torch.bfloat16))
