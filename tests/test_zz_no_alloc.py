"""The allocation-free backward entry point, mxnorm_bwd_noalloc.

It serves callers that cannot allocate device memory at call time (engines
that own every allocation, real-time loops).  It must give the same dx and
dgamma as mxnorm_bwd with a caller-provided workspace, within the backward's
tolerance, on two calls in a row (the second call reuses the library's
scratch array as the first left it).  This file runs last so that a failure
here leaves every other test already run.
"""
import ctypes

import pytest
import torch

from normalisation_row_bf16_b200 import build as nbuild
from normalisation_row_bf16_b200 import ops, synthetic

from parity_util import BWD_RTOL_L2, rel_l2

pytestmark = pytest.mark.gpu


def _call_noalloc(x, dy, g, G, dx, dg):
    """Straight through the C ABI: no workspace argument exists."""
    L = ops.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = L.mxnorm_bwd_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(dy.data_ptr()),
                              ctypes.c_void_p(g.data_ptr()), ctypes.c_void_p(G.data_ptr()),
                              ctypes.c_void_p(dx.data_ptr()), ctypes.c_void_p(dg.data_ptr()),
                              x.shape[0], x.shape[1], stream)
    assert rc == ops.MXN_OK, L.mxnorm_last_error().decode()


@pytest.mark.parametrize("T,D", [(8192, 4096), (300, 1024), (64, 16384), (1024, 16384)])
def test_noalloc_backward_matches_workspace_backward(T, D):
    """(1024, 16384) plans more partial rows than the scratch's 2^21 / D = 128,
    so the call runs on fewer CTAs than mxnorm_bwd; dx is per row and must be
    bit-identical whatever the CTA count, dgamma's summation order differs."""
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    nbuild.build()
    x = synthetic.activations(T, D, "normal", seed=D, device="cuda")
    g = synthetic.gamma(D, seed=D, device="cuda")
    _, _, G = ops.mxnorm_fwd(x, g, 2.0)
    for call in range(2):
        dy = synthetic.upstream_grad(T, D, seed=D + call, device="cuda")
        dx_ref, dg_ref = ops.mxnorm_bwd(x, dy, g, G)
        dx = torch.full_like(x, float("nan"))
        dg = torch.full((D,), float("nan"), dtype=torch.bfloat16, device="cuda")
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        _call_noalloc(x, dy, g, G, dx, dg)
        torch.cuda.synchronize()
        if call == 1:   # the first call looked up the scratch array; later ones allocate nothing
            assert torch.cuda.mem_get_info()[0] == free_before
        assert torch.equal(dx, dx_ref)
        assert rel_l2(dg.float().cpu().numpy(), dg_ref.float().cpu().numpy()) <= BWD_RTOL_L2
        assert torch.isfinite(dg.float()).all()
    assert ops.device_status() == ops.MXN_OK


def test_noalloc_backward_without_dgamma():
    """dgamma = NULL (no gain gradient wanted): the call touches no scratch and
    dx still equals the workspace backward's."""
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    nbuild.build()
    T, D = 777, 4096
    x = synthetic.activations(T, D, "outliers", seed=3, device="cuda")
    g = synthetic.gamma(D, seed=3, device="cuda")
    dy = synthetic.upstream_grad(T, D, seed=3, device="cuda")
    _, _, G = ops.mxnorm_fwd(x, g, 2.0)
    dx_ref, _ = ops.mxnorm_bwd(x, dy, g, G)
    for _ in range(2):
        dx, dg = ops.mxnorm_bwd_noalloc(x, dy, g, G, want_dgamma=False)
        torch.cuda.synchronize()
        assert dg is None
        assert torch.equal(dx, dx_ref)
    assert ops.device_status() == ops.MXN_OK
