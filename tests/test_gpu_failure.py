"""Failure detection on the GPU without a fault: a bounded wait runs out.

A kernel waits on an mbarrier that nothing arrives on, with a 1 ms limit; it
must give up, record MXN_ERR_TIMEOUT in the status word, and leave the context
usable (a normal MXNorm call afterwards still succeeds and the status reads OK).
"""
import ctypes

import pytest
import torch

from normalisation_row_bf16_b200 import build as nbuild
from normalisation_row_bf16_b200 import ops, synthetic

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    nbuild.build()
    L = ops.lib()
    assert ops.device_status() == ops.MXN_OK
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.mxnorm_debug_wait_timeout(ctypes.c_uint64(1_000_000), ctypes.c_void_p(flag.data_ptr()), stream) == 0
    assert ops.device_status() == ops.MXN_ERR_TIMEOUT
    assert int(flag.item()) == 1
    # the status word was cleared by the read, and the context still works
    assert ops.device_status() == ops.MXN_OK
    x = synthetic.activations(64, 1024, "normal", device="cuda")
    q, s, G = ops.mxnorm_fwd(x)
    torch.cuda.synchronize()
    assert torch.isfinite(G).all()
    assert ops.device_status() == ops.MXN_OK
