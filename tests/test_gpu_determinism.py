"""Repeatability of the row kernels under back-to-back launches.

Every launch streams rows through per-group shared-memory stages that a bulk
copy refills as soon as the group hands a stage back.  A stage handed back
before its shared-memory reads have completed can be overwritten by the next
row's copy, which corrupts a few rows at random and only under load.  These
tests launch each kernel many times back to back (outputs rotating over four
buffer sets, inputs over four copies of the same batch, so the launches run at
full rate), then require every launch's outputs to be bit-identical to the
first launch's.  The first launch's values are checked against the oracle by
the parity tests; here only repeatability is at stake.
"""
import pytest
import torch

from normalisation_row_bf16_b200 import build as nbuild
from normalisation_row_bf16_b200 import ops, synthetic

pytestmark = pytest.mark.gpu

T, D = 8192, 4096
N_SETS = 4
ROUNDS = 16          # 64 launches per case


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    nbuild.build()
    ops.lib()
    yield
    assert ops.device_status() == ops.MXN_OK


@pytest.fixture(scope="module")
def batch():
    dev = torch.device("cuda")
    x = synthetic.activations(T, D, "outliers", seed=11, device=dev)
    g = synthetic.gamma(D, seed=11, device=dev)
    return [x] + [x.clone() for _ in range(N_SETS - 1)], g


def _mismatches(outs, ref):
    bad = 0
    for o in outs:
        for a, b in zip(o, ref):
            if a is None:
                continue
            bad += int((a.view(torch.uint8) != b.view(torch.uint8)).sum())
    return bad


def _repeat(launch, outs):
    first = [t.clone() if t is not None else None for t in outs[0]]
    bad = 0
    for _ in range(ROUNDS):
        for i in range(N_SETS):
            launch(i)
        torch.cuda.synchronize()
        bad += _mismatches(outs, first)
    return bad


@pytest.mark.parametrize("fmt,rounding", [("e4m3", "rne"), ("e4m3", "sr"), ("e2m1", "rne"), ("nvfp4", "rne")])
def test_forward_repeats_bit_exactly(batch, fmt, rounding):
    xs, g = batch
    dev = xs[0].device
    cols = D if fmt == "e4m3" else D // 2
    scols = D // 16 if fmt == "nvfp4" else D // 32
    outs = [(torch.empty(T, cols, dtype=torch.uint8, device=dev),
             torch.empty(T, scols, dtype=torch.uint8, device=dev),
             torch.empty(T, dtype=torch.float32, device=dev)) for _ in range(N_SETS)]
    kw = dict(rounding=ops.SR, seed=5) if rounding == "sr" else {}

    def launch(i):
        q, s, G = outs[i]
        if fmt == "e4m3":
            ops.mxnorm_fwd(xs[i], g, 2.0, q=q, scales=s, G=G, **kw)
        else:
            ops.mxnorm_fwd_ex(xs[i], g, 2.0, elem=fmt, q=q, scales=s, G=G, **kw)

    launch(0)
    torch.cuda.synchronize()
    assert _repeat(launch, outs) == 0
    assert ops.device_status() == ops.MXN_OK


def test_backward_repeats_bit_exactly(batch):
    xs, g = batch
    dev = xs[0].device
    dys = [synthetic.upstream_grad(T, D, seed=3, device=dev)] * N_SETS
    G = ops.mxnorm_fwd(xs[0], g, 2.0)[2]
    ws = torch.empty(max(16, ops.bwd_workspace_bytes(T, D)), dtype=torch.uint8, device=dev)
    outs = [(torch.empty(T, D, dtype=torch.bfloat16, device=dev), torch.empty(D, dtype=torch.bfloat16, device=dev))
            for _ in range(N_SETS)]

    def launch(i):
        ops.mxnorm_bwd(xs[i], dys[i], g, G, dx=outs[i][0], dgamma=outs[i][1], workspace=ws)

    launch(0)
    torch.cuda.synchronize()
    assert _repeat(launch, outs) == 0
    assert ops.device_status() == ops.MXN_OK
