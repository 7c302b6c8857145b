"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Every call goes through normalisation_row_bf16_b200.ops (ctypes over
libmxnorm_b200.so).  Inputs come from the seeded generators; the oracle sees
the same bf16 bits.  Tolerances are listed in parity_util.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from normalisation_row_bf16_b200 import build as nbuild
from normalisation_row_bf16_b200 import ops, synthetic

from parity_util import (BWD_RTOL_L2, bf16_ulp_distance, check_bwd_elementwise, check_cast,
                         check_mxnorm_fwd, mma_scale_offset, rel_l2, round_bf16, to_np_u8)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    nbuild.build()
    ops.lib()
    yield
    assert ops.device_status() == ops.MXN_OK


def _dev(t):
    return t.to("cuda")


# ------------------------------------------------------------------ forward

@pytest.mark.parametrize("p", [2.0, 1.0, 4.0, math.inf, 3.3])
@pytest.mark.parametrize("with_gamma", [True, False])
def test_mxnorm_fwd_tiny(p, with_gamma):
    x = synthetic.activations(256, 1024, "normal", seed=0)
    g = synthetic.gamma(1024, seed=0) if with_gamma else None
    xd, gd = _dev(x), (None if g is None else _dev(g))
    q, s, G = ops.mxnorm_fwd(xd, gd, p)
    torch.cuda.synchronize()
    rep = check_mxnorm_fwd(xd, gd, p, 0, 0, q, s, G)
    print(rep)


@pytest.mark.parametrize("T,D", [(1, 32), (3, 96), (5, 160), (257, 1056), (2, 4096), (33, 2080),
                                 (7, 8192), (3, 16384), (2, 32768), (130, 544), (64, 64)])
@pytest.mark.parametrize("kind", ["normal", "student_t"])
def test_mxnorm_fwd_ragged(T, D, kind):
    x = synthetic.activations(T, D, kind, seed=T + D)
    g = synthetic.gamma(D, seed=D)
    xd, gd = _dev(x), _dev(g)
    for p in (2.0, 1.0):
        q, s, G = ops.mxnorm_fwd(xd, gd, p)
        torch.cuda.synchronize()
        check_mxnorm_fwd(xd, gd, p, 0, 0, q, s, G)


def test_mxnorm_fwd_strided_rows():
    T, D, ld = 100, 1024, 1536
    base = synthetic.activations(T, ld, "outliers", seed=5)
    xd = _dev(base)[:, :D]
    assert xd.stride(0) == ld
    g = _dev(synthetic.gamma(D, seed=5))
    q, s, G = ops.mxnorm_fwd(xd, g, 2.0)
    torch.cuda.synchronize()
    check_mxnorm_fwd(xd.contiguous(), g, 2.0, 0, 0, q, s, G)


@pytest.mark.parametrize("p", [2.0, 1.0, math.inf])
def test_mxnorm_fwd_sr_bit_exact(p):
    x = synthetic.activations(300, 2048, "student_t", seed=3)
    g = synthetic.gamma(2048, seed=3)
    xd, gd = _dev(x), _dev(g)
    for seed in (0, 0x1234_5678_9ABC_DEF0):
        q, s, G = ops.mxnorm_fwd(xd, gd, p, rounding=ops.SR, seed=seed)
        torch.cuda.synchronize()
        check_mxnorm_fwd(xd, gd, p, 1, seed, q, s, G)


@pytest.mark.parametrize("T,D", [(1, 32), (3, 96), (5, 160), (64, 64), (130, 544), (257, 1056), (33, 2080),
                                 (7, 8192), (2, 32768)])
def test_mxnorm_fwd_sr_ragged(T, D):
    """Stochastic rounding at every launch shape it plans: rows sharing a warp
    (up to 32 blocks), one block per thread (33..64), two (65..512) and four
    (up to the 32768-column maximum)."""
    x = synthetic.activations(T, D, "student_t", seed=T + D)
    g = synthetic.gamma(D, seed=D)
    xd, gd = _dev(x), _dev(g)
    q, s, G = ops.mxnorm_fwd(xd, gd, 2.0, rounding=ops.SR, seed=D)
    torch.cuda.synchronize()
    check_mxnorm_fwd(xd, gd, 2.0, ops.SR, D, q, s, G)


@pytest.mark.parametrize("D", [1024, 4096])
def test_mxnorm_fwd_sr_small_magnitudes(D):
    """Stochastic rounding where many scaled values fall under 2^-6 (the E4M3
    subnormal steps, where the kernel leaves its integer fast form for the exact
    threshold): each block holds one large value and others spread over 2^-30
    .. 1 of it, with zeros mixed in."""
    T = 96
    gen = torch.Generator().manual_seed(D)
    mag = torch.exp2(-30.0 * torch.rand(T, D, generator=gen))
    sign = torch.where(torch.rand(T, D, generator=gen) < 0.5, -1.0, 1.0)
    x = (sign * mag).view(T, D // 32, 32)
    x[:, :, 0] = 4.0
    x = x.view(T, D)
    x[torch.rand(T, D, generator=gen) < 0.05] = 0.0
    x = x.to(torch.bfloat16)
    xd = _dev(x)
    for seed in (1, 0xDEAD_BEEF_0123):
        q, s, G = ops.mxnorm_fwd(xd, None, 2.0, rounding=ops.SR, seed=seed)
        torch.cuda.synchronize()
        check_mxnorm_fwd(xd, None, 2.0, ops.SR, seed, q, s, G)


def test_mxnorm_fwd_special_rows():
    D = 1024
    x = torch.zeros(8, D, dtype=torch.bfloat16)
    x[1] = 3.0                                   # constant magnitude: G = 3 exactly
    x[1, ::2] = -3.0
    x[2, 100] = 5.0                              # one spike
    x[3] = synthetic.activations(1, D, "normal", seed=1)[0] * 1e-38  # near the subnormal range
    x[4] = synthetic.activations(1, D, "normal", seed=2)[0] * 1e37   # near the top of the range
    x[5, :512] = 1.0                             # half zero
    x[6] = torch.tensor(1.0, dtype=torch.bfloat16)
    x[6, 0] = 2.0**-133                           # smallest bf16 subnormal next to 1
    x[7] = synthetic.activations(1, D, "outliers", seed=3)[0]
    xd = _dev(x)
    for p in (2.0, 1.0, 4.0, math.inf):
        q, s, G = ops.mxnorm_fwd(xd, None, p)
        torch.cuda.synchronize()
        check_mxnorm_fwd(xd, None, p, 0, 0, q, s, G)
        Gh = G.cpu()
        assert Gh[0] == 0 and Gh[1] == 3.0


@pytest.mark.parametrize("D", [512, 1024, 3072, 8192])
@pytest.mark.parametrize("p", [2.0, 1.0, 4.0])
def test_mxnorm_fwd_wide_range_rows(D, p):
    """Rows whose block maxima span up to 2^-40 of the row maximum: the p-mean's
    terms then fall outside the range the fp32 hi/lo sum holds exactly, and the
    kernel sums them in double; the strict clause (scales and codes equal to the
    oracle's own result) must still hold."""
    T = 48
    x = synthetic.activations(T, D, "normal", seed=D + 1)
    gen = torch.Generator().manual_seed(D)
    k = torch.randint(0, 41, (T, D // 32), generator=gen).float()
    k[:, 0] = 0.0                                          # one block at full size per row
    x = (x.float().view(T, D // 32, 32) * torch.exp2(-k)[:, :, None]).view(T, D).to(torch.bfloat16)
    xd = _dev(x)
    gd = _dev(synthetic.gamma(D, seed=D))
    q, s, G = ops.mxnorm_fwd(xd, gd, p)
    torch.cuda.synchronize()
    rep = check_mxnorm_fwd(xd, gd, p, 0, 0, q, s, G)
    assert rep["strict_G_bit_mismatch_rows"] == 0, rep


def test_mxnorm_fwd_nonfinite_blocks():
    """Out of contract but defined: NaN/inf mark their blocks (scale 0xFF, code 0x7F)."""
    D = 128
    x = torch.ones(3, D, dtype=torch.bfloat16)
    x[0, 5] = float("nan")
    x[1, 70] = float("inf")
    x[2, 33] = -float("inf")
    xd = _dev(x)
    q, s, G = ops.mxnorm_fwd(xd, None, 2.0)
    torch.cuda.synchronize()
    q_ref, s_ref, _ = oracle.mxnorm_fwd(x, None, 2.0, G_in=G.cpu().numpy())
    assert np.array_equal(to_np_u8(s), s_ref) and np.array_equal(to_np_u8(q), q_ref)
    assert math.isnan(float(G[0])) and math.isinf(float(G[1]))


def test_mxnorm_fwd_mma_scale_layout():
    """Scales in the tcgen05 128 x 4 layout: every (row, block) byte equals the
    oracle's own scale (the strict clause), codes and G equal the row-major
    call's, which is checked against the oracle, and the layout's padding rows
    and columns stay untouched."""
    T, D = 300, 4128          # ragged in both padded dimensions
    x = _dev(synthetic.activations(T, D, "normal", seed=9))
    g = _dev(synthetic.gamma(D, seed=9))
    K = D // 32
    kp4 = (K + 3) // 4 * 4
    s1 = torch.full((ops.scales_bytes(T, D, ops.SCALES_MMA),), 0xAB, dtype=torch.uint8, device="cuda")
    q1, s1, G1 = ops.mxnorm_fwd(x, g, 2.0, scale_layout=ops.SCALES_MMA, scales=s1)
    q0, s0, G0 = ops.mxnorm_fwd(x, g, 2.0)
    torch.cuda.synchronize()
    check_mxnorm_fwd(x, g, 2.0, 0, 0, q0, s0, G0)
    assert torch.equal(q1, q0) and torch.equal(G1, G0)
    _, s_ref, _ = oracle.mxnorm_fwd(x.cpu(), g.cpu(), 2.0)
    rows, ks = np.meshgrid(np.arange(T), np.arange(K), indexing="ij")
    off = mma_scale_offset(rows, ks, kp4)
    sh = to_np_u8(s1)
    assert np.array_equal(sh[off], s_ref)
    untouched = np.ones(sh.size, bool)
    untouched[off.ravel()] = False
    assert np.all(sh[untouched] == 0xAB)


# ------------------------------------------------------------------- MXCast

@pytest.mark.parametrize("rounding", [ops.RNE, ops.SR])
@pytest.mark.parametrize("T,D", [(64, 1024), (3, 96), (17, 4128)])
def test_mxfp8_cast(rounding, T, D):
    x = _dev(synthetic.activations(T, D, "student_t", seed=D))
    q, s = ops.mxfp8_cast(x, rounding=rounding, seed=77)
    torch.cuda.synchronize()
    check_cast(x, rounding, 77, q, s)


def test_cast_every_bf16_pattern():
    """Every finite bf16 value through the cast: each block holds one anchor that
    fixes its scale and 31 test values, so the E4M3 conversion of every bf16
    magnitude at several scales is compared with the oracle's rounding."""
    bits = np.arange(65536, dtype=np.uint32)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    vals = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float()
    rows = []
    for anchor in (448.0, 2.0**100, 2.0**-100, 1.0, 3.0e38):
        n = vals.numel()
        nb = (n + 30) // 31
        blk = torch.zeros(nb, 32)
        blk[:, 0] = anchor
        flat = torch.zeros(nb * 31)
        flat[:n] = vals.clamp(-anchor, anchor)
        blk[:, 1:] = flat.view(nb, 31)
        rows.append(blk.reshape(-1))
    x = torch.cat(rows)
    x = x[: x.numel() // 1024 * 1024].view(-1, 1024).to(torch.bfloat16)
    xd = _dev(x)
    for rounding in (ops.RNE, ops.SR):
        q, s = ops.mxfp8_cast(xd, rounding=rounding, seed=5)
        torch.cuda.synchronize()
        check_cast(xd, rounding, 5, q, s)


# ---------------------------------------------------- RMSNorm + two-pass

@pytest.mark.parametrize("T,D", [(256, 1024), (33, 4096), (5, 96), (3, 16384)])
def test_rmsnorm_and_two_pass(T, D):
    x = _dev(synthetic.activations(T, D, "outliers", seed=D))
    g = _dev(synthetic.gamma(D, seed=D))
    q, s, y = ops.rmsnorm_then_mxcast(x, g, 1e-5)
    torch.cuda.synchronize()
    y_ref = oracle.rmsnorm(x.cpu(), g.cpu(), eps=1e-5)
    d = bf16_ulp_distance(y.cpu().view(torch.int16).numpy().view(np.uint16), y_ref)
    assert d.max() <= 1, f"RMSNorm differs by {d.max()} bf16 steps"
    check_cast(y, ops.RNE, 0, q, s)      # the cast of the kernel's y is exact


# ----------------------------------------------------------------- backward

@pytest.mark.parametrize("T,D", [(256, 1024), (64, 4096), (5, 96), (3, 16384), (130, 544)])
@pytest.mark.parametrize("with_gamma", [True, False])
def test_mxnorm_bwd(T, D, with_gamma):
    x = _dev(synthetic.activations(T, D, "normal", seed=D))
    g = _dev(synthetic.gamma(D, seed=D)) if with_gamma else None
    dy = _dev(synthetic.upstream_grad(T, D, seed=D))
    _, _, G = ops.mxnorm_fwd(x, g, 2.0)
    dx, dg = ops.mxnorm_bwd(x, dy, g, G)
    torch.cuda.synchronize()
    dx_ref, dg_ref = oracle.mxnorm_bwd(x.cpu(), dy.cpu(), None if g is None else g.cpu(), G.cpu().numpy())
    assert rel_l2(dx.float().cpu().numpy(), round_bf16(dx_ref)) <= BWD_RTOL_L2
    check_bwd_elementwise(dx, dx_ref, 1)
    if with_gamma:
        assert rel_l2(dg.float().cpu().numpy(), round_bf16(dg_ref)) <= BWD_RTOL_L2
        check_bwd_elementwise(dg, dg_ref, None)
        # deterministic: a second call gives the same bits
        _, dg2 = ops.mxnorm_bwd(x, dy, g, G)
        assert torch.equal(dg, dg2)


# ------------------------------------------------------- full-size workloads

def _sample_rows(T, n=48):
    r = np.unique(np.concatenate([[0, 1, T // 2, T - 2, T - 1],
                                  np.random.default_rng(T).integers(0, T, n)]))
    return r


def test_llama8b_shape_sampled_rows():
    """8192 x 4096, 1% outlier channels x50, p = 2, gamma: the launch the bench times."""
    w = synthetic.WORKLOADS["llama8b_8192x4096_outliers_p2"]
    x = synthetic.activations(w["T"], w["D"], w["kind"], seed=0, device="cuda")
    g = synthetic.gamma(w["D"], seed=0, device="cuda")
    q, s, G = ops.mxnorm_fwd(x, g, 2.0)
    torch.cuda.synchronize()
    rep = check_mxnorm_fwd(x, g, 2.0, 0, 0, q, s, G, rows=_sample_rows(w["T"]))
    print(rep)
    # whole-tensor properties: every block fits its scale, nothing saturates to NaN
    assert not torch.any((q & 0x7F) == 0x7F)
    assert int(s.min()) > 0 and int(s.max()) < 0xFF


@pytest.mark.parametrize("D", [2048, 4096, 8192, 16384])
def test_sweep_sampled_rows(D):
    x = synthetic.activations(16384, D, "student_t", seed=1, device="cuda")
    rows = _sample_rows(16384, n=16)
    for p in synthetic.SWEEP_P:
        for rounding in (ops.RNE, ops.SR):
            q, s, G = ops.mxnorm_fwd(x, None, p, rounding=rounding, seed=0)
            torch.cuda.synchronize()
            check_mxnorm_fwd(x, None, p, rounding, 0, q, s, G, rows=rows)
    del x
    torch.cuda.empty_cache()


def test_bwd_full_size_sampled():
    T, D = 8192, 4096
    x = synthetic.activations(T, D, "normal", seed=0, device="cuda")
    g = synthetic.gamma(D, seed=0, device="cuda")
    dy = synthetic.upstream_grad(T, D, seed=0, device="cuda")
    _, _, G = ops.mxnorm_fwd(x, g, 2.0)
    dx, dg = ops.mxnorm_bwd(x, dy, g, G)
    torch.cuda.synchronize()
    rows = _sample_rows(T)
    dx_ref, _ = oracle.mxnorm_bwd(x.cpu(), dy.cpu(), g.cpu(), G.cpu().numpy()[rows], rows=rows)
    assert rel_l2(dx.float().cpu().numpy()[rows], round_bf16(dx_ref)) <= BWD_RTOL_L2
    check_bwd_elementwise(dx.cpu()[torch.from_numpy(rows)], dx_ref, 1)
    _, dg_ref = oracle.mxnorm_bwd(x.cpu(), dy.cpu(), g.cpu(), G.cpu().numpy())
    assert rel_l2(dg.float().cpu().numpy(), round_bf16(dg_ref)) <= BWD_RTOL_L2
    check_bwd_elementwise(dg, dg_ref, None)


def test_tuning_variants_agree():
    """Every launch shape computes the same bits."""
    x = _dev(synthetic.activations(999, 4096, "outliers", seed=4))
    g = _dev(synthetic.gamma(4096, seed=4))
    ref = ops.mxnorm_fwd(x, g, 2.0)
    try:
        for nct, st, cps in [(256, 4, 0), (512, 2, 1), (128, 16, 2), (128, 2, 8)]:
            ops.set_tuning(nct, st, cps)
            out = ops.mxnorm_fwd(x, g, 2.0)
            for a, b in zip(ref, out):
                assert torch.equal(a, b)
    finally:
        ops.set_tuning(0, 0, 0)


def test_status_clean_and_empty_input():
    x = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    q, s, G = ops.mxnorm_fwd(x)
    assert q.numel() == 0
    assert ops.device_status() == ops.MXN_OK


def test_more_than_2_31_elements_sampled_rows():
    """A 524800 x 4096 tensor (2.15e9 elements, past 32-bit element indices):
    forward (nearest-even, and stochastic, whose Philox counter is the 64-bit
    element index / 4) and backward, checked on rows at both ends and around
    the 2^31-element mark."""
    T, D = 524800, 4096
    x = synthetic.activations(T, D, "normal", seed=3, device="cuda")
    g = synthetic.gamma(D, seed=3, device="cuda")
    rows = np.array([0, 1, 524287, 524288, T - 2, T - 1])
    for rounding in (ops.RNE, ops.SR):
        q, s, G = ops.mxnorm_fwd(x, g, 2.0, rounding=rounding, seed=11)
        torch.cuda.synchronize()
        check_mxnorm_fwd(x, g, 2.0, rounding, 11, q, s, G, rows=rows)
        del q, s, G
        torch.cuda.empty_cache()
    dy = synthetic.upstream_grad(T, D, seed=3, device="cuda")
    _, _, G = ops.mxnorm_fwd(x, g, 2.0)
    dx, dg = ops.mxnorm_bwd(x, dy, g, G)
    torch.cuda.synchronize()
    sel = torch.from_numpy(rows).cuda()
    dx_ref, _ = oracle.mxnorm_bwd(x[sel].cpu(), dy[sel].cpu(), g.cpu(), G[sel].cpu().numpy())
    assert rel_l2(dx[sel].double().cpu().numpy(), round_bf16(dx_ref)) <= BWD_RTOL_L2
    check_bwd_elementwise(dx[sel], dx_ref, 1)
    assert torch.isfinite(dg.float()).all()
    del x, dy, dx, G
    torch.cuda.empty_cache()
