"""GPU parity of the block-scaled MXFP8 GEMM (tcgen05) against the oracle.

The operands come from the path itself: x -> mxnorm_fwd -> A (codes, scales in
the MMA layout), the weight W [K, N] -> W^T [N, K] -> mxfp8_cast -> B.  The
oracle computes C entries in float64 from the same codes and (row-major)
scales.  Tolerance per entry: bf16 output rounding (2^-8 |C|) plus the fp32
accumulation bound K * 2^-24 * sum_k |a_k b_k| (products of E4M3 values with
power-of-two scales are exact in fp32; only the additions round).
"""
import numpy as np
import pytest
import torch

import oracle
from normalisation_row_bf16_b200 import build as nbuild
from normalisation_row_bf16_b200 import ops, synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    nbuild.build()
    ops.lib()
    yield
    assert ops.device_status() == ops.MXN_OK


def _dequant(q, s):
    v = torch.from_numpy(q).view(torch.float8_e4m3fn).double()
    sc = torch.from_numpy(s).view(torch.float8_e8m0fnu).double()
    return (v.reshape(q.shape[0], -1, 32) * sc[:, :, None]).reshape(q.shape)


def _operands(M, N, K, seed):
    x = synthetic.activations(M, K, "normal", seed=seed, device="cuda")
    g = synthetic.gamma(K, seed=seed, device="cuda")
    w = synthetic.gemm_weight(N, K, seed=seed, device="cuda")          # W^T, [N, K]
    aq, a_s_mma, _ = ops.mxnorm_fwd(x, g, 2.0, scale_layout=ops.SCALES_MMA)
    _, a_s, _ = ops.mxnorm_fwd(x, g, 2.0)
    bq, b_s_mma = ops.mxfp8_cast(w, scale_layout=ops.SCALES_MMA)
    _, b_s = ops.mxfp8_cast(w)
    return aq, a_s_mma, a_s, bq, b_s_mma, b_s


def _check(aq, a_s, bq, b_s, c, ii, jj):
    aqh, ash = aq.cpu().numpy(), a_s.cpu().numpy()
    bqh, bsh = bq.cpu().numpy(), b_s.cpu().numpy()
    ref = oracle.mxfp8_gemm_entries(aqh, ash, bqh, bsh, ii, jj)
    A = _dequant(aqh, ash)
    B = _dequant(bqh, bsh)
    absdot = (A[ii].abs() * B[jj].abs()).sum(dim=1).numpy()
    got = c.float().cpu().numpy()[ii, jj].astype(np.float64)
    K = aqh.shape[1]
    tol = 2.0**-8 * np.abs(ref) + K * 2.0**-24 * absdot
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{bad.sum()} entries out of tolerance; worst {np.max(np.abs(got - ref) / (tol + 1e-30)):.2f}x"


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (256, 512, 384), (384, 256, 1024)])
def test_gemm_small_all_entries(M, N, K):
    aq, a_s_mma, a_s, bq, b_s_mma, b_s = _operands(M, N, K, seed=M + N + K)
    c = ops.mxfp8_gemm(aq, a_s_mma, bq, b_s_mma, M, N, K)
    torch.cuda.synchronize()
    ii, jj = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    _check(aq, a_s, bq, b_s, c, ii.ravel(), jj.ravel())


def test_gemm_llama8b_qkv_sampled():
    """8192 x 4096 MXNorm output times the fused QKV weight [4096 x 6144]."""
    M, K, N = 8192, 4096, 6144
    aq, a_s_mma, a_s, bq, b_s_mma, b_s = _operands(M, N, K, seed=0)
    c = ops.mxfp8_gemm(aq, a_s_mma, bq, b_s_mma, M, N, K)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    ii = np.concatenate([rng.integers(0, M, 400), [0, M - 1, 127, 128]])
    jj = np.concatenate([rng.integers(0, N, 400), [0, N - 1, 255, 256]])
    _check(aq, a_s, bq, b_s, c, ii, jj)
    assert torch.isfinite(c.float()).all()


@pytest.mark.parametrize("M,N,K", [(4352, 2560, 512), (128 * 149, 256, 256), (256, 256 * 3, 2048)])
def test_gemm_persistent_uneven_tiles_sampled(M, N, K):
    """Tile counts that do not divide evenly over the persistent CTAs (340 and
    149 tiles on 148 SMs, and fewer tiles than SMs); every tile sampled."""
    aq, a_s_mma, a_s, bq, b_s_mma, b_s = _operands(M, N, K, seed=M + 7)
    c = ops.mxfp8_gemm(aq, a_s_mma, bq, b_s_mma, M, N, K)
    torch.cuda.synchronize()
    rng = np.random.default_rng(M)
    mt, nt = M // 128, N // 256
    ti, tj = np.meshgrid(np.arange(mt), np.arange(nt), indexing="ij")
    ii = (ti.ravel() * 128 + rng.integers(0, 128, ti.size))
    jj = (tj.ravel() * 256 + rng.integers(0, 256, tj.size))
    ii = np.concatenate([ii, [0, M - 1]])
    jj = np.concatenate([jj, [N - 1, 0]])
    _check(aq, a_s, bq, b_s, c, ii, jj)


@pytest.mark.parametrize("M,N,K", [(256, 256, 128), (2048, 1536, 1024), (8192, 6144, 4096)])
def test_gemm_pair_tiles_match_single_cta_tiles(M, N, K):
    """256 x 256 tiles on CTA pairs (selected with set_gemm_tiles(1)) against
    the default 128 x 256 tiles on single CTAs: the same products accumulated
    in the same order per output, so the outputs are identical; the pair
    kernel's result is also checked against the oracle on sampled entries."""
    aq, a_s_mma, a_s, bq, b_s_mma, b_s = _operands(M, N, K, seed=M + N)
    ops.set_gemm_tiles(2)
    try:
        c_single = ops.mxfp8_gemm(aq, a_s_mma, bq, b_s_mma, M, N, K)
        ops.set_gemm_tiles(1)
        c_pair = ops.mxfp8_gemm(aq, a_s_mma, bq, b_s_mma, M, N, K)
    finally:
        ops.set_gemm_tiles(0)
    torch.cuda.synchronize()
    assert torch.equal(c_pair, c_single)
    rng = np.random.default_rng(M + 1)
    ii = np.concatenate([rng.integers(0, M, 256), [0, M - 1, 127, 128, 255]])
    jj = np.concatenate([rng.integers(0, N, 256), [0, N - 1, 127, 128, 255]])
    _check(aq, a_s, bq, b_s, c_pair, ii, jj)


@pytest.mark.parametrize("M,N,K", [(256, 768, 128), (512, 1536, 256), (2048, 1536, 1024), (8192, 6144, 4096)])
def test_gemm_wide_tiles_match_128x256_tiles(M, N, K):
    """The default 256 x 192 tiles (these shapes have M % 256 == 0 and N % 384
    == 0): odd N-tiles start 64 rows into a 128-row scale atom, which the
    kernel rebuilds in tile order; the outputs must equal the 128 x 256
    kernel's (set_gemm_tiles(2)), and sampled entries the oracle's (including
    both sides of every atom and tile boundary)."""
    aq, a_s_mma, a_s, bq, b_s_mma, b_s = _operands(M, N, K, seed=M + 3 * N)
    c_wide = ops.mxfp8_gemm(aq, a_s_mma, bq, b_s_mma, M, N, K)
    ops.set_gemm_tiles(2)
    try:
        c_single = ops.mxfp8_gemm(aq, a_s_mma, bq, b_s_mma, M, N, K)
    finally:
        ops.set_gemm_tiles(0)
    torch.cuda.synchronize()
    assert torch.equal(c_wide, c_single)
    rng = np.random.default_rng(M + 2)
    edges = [0, 63, 64, 127, 128, 191, 192, 255, 256, 383]
    ii = np.concatenate([rng.integers(0, M, 256), [e % M for e in edges], [M - 1]])
    jj = np.concatenate([rng.integers(0, N, 256), [e % N for e in edges], [N - 1]])
    jj = np.concatenate([jj, [e % N for e in edges]])
    ii = np.concatenate([ii, [(M - 1 - e) % M for e in edges]])
    _check(aq, a_s, bq, b_s, c_wide, ii, jj)
