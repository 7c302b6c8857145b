"""GPU parity of the MXNorm variants against the CPU oracle, through the C ABI.

* MXFP4 (E2M1 codes, two per byte) forward and cast, nearest-even and
  stochastic: two-stage parity as for MXFP8 (G within 1e-6, then scales and
  code bytes bit-exact from the kernel's G).
* Scale-reuse statistic (G from the blocks' power-of-two scales), both formats.
* Gain cast and MXNormLinear weight folding: bit-exact codes and scales; the
  folded chain MXNorm(gamma = NULL) -> GEMM(folded weight) against the oracle's
  chain entry by entry, and against the unfolded chain within quantisation
  error.
* Every finite bf16 value through the FP4 casts, and every finite bf16
  magnitude as a block's absmax under each format's scale rule.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from normalisation_row_bf16_b200 import build as nbuild
from normalisation_row_bf16_b200 import ops, synthetic

from parity_util import check_cast, check_mxnorm_fwd, mma_scale_offset, to_np_u8

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


# ------------------------------------------------------------------- MXFP4

@pytest.mark.parametrize("T,D,kind", [(64, 1024, "normal"), (37, 4096, "outliers"), (5, 96, "student_t"),
                                      (130, 2048, "student_t"), (9, 8192, "outliers"), (3, 16384, "normal"),
                                      (1, 32, "normal"), (33, 2080, "student_t"), (2, 32768, "student_t")])
@pytest.mark.parametrize("rounding", [ops.RNE, ops.SR])
def test_mxfp4_forward(T, D, kind, rounding):
    x = _dev(synthetic.activations(T, D, kind, seed=T + D))
    g = _dev(synthetic.gamma(D, seed=T))
    q, s, G = ops.mxnorm_fwd_ex(x, g, 2.0, rounding=rounding, seed=77, elem="e2m1")
    torch.cuda.synchronize()
    assert q.shape == (T, D // 2)
    check_mxnorm_fwd(x, g, 2.0, rounding, 77, q, s, G, fmt="e2m1")


@pytest.mark.parametrize("p", [1.0, 4.0, math.inf, 2.5])
def test_mxfp4_forward_p_and_no_gamma(p):
    T, D = 50, 2080
    x = _dev(synthetic.activations(T, D, "outliers", seed=3))
    q, s, G = ops.mxnorm_fwd_ex(x, None, p, elem="e2m1")
    torch.cuda.synchronize()
    check_mxnorm_fwd(x, None, p, ops.RNE, 0, q, s, G, fmt="e2m1")


def test_mxfp4_codes_match_e2m1_cast_of_kernel_y():
    """The packed nibbles decode (ml-dtypes-free: via the oracle's value table)
    to values within the scaled block range, and the even column is the low nibble."""
    T, D = 8, 256
    x = _dev(synthetic.activations(T, D, "normal", seed=4))
    q, s, G = ops.mxnorm_fwd_ex(x, None, 2.0, elem="e2m1")
    qh = to_np_u8(q)
    lo, hi = qh & 0xF, qh >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(T, D)
    vals = np.array([oracle.e2m1_value(c & 7) for c in range(16)]) * np.where(np.arange(16) & 8, -1, 1)
    dec = vals[codes] * np.repeat(2.0 ** (to_np_u8(s).astype(np.int64) - 127), 32, axis=1)
    y = x.float().cpu().numpy() / G.cpu().numpy()[:, None]
    blk = np.repeat(2.0 ** (to_np_u8(s).astype(np.int64) - 127), 32, axis=1)
    assert np.all(np.abs(dec - y) <= blk * 1.0 + 1e-30)        # within one E2M1 step (<= 2 * 2^e / 2)


def test_mxfp4_mma_scale_layout():
    T, D = 260, 4224
    x = _dev(synthetic.activations(T, D, "normal", seed=2))
    q0, s0, G0 = ops.mxnorm_fwd_ex(x, None, 2.0, elem="e2m1")
    q1, s1, G1 = ops.mxnorm_fwd_ex(x, None, 2.0, elem="e2m1", scale_layout=ops.SCALES_MMA)
    torch.cuda.synchronize()
    assert torch.equal(q0, q1) and torch.equal(G0, G1)
    K = D // 32
    rows, ks = np.meshgrid(np.arange(T), np.arange(K), indexing="ij")
    off = mma_scale_offset(rows, ks, (K + 3) // 4 * 4)
    assert np.array_equal(to_np_u8(s1)[off], to_np_u8(s0))


@pytest.mark.parametrize("rounding", [ops.RNE, ops.SR])
@pytest.mark.parametrize("with_gain", [False, True])
def test_mxfp4_cast(rounding, with_gain):
    T, D = 33, 4096
    x = _dev(synthetic.activations(T, D, "student_t", seed=12))
    gain = _dev(synthetic.gamma(D, seed=12)) if with_gain else None
    q, s = ops.mx_cast(x, gain, rounding=rounding, seed=5, elem="e2m1")
    torch.cuda.synchronize()
    check_cast(x, rounding, 5, q, s, gain_dev=gain, fmt="e2m1")


def test_mxfp4_nonfinite_block():
    T, D = 3, 128
    x = synthetic.activations(T, D, "normal", seed=1)
    x[1, 40] = float("nan")
    x[2, 100] = float("inf")
    xd = _dev(x)
    q, s = ops.mx_cast(xd, elem="e2m1")
    torch.cuda.synchronize()
    check_cast(xd, ops.RNE, 0, q, s, fmt="e2m1")
    assert to_np_u8(s)[1, 1] == 0xFF and np.all(to_np_u8(q)[1, 16:32] == 0x77)


# -------------------------------------------------------------- scale reuse

@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
@pytest.mark.parametrize("p", [2.0, 1.0, 4.0, math.inf])
@pytest.mark.parametrize("T,D", [(40, 4096), (7, 1024), (3, 8192)])
def test_scale_reuse_forward(fmt, p, T, D):
    x = _dev(synthetic.activations(T, D, "outliers", seed=D + 1))
    g = _dev(synthetic.gamma(D, seed=1))
    q, s, G = ops.mxnorm_fwd_ex(x, g, p, elem=fmt, stat="scale_exp")
    torch.cuda.synchronize()
    check_mxnorm_fwd(x, g, p, ops.RNE, 0, q, s, G, stat="scale_exp", fmt=fmt)


def test_scale_reuse_zero_and_tiny_blocks():
    T, D = 4, 256
    x = torch.zeros(T, D, dtype=torch.bfloat16)
    x[1, 3] = 1e-38                        # a block whose scale clamps at 2^-127
    x[2, :] = 1.0
    x[3, 200] = 3e38
    xd = _dev(x)
    q, s, G = ops.mxnorm_fwd_ex(xd, None, 2.0, stat="scale_exp")
    torch.cuda.synchronize()
    check_mxnorm_fwd(xd, None, 2.0, ops.RNE, 0, q, s, G, stat="scale_exp")


# ------------------------------------------------------ gain cast / folding

@pytest.mark.parametrize("rounding", [ops.RNE, ops.SR])
@pytest.mark.parametrize("T,D", [(6144, 4096), (17, 4128), (3, 96)])
def test_gain_cast_e4m3(rounding, T, D):
    w = _dev(synthetic.gemm_weight(T, D, seed=D))
    g = _dev(synthetic.gamma(D, seed=D))
    q, s = ops.mx_cast(w, g, rounding=rounding, seed=3)
    torch.cuda.synchronize()
    if T > 512:                           # full weight: rows sampled, every row of the sample checked
        rows = np.random.default_rng(0).choice(T, 256, replace=False)
        q_ref, s_ref = oracle.mx_cast(w.cpu(), g.cpu(), rows=rows, rounding=rounding, seed=3)
        assert np.array_equal(to_np_u8(s)[rows], s_ref) and np.array_equal(to_np_u8(q)[rows], q_ref)
    else:
        check_cast(w, rounding, 3, q, s, gain_dev=g)


def _dequant_e4m3(q, s):
    v = torch.from_numpy(q).view(torch.float8_e4m3fn).double()
    sc = torch.from_numpy(s).view(torch.float8_e8m0fnu).double()
    return (v.reshape(q.shape[0], -1, 32) * sc[:, :, None]).reshape(q.shape)


def test_folded_linear_chain():
    """MXNorm(x, gamma = NULL) @ fold(W, gamma)^T against the oracle's chain,
    and against the unfolded chain MXNorm(x, gamma) @ cast(W)^T."""
    M, K, N = 256, 2048, 512
    x = _dev(synthetic.activations(M, K, "outliers", seed=21))
    g = _dev(synthetic.gamma(K, seed=21))
    w = _dev(synthetic.gemm_weight(N, K, seed=21))
    aq, a_s, _ = ops.mxnorm_fwd(x, None, 2.0, scale_layout=ops.SCALES_MMA)
    bq, b_s = ops.fold_weight(w, g)
    c = ops.mxfp8_gemm(aq, a_s, bq, b_s, M, N, K)
    torch.cuda.synchronize()
    # oracle chain from the host copies of the inputs (the codes of A from the
    # kernel's G bits: two-stage parity)
    _, as_row, G_k = ops.mxnorm_fwd(x, None, 2.0)
    _, bs_row = ops.mx_cast(w, g)
    aq_r, as_r, _ = oracle.mxnorm_fwd(x.cpu(), None, 2.0, G_in=G_k.cpu().numpy())
    bq_r, bs_r = oracle.mx_cast(w.cpu(), g.cpu())
    assert np.array_equal(to_np_u8(aq), aq_r) and np.array_equal(to_np_u8(as_row), as_r)
    assert np.array_equal(to_np_u8(bq), bq_r) and np.array_equal(to_np_u8(bs_row), bs_r)
    ii, jj = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    ii, jj = ii.ravel(), jj.ravel()
    ref = oracle.mxfp8_gemm_entries(aq_r, as_r, bq_r, bs_r, ii, jj)
    A, B = _dequant_e4m3(aq_r, as_r), _dequant_e4m3(bq_r, bs_r)
    absdot = (A[ii].abs() * B[jj].abs()).sum(dim=1).numpy()
    got = c.float().cpu().numpy()[ii, jj].astype(np.float64)
    tol = 2.0 ** -8 * np.abs(ref) + K * 2.0 ** -24 * absdot
    assert np.all(np.abs(got - ref) <= tol)
    # the folded and the unfolded layer agree to within the two quantisations
    aq2, a_s2, _ = ops.mxnorm_fwd(x, g, 2.0, scale_layout=ops.SCALES_MMA)
    bq2, b_s2 = ops.mxfp8_cast(w, scale_layout=ops.SCALES_MMA)
    c2 = ops.mxfp8_gemm(aq2, a_s2, bq2, b_s2, M, N, K)
    xf = x.double().cpu().numpy()
    G = np.array([oracle.pmean(np.abs(xf[t].reshape(-1, 32)).max(1), 2.0) for t in range(M)])
    ref_exact = ((xf / G[:, None]) * g.double().cpu().numpy()) @ w.double().cpu().numpy().T
    e1 = np.linalg.norm(c.double().cpu().numpy() - ref_exact) / np.linalg.norm(ref_exact)
    e2 = np.linalg.norm(c2.double().cpu().numpy() - ref_exact) / np.linalg.norm(ref_exact)
    assert e1 < 0.05 and e2 < 0.05 and abs(e1 - e2) < 0.02


def test_fold_weight_requires_gamma_and_checks_format():
    w = _dev(synthetic.gemm_weight(4, 64, seed=0))
    q = torch.empty(4, 64, dtype=torch.uint8, device="cuda")
    s = torch.empty(4, 2, dtype=torch.uint8, device="cuda")
    L = ops.lib()
    st = ops._stream(None)
    assert L.mxnorm_fold_weight(w.data_ptr(), None, q.data_ptr(), s.data_ptr(), 4, 64, 64, 0, 0, st) == ops.MXN_ERR_ARG
    g = _dev(synthetic.gamma(64, seed=0))
    assert L.mxnorm_fold_weight(w.data_ptr(), g.data_ptr(), q.data_ptr(), s.data_ptr(), 4, 64, 64, 7, 0, st) == ops.MXN_ERR_ARG
    assert L.mxnorm_fwd_ex(w.data_ptr(), None, q.data_ptr(), s.data_ptr(), None, 4, 64, 64, 2.0, 0, 0, 0, 0, 5, st) == ops.MXN_ERR_ARG


@pytest.mark.parametrize("elem,stat", [("e2m1", "absmax"), ("e4m3", "scale_exp"), ("e2m1", "scale_exp")])
def test_variants_llama8b_shape_sampled_rows(elem, stat):
    """The 8192 x 4096 outlier batch with gamma, p = 2: the launches the
    bench's mxfp4 and scale-reuse legs time, on sampled rows."""
    w = synthetic.WORKLOADS["llama8b_8192x4096_outliers_p2"]
    x = synthetic.activations(w["T"], w["D"], w["kind"], seed=0, device="cuda")
    g = synthetic.gamma(w["D"], seed=0, device="cuda")
    q, s, G = ops.mxnorm_fwd_ex(x, g, 2.0, elem=elem, stat=stat)
    torch.cuda.synchronize()
    rows = np.concatenate([np.arange(0, 8), np.random.default_rng(2).choice(w["T"], 40, replace=False),
                           np.arange(w["T"] - 8, w["T"])])
    check_mxnorm_fwd(x, g, 2.0, ops.RNE, 0, q, s, G, rows=rows, stat=stat, fmt=elem)
    for rnd in (ops.SR,):
        q, s, G = ops.mxnorm_fwd_ex(x, g, 2.0, rounding=rnd, seed=5, elem=elem, stat=stat)
        torch.cuda.synchronize()
        check_mxnorm_fwd(x, g, 2.0, rnd, 5, q, s, G, rows=rows[:16], stat=stat, fmt=elem)


def test_fold_weight_full_qkv_sampled_rows():
    """The bench's fold_weight launch: the 6144 x 4096 QKV weight times gamma."""
    w = synthetic.gemm_weight(6144, 4096, seed=0, device="cuda")
    g = synthetic.gamma(4096, seed=0, device="cuda")
    q, s = ops.fold_weight(w, g, scale_layout=ops.SCALES_ROWMAJOR)
    torch.cuda.synchronize()
    rows = np.random.default_rng(4).choice(6144, 64, replace=False)
    q_ref, s_ref = oracle.mx_cast(w.cpu(), g.cpu(), rows=rows)
    assert np.array_equal(to_np_u8(q)[rows], q_ref) and np.array_equal(to_np_u8(s)[rows], s_ref)


# ------------------------------------------------------------------- NVFP4

@pytest.mark.parametrize("T,D,kind", [(64, 1024, "normal"), (37, 4096, "outliers"), (5, 96, "student_t"),
                                      (130, 2048, "student_t"), (9, 8192, "outliers"), (3, 16384, "normal"),
                                      (1, 32, "normal"), (33, 2080, "student_t"), (2, 32768, "student_t")])
@pytest.mark.parametrize("rounding", [ops.RNE, ops.SR])
def test_nvfp4_forward(T, D, kind, rounding):
    x = _dev(synthetic.activations(T, D, kind, seed=T + 2 * D))
    g = _dev(synthetic.gamma(D, seed=T + 1))
    q, s, G = ops.mxnorm_fwd_ex(x, g, 2.0, rounding=rounding, seed=31, elem="nvfp4")
    torch.cuda.synchronize()
    assert q.shape == (T, D // 2) and s.shape == (T, D // 16)
    check_mxnorm_fwd(x, g, 2.0, rounding, 31, q, s, G, fmt="nvfp4")


@pytest.mark.parametrize("p", [1.0, 4.0, math.inf, 2.5])
@pytest.mark.parametrize("stat", ["absmax", "scale_exp"])
def test_nvfp4_forward_p_stat_no_gamma(p, stat):
    T, D = 50, 2080
    x = _dev(synthetic.activations(T, D, "outliers", seed=5))
    q, s, G = ops.mxnorm_fwd_ex(x, None, p, elem="nvfp4", stat=stat)
    torch.cuda.synchronize()
    check_mxnorm_fwd(x, None, p, ops.RNE, 0, q, s, G, fmt="nvfp4", stat=stat)


@pytest.mark.parametrize("rounding", [ops.RNE, ops.SR])
@pytest.mark.parametrize("with_gain", [False, True])
def test_nvfp4_cast(rounding, with_gain):
    T, D = 33, 4096
    x = _dev(synthetic.activations(T, D, "student_t", seed=14))
    gain = _dev(synthetic.gamma(D, seed=14)) if with_gain else None
    q, s = ops.mx_cast(x, gain, rounding=rounding, seed=6, elem="nvfp4")
    torch.cuda.synchronize()
    check_cast(x, rounding, 6, q, s, gain_dev=gain, fmt="nvfp4")


def test_nvfp4_zero_and_nonfinite_blocks():
    T, D = 4, 128
    x = synthetic.activations(T, D, "normal", seed=8)
    x[1, 16:32] = 0.0
    x[1, 48:64] = -0.0
    x[2, 70] = float("nan")
    x[3, 100] = float("-inf")
    xd = _dev(x)
    q, s = ops.mx_cast(xd, elem="nvfp4")
    torch.cuda.synchronize()
    check_cast(xd, ops.RNE, 0, q, s, fmt="nvfp4")
    sh = to_np_u8(s)
    assert sh[1, 1] == 0 and sh[1, 3] == 0 and sh[2, 4] == 0x7F and sh[3, 6] == 0x7F
    with pytest.raises(ops.MXNormError):
        ops.mxnorm_fwd_ex(xd, None, 2.0, elem="nvfp4", scale_layout=ops.SCALES_MMA)


def _finite_bf16_values(positive_only=False):
    bits = np.arange(65536, dtype=np.uint32)
    keep = ((bits >> 7) & 0xFF) != 0xFF
    if positive_only:
        keep &= bits < 0x8000
    return torch.from_numpy(bits[keep].astype(np.uint16).view(np.int16)).view(torch.bfloat16).float()


@pytest.mark.parametrize("elem", ["e2m1", "nvfp4"])
def test_fp4_cast_every_bf16_pattern(elem):
    """Every finite bf16 value through the FP4 casts: each block of 32 holds one
    anchor that fixes the scale(s) and 31 test values, at several anchors, so
    the E2M1 conversion of every bf16 magnitude is compared with the oracle's
    rounding under MX (E8M0) and NVFP4 (E4M3) scales, nearest-even and
    stochastic."""
    vals = _finite_bf16_values()
    rows = []
    for anchor in (6.0, 2.0**100, 2.0**-100, 1.0, 3.0e38, 2688.0):
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
        q, s = ops.mx_cast(xd, rounding=rounding, seed=9, elem=elem)
        torch.cuda.synchronize()
        check_cast(xd, rounding, 9, q, s, fmt=elem)


@pytest.mark.parametrize("elem", ["e4m3", "e2m1", "nvfp4"])
def test_block_scale_every_bf16_amax(elem):
    """Every finite non-negative bf16 magnitude as the absmax of its own block
    (at a random position, random sign, the other elements random fractions of
    it), so each format's scale rule meets every bf16 amax, including the
    E4M3-subnormal and saturated NVFP4 scales and the E8M0 boundaries."""
    amax = _finite_bf16_values(positive_only=True)
    B = 16 if elem == "nvfp4" else 32
    nb = amax.numel()
    rng = torch.Generator().manual_seed(11)
    frac = torch.rand(nb, B, generator=rng) * 2.0 - 1.0
    blk = (amax[:, None] * frac).to(torch.bfloat16).float()
    pos = torch.randint(0, B, (nb,), generator=rng)
    sign = torch.where(torch.rand(nb, generator=rng) < 0.5, -1.0, 1.0)
    blk[torch.arange(nb), pos] = amax * sign
    x = blk.reshape(-1)
    pad = (-x.numel()) % 1024
    x = torch.cat([x, torch.zeros(pad)]).view(-1, 1024).to(torch.bfloat16)
    xd = _dev(x)
    for rounding in (ops.RNE, ops.SR):
        q, s = ops.mx_cast(xd, rounding=rounding, seed=12, elem=elem)
        torch.cuda.synchronize()
        check_cast(xd, rounding, 12, q, s, fmt=elem)


def test_nvfp4_llama8b_shape_sampled_rows():
    w = synthetic.WORKLOADS["llama8b_8192x4096_outliers_p2"]
    x = synthetic.activations(w["T"], w["D"], w["kind"], seed=0, device="cuda")
    g = synthetic.gamma(w["D"], seed=0, device="cuda")
    rows = np.concatenate([np.arange(0, 8), np.random.default_rng(3).choice(w["T"], 40, replace=False),
                           np.arange(w["T"] - 8, w["T"])])
    for rnd in (ops.RNE, ops.SR):
        q, s, G = ops.mxnorm_fwd_ex(x, g, 2.0, rounding=rnd, seed=2, elem="nvfp4")
        torch.cuda.synchronize()
        check_mxnorm_fwd(x, g, 2.0, rnd, 2, q, s, G, rows=rows, fmt="nvfp4")


def test_binding_rejects_undersized_outputs():
    x = _dev(synthetic.activations(4, 64, "normal", seed=0))
    with pytest.raises(ValueError):
        ops.mxnorm_fwd(x, q=torch.empty(4, 32, dtype=torch.uint8, device="cuda"))
    with pytest.raises(ValueError):
        ops.mxnorm_fwd(x, G=torch.empty(3, dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError):
        ops.mxnorm_fwd(x, q=torch.empty(4, 64, dtype=torch.int8, device="cuda"))
    with pytest.raises(ValueError):
        ops.mxnorm_fwd_ex(x, elem="nvfp4", scales=torch.empty(4, 2, dtype=torch.uint8, device="cuda"))
    with pytest.raises(ValueError):
        ops.mxnorm_fwd(x, scale_layout=ops.SCALES_MMA, scales=torch.empty(64, dtype=torch.uint8, device="cuda"))
    dy = _dev(synthetic.upstream_grad(4, 64, seed=0))
    _, _, G = ops.mxnorm_fwd(x)
    with pytest.raises(ValueError):
        ops.mxnorm_bwd(x, dy, None, G, dx=torch.empty(4, 32, dtype=torch.bfloat16, device="cuda"))
    # right-sized buffers pass and are used in place
    q = torch.empty(4, 64, dtype=torch.uint8, device="cuda")
    q2, _, _ = ops.mxnorm_fwd(x, q=q)
    assert q2.data_ptr() == q.data_ptr()
