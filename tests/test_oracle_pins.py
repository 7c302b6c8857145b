"""Pins for the CPU oracle: each check compares it with something other than itself.

* E4M3 rounding: a brute-force nearest-value search over the grid that torch's
  float8_e4m3fn decoder produces, and torch's own fp32 -> e4m3 cast where that
  cast is defined (|v| <= 464); saturation and NaN from the FP8 formats paper.
* E8M0 exponent: the closed form e = floor(log2 a) - 8 + [mantissa > 1.75]
  (448 = 1.75 * 2^8), derived from the bit layout, on every positive bf16 and a
  structured set of fp32 patterns; torch's float8_e8m0fnu decoder for the bias.
* p-mean: scipy.stats.pmean, numpy mean / max, constant rows, one-block rows.
* Theorem 1 (MXNorm page, technical summary section 2.2): G / RMS of a long
  i.i.d. N(0,1) row against the limit constant c(p, 32) by quadrature.
* Output bound (section 2.2 / 3.1): max|y| <= K^(1/p) max|gamma|, attained by a
  single-spike row; RMSNorm's sqrt(D) likewise.
* Invariants: 2^k input scaling, sign symmetry, G depends on the K block maxima
  only (the 32x smaller reduction of the lay summary, section 3).
* Stochastic rounding (aibr.jp SR article, section 3): unbiased, lands on one of
  the two neighbours, P(up) = frac; Philox4x32-10 known-answer values.
* Backward (section 2.3): finite differences of x -> x * gamma / (c rms(x)),
  orthogonality x . dx = 0, linearity in gamma.
* RMSNorm: torch.nn.functional.rms_norm in float64 rounded to bf16.
* GEMM entries: torch dequantisation (float8 decoders) and float64 matmul.
* Brute force on tiny rows: every assignment of a small value set to three
  columns of a two-block row, against the closed-form G and a Python
  evaluation of the definitions (scale by scanning e, nearest-grid codes).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from normalisation_row_bf16_b200 import synthetic

E4M3_GRID = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def _bf16_all_finite():
    """Every finite bf16 bit pattern, as float32 values."""
    bits = np.arange(65536, dtype=np.uint32)
    exp = (bits >> 7) & 0xFF
    bits = bits[exp != 0xFF]
    return (bits << 16).view(np.float32)


def _fp32_structured(rng):
    """fp32 patterns covering every round/sticky combination for E4M3 rounding:
    all 2^11 settings of mantissa bits 12..22, each exponent, both signs, and
    several low-bit fillers (incl. exact ties)."""
    hi = np.arange(2048, dtype=np.uint32) << 12
    lows = np.array([0, 1, 0x7FF, 0x800, 0x801, 0xFFF], dtype=np.uint32)
    exps = np.arange(0, 255, dtype=np.uint32) << 23
    m = (hi[:, None] | lows[None, :]).reshape(-1)
    pats = (exps[:, None] | m[None, :]).reshape(-1)
    pats = np.concatenate([pats, pats | 0x80000000,
                           rng.integers(0, 2**32, 200_000, dtype=np.uint64).astype(np.uint32)])
    v = pats.view(np.float32)
    return v[np.isfinite(v)]


def _brute_e4m3_rne(v):
    """Nearest grid value by search; ties to the even code; |v| >= 448 -> 448."""
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    idx = np.clip(np.searchsorted(E4M3_GRID, a), 1, len(E4M3_GRID) - 1)
    lo_i, hi_i = idx - 1, idx
    dlo = a - E4M3_GRID[lo_i]
    dhi = E4M3_GRID[hi_i] - a
    pick = np.where(dlo < dhi, lo_i, np.where(dhi < dlo, hi_i, np.where(lo_i % 2 == 0, lo_i, hi_i)))
    pick = np.where(a >= 448.0, 126, pick)
    pick = np.where(a <= 0.0, 0, pick)
    return (pick.astype(np.uint8) | np.where(np.signbit(v), 0x80, 0).astype(np.uint8))


# ----------------------------------------------------------------- E4M3

def test_e4m3_format_facts(golden_dir):
    facts = {}
    for line in open(os.path.join(golden_dir, "e4m3_format_facts.txt")):
        if line.strip() and not line.startswith("#"):
            k, v = line.split()
            facts[k] = float.fromhex(v) if v.startswith("0x") else float(v)
    assert oracle.e4m3_value(int(facts["max_finite_code"])) == facts["max_finite"]
    assert oracle.e4m3_value(0x08) == facts["min_normal"]
    assert oracle.e4m3_value(0x01) == facts["min_subnormal"]
    assert oracle.e4m3_rne([math.nan])[0] & 0x7F == int(facts["nan_code_positive"])
    # no infinities: huge values saturate to the largest finite code
    assert list(oracle.e4m3_rne([1e30, -1e30, math.inf, -math.inf])) == [0x7E, 0xFE, 0x7E, 0xFE]
    # the oracle's decoder agrees with torch's for every finite code
    for c in range(127):
        assert oracle.e4m3_value(c) == E4M3_GRID[c]


def test_e4m3_rne_all_bf16_vs_bruteforce():
    v = _bf16_all_finite()
    assert np.array_equal(oracle.e4m3_rne(v), _brute_e4m3_rne(v))


def test_e4m3_rne_structured_fp32_vs_bruteforce():
    v = _fp32_structured(np.random.default_rng(1))
    assert np.array_equal(oracle.e4m3_rne(v), _brute_e4m3_rne(v))


def test_e4m3_rne_vs_torch_cast_below_464():
    v = np.concatenate([_bf16_all_finite(), _fp32_structured(np.random.default_rng(2))])
    v = v[np.abs(v) <= 464.0]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_rne(v), ref)


def test_e4m3_saturation_and_signs():
    got = oracle.e4m3_rne([448.0, 449.0, 463.99, 464.0, 465.0, 3e38, -465.0, 0.0, -0.0, -1e-30])
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x80, 0x80]
    v = _fp32_structured(np.random.default_rng(3))
    assert np.array_equal(oracle.e4m3_rne(-v), oracle.e4m3_rne(v) ^ 0x80)


# ----------------------------------------------------------------- E8M0

def _e8m0_closed_form(a):
    a = np.abs(np.asarray(a, np.float32))
    bits = a.view(np.uint32)
    expf = ((bits >> 23) & 0xFF).astype(np.int64)
    mant = bits & 0x7FFFFF
    e = expf - 127 - 8 + (mant > 0x600000)
    e = np.where(expf == 0, -127, e)          # zero and fp32 subnormals
    return np.clip(e, -127, 127)


def test_e8m0_closed_form_all_bf16():
    v = _bf16_all_finite()
    assert np.array_equal(oracle.e8m0_exponent(v), _e8m0_closed_form(v))


def test_e8m0_closed_form_structured_fp32():
    v = _fp32_structured(np.random.default_rng(4))
    assert np.array_equal(oracle.e8m0_exponent(v), _e8m0_closed_form(v))


def test_e8m0_edges_and_torch_decode():
    for k in (-100, -8, 0, 5, 100):
        a = np.float32(448.0 * 2.0**k)
        assert oracle.e8m0_exponent([a])[0] == k
        assert oracle.e8m0_exponent([np.nextafter(a, np.float32(np.inf))])[0] == k + 1
        assert oracle.e8m0_exponent([np.nextafter(a, np.float32(0))])[0] == k
    assert oracle.e8m0_exponent([0.0])[0] == -127
    assert oracle.e8m0_exponent([np.finfo(np.float32).max])[0] == 120
    assert oracle.e8m0_exponent([math.nan, math.inf])[0] == 128
    # scale code = e + 127 decodes (torch) to 2^e, and the block then fits.
    a = np.abs(np.random.default_rng(5).standard_normal(1000).astype(np.float32)) * 1e3
    e = oracle.e8m0_exponent(a)
    dec = torch.from_numpy((e + 127).astype(np.uint8)).view(torch.float8_e8m0fnu).double().numpy()
    assert np.all(a <= 448.0 * dec) and np.all(a > 224.0 * dec)


# ---------------------------------------------------------------- p-mean

def test_pmean_special_cases_and_scipy():
    from scipy.stats import pmean as scipy_pmean
    rng = np.random.default_rng(6)
    m = np.abs(rng.standard_normal(128)) + 0.01
    assert oracle.pmean(m, 1.0) == pytest.approx(np.mean(m), rel=1e-14)
    assert oracle.pmean(m, 2.0) == pytest.approx(np.sqrt(np.mean(m**2)), rel=1e-14)
    assert oracle.pmean(m, math.inf) == np.max(m)
    for p in (0.5, 1.0, 2.0, 3.5, 4.0, 8.0):
        assert oracle.pmean(m, p) == pytest.approx(float(scipy_pmean(m, p)), rel=1e-12)
    # a single nonzero block among K: G = M * K^(-1/p)
    mm = np.zeros(64)
    mm[17] = 3.0
    for p in (1.0, 2.0, 4.0):
        assert oracle.pmean(mm, p) == pytest.approx(3.0 * 64 ** (-1 / p), rel=1e-14)


def test_constant_magnitude_row_gives_exact_G():
    D = 4096
    for val in (1.0, 0.3125, 3.0e-20, 7.0e25):
        signs = np.where(np.random.default_rng(7).random(D) < 0.5, -1.0, 1.0)
        x = torch.tensor(signs * val, dtype=torch.float32).to(torch.bfloat16)[None, :]
        ref = float(x.abs().max())
        for p in (1.0, 2.0, 4.0, 3.3, math.inf):
            _, _, G = oracle.mxnorm_fwd(x, None, p)
            assert G[0] == np.float32(ref)


def test_G_is_a_function_of_the_K_block_maxima_only():
    """The statistic reduces K = D/32 numbers, not D (lay summary section 3)."""
    D = 2048
    x = synthetic.activations(4, D, "normal", seed=3)
    xa = x.float().abs().reshape(4, D // 32, 32)
    for p in (1.0, 2.0, math.inf):
        _, _, G = oracle.mxnorm_fwd(x, None, p)
        for r in range(4):
            m = xa[r].max(dim=1).values.double().numpy()
            assert m.size == D // 32
            assert G[r] == np.float32(oracle.pmean(m, p))
    # perturbing a non-maximal element of a block leaves G unchanged
    y = x.clone()
    blk = xa[0, 5]
    j = int(torch.argmin(blk))
    y[0, 5 * 32 + j] = (y[0, 5 * 32 + j].float() * 0.5).to(torch.bfloat16)
    for p in (1.0, 2.0, 4.0):
        assert oracle.mxnorm_fwd(x, None, p)[2][0] == oracle.mxnorm_fwd(y, None, p)[2][0]


def _c_limit(p, B=32):
    """c(p, B) = (E[m^p])^(1/p) for m the max of B i.i.d. |N(0,1)| (RMS = 1)."""
    from scipy.integrate import quad
    from scipy.special import erf
    f = lambda z: p * z ** (p - 1) * (1.0 - erf(z / math.sqrt(2.0)) ** B)
    val, _ = quad(f, 0.0, 40.0, limit=400)
    return val ** (1.0 / p)


@pytest.mark.slow
def test_theorem1_pmean_over_rms_converges_to_c():
    assert _c_limit(1.0) == pytest.approx(2.3470, abs=2e-3)
    assert _c_limit(2.0) == pytest.approx(2.3895, abs=2e-3)
    assert _c_limit(4.0) == pytest.approx(2.4774, abs=2e-3)
    D = 1 << 20
    x = synthetic.activations(1, D, "normal", seed=11)
    rms = float(torch.sqrt((x.double() ** 2).mean()))
    for p in (1.0, 2.0, 4.0):
        _, _, G = oracle.mxnorm_fwd(x, None, p)
        assert G[0] / rms == pytest.approx(_c_limit(p), rel=1e-2)


# ------------------------------------------------------------ output bounds

def _dequant(q, s):
    v = torch.from_numpy(q).view(torch.float8_e4m3fn).double()
    sc = torch.from_numpy(s).view(torch.float8_e8m0fnu).double()
    return (v.reshape(q.shape[0], -1, 32) * sc[:, :, None]).reshape(q.shape).numpy()


def test_output_bound_K_to_the_1_over_p():
    D = 4096
    K = D // 32
    x = synthetic.activations(8, D, "outliers", seed=4)
    g = synthetic.gamma(D, seed=4)
    gmax = float(g.float().abs().max())
    for p in (1.0, 2.0, 4.0):
        q, s, _ = oracle.mxnorm_fwd(x, g, p)
        assert np.abs(_dequant(q, s)).max() <= K ** (1 / p) * gmax * (1 + 1 / 16)
    # attained by a single spike: y = K^(1/p) * gamma at the spike
    spike = torch.zeros(1, D, dtype=torch.bfloat16)
    spike[0, 100] = 3.0
    for p in (1.0, 2.0, 4.0):
        q, s, G = oracle.mxnorm_fwd(spike, None, p)
        y = _dequant(q, s)[0, 100]
        assert y == pytest.approx(K ** (1 / p), rel=1 / 16)
        assert G[0] == pytest.approx(3.0 * K ** (-1 / p), rel=1e-7)
    # RMSNorm: the same spike reaches sqrt(D)
    y = oracle.rmsnorm(spike, None, eps=0.0)
    yv = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).float()[0, 100]
    assert float(yv) == pytest.approx(math.sqrt(D), rel=2**-8)


# ------------------------------------------------------------- invariants

def test_power_of_two_scaling_invariance():
    D = 1024
    x = synthetic.activations(16, D, "normal", seed=5)
    g = synthetic.gamma(D, seed=5)
    for k in (-7, 3, 20):
        xs = (x.float() * 2.0**k).to(torch.bfloat16)
        assert torch.equal(xs.float(), x.float() * 2.0**k)
        for p in (1.0, 2.0, 4.0, math.inf):
            q0, s0, G0 = oracle.mxnorm_fwd(x, g, p)
            q1, s1, G1 = oracle.mxnorm_fwd(xs, g, p)
            assert np.array_equal(q0, q1) and np.array_equal(s0, s1)
            assert np.array_equal(G1, G0 * np.float32(2.0**k))
        q0, s0 = oracle.mxfp8_cast(x)
        q1, s1 = oracle.mxfp8_cast(xs)
        assert np.array_equal(q0, q1)
        assert np.array_equal(s1.astype(int), s0.astype(int) + k)


def test_sign_symmetry():
    D = 1024
    x = synthetic.activations(8, D, "student_t", seed=6)
    g = synthetic.gamma(D, seed=6)
    for rounding in (0, 1):
        q0, s0, _ = oracle.mxnorm_fwd(x, g, 2.0, rounding=rounding, seed=9)
        q1, s1, _ = oracle.mxnorm_fwd(-x, g, 2.0, rounding=rounding, seed=9)
        assert np.array_equal(q1, q0 ^ 0x80) and np.array_equal(s0, s1)
        q0, s0 = oracle.mxfp8_cast(x, rounding=rounding, seed=9)
        q1, s1 = oracle.mxfp8_cast(-x, rounding=rounding, seed=9)
        assert np.array_equal(q1, q0 ^ 0x80) and np.array_equal(s0, s1)


def test_zero_row_and_zero_block():
    D = 256
    x = torch.zeros(2, D, dtype=torch.bfloat16)
    x[1, 40:] = 1.0   # block 0 and the first half of block 1 stay zero
    q, s, G = oracle.mxnorm_fwd(x, None, 2.0)
    assert G[0] == 0 and np.all(q[0] == 0) and np.all(s[0] == 0)
    assert s[1, 0] == 0 and np.all(q[1, :32] == 0)


def test_nonfinite_inputs_mark_blocks_nan():
    """Out of contract, but defined: NaN/inf give scale 0xFF and code 0x7F per block."""
    D = 128
    x = torch.ones(3, D, dtype=torch.bfloat16)
    x[0, 5] = float("nan")
    x[1, 70] = float("inf")
    x[2, 33] = -float("inf")
    q, s, G = oracle.mxnorm_fwd(x, None, 2.0)
    assert math.isnan(G[0]) and np.all(s[0] == 0xFF) and np.all(q[0] == 0x7F)
    # an infinite row statistic: s = 1/inf = 0, so only the inf element's block is NaN
    assert math.isinf(G[1]) and list(s[1]) == [0, 0, 0xFF, 0]
    assert np.all(q[1, 64:96] == 0x7F) and np.all(q[1, :64] == 0)
    assert list(s[2]) == [0, 0xFF, 0, 0] and np.all(q[2, 32:64] == 0x7F)
    qc, sc = oracle.mxfp8_cast(x)
    assert list(sc[1]) == [0x77, 0x77, 0xFF, 0x77] and np.all(qc[1, 64:96] == 0x7F)


def test_scales_fit_and_are_minimal():
    """Every block fits under its scale, and would not under half of it."""
    D = 2048
    x = synthetic.activations(32, D, "outliers", seed=8)
    g = synthetic.gamma(D, seed=8)
    q, s, G = oracle.mxnorm_fwd(x, g, 2.0)
    y = (x.float() * (1.0 / torch.from_numpy(G))[:, None]) * g.float()[None, :]
    a = y.abs().reshape(32, -1, 32).amax(dim=2).double().numpy()
    sc = 2.0 ** (s.astype(np.float64) - 127)
    assert np.all(a <= 448 * sc) and np.all(a > 224 * sc)
    assert np.all(q & 0x7F != 0x7F)   # never NaN, never saturated beyond 448


# ------------------------------------------------------- stochastic rounding

def test_philox_known_answers(golden_dir):
    n = 0
    for line in open(os.path.join(golden_dir, "philox4x32_10_kat.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        w = [int(t, 16) for t in line.split()]
        assert list(oracle.philox4x32_10(w[0:4], w[4:6])) == w[6:10]
        n += 1
    assert n == 3


def test_sr_word_layout():
    seed = 0x1234_5678_9ABC_DEF0
    idx = np.arange(0, 4 * 100, dtype=np.uint64) + (np.uint64(1) << np.uint64(40))
    w = oracle.sr_words(seed, idx)
    for t in range(0, 400, 37):
        i = int(idx[t])
        c = i >> 2
        out = oracle.philox4x32_10([c & 0xFFFFFFFF, c >> 32, 0, 0],
                                   [seed & 0xFFFFFFFF, seed >> 32])
        assert w[t] == out[i & 3]


def test_sr_unbiased_and_neighbours():
    rng = np.random.default_rng(10)
    vals = np.array([1.0 + 1 / 3, 300.7, 0.0041, 0.0003, 440.0, 2**-6 * 0.77, -5.3, 0.75],
                    np.float32)
    n = 1 << 16
    for v in vals:
        words = rng.integers(0, 2**32, n, dtype=np.uint64).astype(np.uint32)
        codes = oracle.e4m3_sr(np.full(n, v, np.float32), words)
        dec = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
        a = abs(float(v))
        lo = E4M3_GRID[E4M3_GRID <= a].max()
        hi = E4M3_GRID[E4M3_GRID > a].min()
        assert set(np.unique(np.abs(dec))) <= {lo, hi}
        frac = (a - lo) / (hi - lo)
        sigma = (hi - lo) * math.sqrt(frac * (1 - frac) / n)
        assert abs(np.abs(dec).mean() - a) <= 5 * sigma + 1e-12
        assert np.all(np.sign(dec[dec != 0]) == np.sign(v))


def test_sr_exact_threshold_and_grid_values():
    on_grid = E4M3_GRID[::5].astype(np.float32)
    r = np.full(on_grid.shape, 0, np.uint32)
    assert np.array_equal(oracle.e4m3_sr(on_grid, r), oracle.e4m3_rne(on_grid))
    # v = 1 + 1/16 sits at frac = 1/2: up iff r < 2^31
    v = np.full(4, 1.0625, np.float32)
    r = np.array([0, 2**31 - 1, 2**31, 2**32 - 1], np.uint32)
    assert list(oracle.e4m3_sr(v, r)) == [0x39, 0x39, 0x38, 0x38]
    # 2^-30: frac * 2^32 = 2^11, so up iff r < 2048
    t = np.full(3, 2.0**-30, np.float32)
    assert list(oracle.e4m3_sr(t, np.array([0, 2047, 2048], np.uint32))) == [0x01, 0x01, 0x00]
    # 2^-45: frac * 2^32 = 1/16, so only r = 0 rounds up to the smallest subnormal
    t = np.full(2, 2.0**-45, np.float32)
    assert list(oracle.e4m3_sr(t, np.array([0, 1], np.uint32))) == [0x01, 0x00]


# ---------------------------------------------------------------- backward

def test_backward_finite_differences():
    rng = np.random.default_rng(12)
    D = 64
    x = synthetic.activations(3, D, "normal", seed=12)
    g = synthetic.gamma(D, seed=12)
    dy = synthetic.upstream_grad(3, D, seed=12, std=1.0)
    c = 2.3895
    xd, gd, dyd = x.double().numpy(), g.double().numpy(), dy.double().numpy()
    rms = np.sqrt((xd**2).mean(axis=1))
    G = (c * rms).astype(np.float32)
    dx, dgam = oracle.mxnorm_bwd(x, dy, g, G)

    def L(xr, gg, dyr):
        return float(np.sum(dyr * xr * gg / (c * np.sqrt((xr**2).mean()))))

    h = 1e-6
    for r in range(3):
        fd = np.empty(D)
        for j in range(D):
            e = np.zeros(D)
            e[j] = h
            fd[j] = (L(xd[r] + e, gd, dyd[r]) - L(xd[r] - e, gd, dyd[r])) / (2 * h)
        # G enters the oracle as fp32: allow its rounding (~6e-8 relative)
        assert np.allclose(dx[r], fd, rtol=1e-5, atol=1e-7 * np.abs(fd).max())
        assert abs(np.dot(xd[r], dx[r])) <= 1e-12 * np.abs(xd[r]).sum() * np.abs(dx[r]).max()
    # gamma enters linearly and G does not depend on it
    def Lg(gg):
        return float(sum(np.sum(dyd[r] * xd[r] * gg / np.float64(G[r])) for r in range(3)))

    fdg = np.zeros(D)
    for j in range(D):
        e = np.zeros(D)
        e[j] = h
        fdg[j] = (Lg(gd + e) - Lg(gd - e)) / (2 * h)
    assert np.allclose(dgam, fdg, rtol=1e-6)
    dx_t, _ = oracle.mxnorm_bwd(x, dy, g, G, true_rms=True)
    assert np.allclose(dx_t, dx * (G.astype(np.float64) / rms)[:, None], rtol=1e-12)


# ----------------------------------------------------------------- RMSNorm

def test_rmsnorm_vs_torch_float64():
    """The oracle's bf16 output is the bf16 value nearest to torch's float64 RMSNorm
    (checked against both bf16 neighbours; torch's own float64 -> bf16 conversion
    rounds twice, through fp32, so it is not used)."""
    D = 1024
    x = synthetic.activations(64, D, "outliers", seed=13)
    g = synthetic.gamma(D, seed=13)
    ref = torch.nn.functional.rms_norm(x.double(), (D,), g.double(),
                                       eps=float(np.float32(1e-5))).numpy()
    got = oracle.rmsnorm(x, g, eps=1e-5)
    b = got.astype(np.uint32)
    val = (b << 16).view(np.float32).astype(np.float64)
    up = ((b + 1) << 16).view(np.float32).astype(np.float64)
    dn = ((b - 1) << 16).view(np.float32).astype(np.float64)
    err = np.abs(val - ref)
    assert np.all(err <= np.abs(up - ref)) and np.all(err <= np.abs(dn - ref))
    assert np.all(np.sign(val) == np.sign(ref))


# -------------------------------------------------------------------- GEMM

def test_gemm_entries_vs_torch_dequant():
    rng = np.random.default_rng(14)
    M, N, K = 16, 12, 128
    aq = rng.integers(0, 256, (M, K), dtype=np.uint8)
    bq = rng.integers(0, 256, (N, K), dtype=np.uint8)
    aq[(aq & 0x7F) == 0x7F] = 0x11
    bq[(bq & 0x7F) == 0x7F] = 0x22
    a_s = rng.integers(117, 137, (M, K // 32), dtype=np.uint8)
    b_s = rng.integers(117, 137, (N, K // 32), dtype=np.uint8)

    def deq(q, s):
        v = torch.from_numpy(q).view(torch.float8_e4m3fn).double()
        sc = torch.from_numpy(s).view(torch.float8_e8m0fnu).double()
        return (v.reshape(q.shape[0], -1, 32) * sc[:, :, None]).reshape(q.shape)

    ref = deq(aq, a_s) @ deq(bq, b_s).T
    ii, jj = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    c = oracle.mxfp8_gemm_entries(aq, a_s, bq, b_s, ii.ravel(), jj.ravel())
    assert np.allclose(c.reshape(M, N), ref.numpy(), rtol=1e-12, atol=1e-300)


def _brute_row(xrow, G, gamma=None):
    """Codes and scales of one row from the definitions, in Python: y by numpy
    float32 operations, the scale by scanning e, codes by nearest-grid search
    (ties to the even code) on the E4M3 grid."""
    s = np.float32(0.0) if G == 0 else np.float32(1.0) / np.float32(G)
    y = (xrow.astype(np.float32) * s).astype(np.float32)
    if gamma is not None:
        y = (y * gamma.astype(np.float32)).astype(np.float32)
    codes, scales = [], []
    for k in range(y.size // 32):
        blk = y[32 * k:32 * (k + 1)]
        a = float(np.max(np.abs(blk.astype(np.float64))))
        e = next(e for e in range(-127, 128) if a <= 448.0 * 2.0 ** e)
        scales.append(e + 127)
        v = (blk * np.float32(2.0 ** -e)).astype(np.float32).astype(np.float64)
        av = np.minimum(np.abs(v), 448.0)
        d = np.abs(av[:, None] - E4M3_GRID[None, :])
        best = d.min(axis=1, keepdims=True)
        cand = d == best
        even = cand & (np.arange(E4M3_GRID.size)[None, :] % 2 == 0)
        idx = np.where(cand.sum(1) > 1, even.argmax(1), cand.argmax(1))
        codes.append((idx | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8))
    return np.concatenate(codes), np.array(scales, np.uint8)


def test_brute_force_tiny_rows_every_pattern():
    """D = 64 (K = 2): every assignment of {0, 1, -1.5, 3.25, -96, 2^-20} to
    columns 0, 5 (block 0) and 40 (block 1), the rest zero; p = 2 and inf,
    without and with a gain.  G against the closed form, codes and scales
    against the brute-force row."""
    import itertools
    vals = [0.0, 1.0, -1.5, 3.25, -96.0, 2.0 ** -20]
    rows = []
    for a, b, c in itertools.product(vals, repeat=3):
        r = np.zeros(64, np.float32)
        r[0], r[5], r[40] = a, b, c
        rows.append(r)
    x = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    xf = x.float().numpy()
    gam = torch.from_numpy((1.0 + 0.25 * np.arange(64) / 64).astype(np.float32)).to(torch.bfloat16)
    for p in (2.0, math.inf):
        for g in (None, gam):
            q, s, G = oracle.mxnorm_fwd(x, g, p)
            for t in range(xf.shape[0]):
                m = np.abs(xf[t].astype(np.float64)).reshape(2, 32).max(1)
                Gw = m.max() if math.isinf(p) else math.sqrt((m[0] ** 2 + m[1] ** 2) / 2)
                assert abs(float(G[t]) - Gw) <= 6e-8 * Gw
                qb, sb = _brute_row(xf[t], G[t], None if g is None else g.float().numpy())
                assert np.array_equal(q[t], qb) and np.array_equal(s[t], sb), (p, t)
