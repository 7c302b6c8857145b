"""Pins for the oracle's MXFP4 and NVFP4 formats, scale-reuse statistic and gain cast.

Each check compares the oracle with something other than itself:

* E2M1 rounding: ml_dtypes' float4_e2m1fn cast (a library routine, nearest-even
  and saturating) on every finite bf16 and on structured fp32 patterns, and a
  brute-force nearest-value search over the eight magnitudes the format has.
* The E8M0 exponent for an element maximum of 6: the closed form
  e = floor(log2 a) - 2 + [mantissa > 1.5] (6 = 1.5 * 2^2) and a direct scan.
* E2M1 stochastic rounding: unbiased, lands on a neighbour, exact threshold.
* MXFP4 rows: scales found by scanning e and codes by ml_dtypes, on rows whose
  y values are computed in numpy float32 (one rounding per operation).
* Scale reuse (the block statistic replaced by the block's power-of-two scale,
  as the MXNorm title reads): a direct evaluation with scipy's power mean,
  the bracket G/max <= G' < 2 G/max, exact 2^t scaling, and rows whose block
  maxima are max * 2^j exactly.
* Gain cast (MXNormLinear's folded weight, MXNorm summary section 2.3): gamma
  of ones gives the plain cast, power-of-two gains only move the scales, and a
  float32 recomputation with torch's float8 cast.
* NVFP4 (E2M1 in blocks of 16 with E4M3 scales, read as having no tensor-wide
  scale): the scale code against a search of torch's float8_e4m3fn grid, whole
  rows against a python recomputation (scipy p-mean over the 16-element block
  maxima, grid search for the scales, ml_dtypes for the codes), 2^t scaling,
  zero blocks, the gain cast and the scale-reuse statistic.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import scipy.stats
import torch

import oracle
from normalisation_row_bf16_b200 import synthetic

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _bf16_all_finite():
    bits = np.arange(65536, dtype=np.uint32)
    exp = (bits >> 7) & 0xFF
    bits = bits[exp != 0xFF]
    return (bits << 16).view(np.float32)


def _fp32_structured(rng):
    """Every setting of mantissa bits 19..22 with sticky fillers below (all
    round / tie cases of a 1-bit mantissa), exponents around the E2M1 range,
    both signs, plus random patterns."""
    hi = np.arange(16, dtype=np.uint32) << 19
    lows = np.array([0, 1, 0x3FFFF, 0x40000, 0x40001, 0x7FFFF], dtype=np.uint32)
    exps = np.arange(100, 140, dtype=np.uint32) << 23
    m = (hi[:, None] | lows[None, :]).reshape(-1)
    pats = (exps[:, None] | m[None, :]).reshape(-1)
    pats = np.concatenate([pats, pats | 0x80000000,
                           rng.integers(0, 2**32, 100_000, dtype=np.uint64).astype(np.uint32)])
    v = pats.view(np.float32)
    return v[np.isfinite(v)]


def _ml_e2m1_codes(v):
    return np.asarray(v, np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


def _brute_e2m1_rne(v):
    a = np.minimum(np.abs(v.astype(np.float64)), 6.0)
    d = np.abs(a[:, None] - E2M1_GRID[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # ties: the even code (codes are the grid indices)
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    idx = np.where(cand.sum(1) > 1, even.argmax(1), cand.argmax(1))
    return (idx | np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def test_e2m1_values_match_ml_dtypes():
    dec = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for c in range(8):
        assert oracle.e2m1_value(c) == dec[c] == E2M1_GRID[c]
    assert np.array_equal(dec[8:], -E2M1_GRID)


def test_e2m1_rne_all_bf16():
    v = _bf16_all_finite()
    got = oracle.e2m1_rne(v)
    assert np.array_equal(got, _ml_e2m1_codes(v))
    assert np.array_equal(got, _brute_e2m1_rne(v))


def test_e2m1_rne_structured_fp32():
    v = _fp32_structured(np.random.default_rng(5))
    got = oracle.e2m1_rne(v)
    assert np.array_equal(got, _ml_e2m1_codes(v))
    assert np.array_equal(got, _brute_e2m1_rne(v))


def test_mx_exponent_for_e2m1_closed_form():
    v = _bf16_all_finite()
    v = v[v > 0]
    got = oracle.mx_exponent(v, 6.0)
    m, E = np.frexp(v.astype(np.float64))           # v = m * 2^E, m in [0.5, 1)
    want = (E - 1) - 2 + (2 * m > 1.5)
    want = np.clip(want, -127, 127)
    assert np.array_equal(got, want)
    # a direct scan on a sample
    for a in (1e-40, 0.1, 1.5, 6.0, 6.000001, 7.0, 12.0, 12.5, 3e38):
        e = next(e for e in range(-127, 128) if a <= 6.0 * 2.0 ** e)
        assert oracle.mx_exponent([a], 6.0)[0] == e
    assert oracle.mx_exponent([0.0], 6.0)[0] == -127
    assert oracle.mx_exponent([np.inf], 6.0)[0] == 128


def test_e2m1_sr_unbiased_and_threshold():
    rng = np.random.default_rng(2)
    for v in (0.3, 0.75, 1.2, 2.5, 3.9, 5.0, -4.4):
        words = rng.integers(0, 2**32, 1 << 16, dtype=np.uint64).astype(np.uint32)
        codes = oracle.e2m1_sr(np.full(words.shape, v, np.float32), words)
        vals = np.array([oracle.e2m1_value(int(c) & 7) for c in range(8)])[codes & 7]
        vals = np.where(codes & 8, -vals, vals)
        a = abs(float(np.float32(v)))
        lo = E2M1_GRID[E2M1_GRID <= a].max()
        hi = E2M1_GRID[E2M1_GRID > a].min()
        assert set(np.unique(np.abs(vals))) <= {lo, hi}
        frac = (a - lo) / (hi - lo)
        assert abs(vals.mean() - float(np.float32(v))) < 5 * (hi - lo) * math.sqrt(frac * (1 - frac) / len(words)) + 1e-12
        # exact threshold: up iff r32 < frac * 2^32
        t = frac * 2.0 ** 32
        for r, up in ((math.ceil(t) - 1, True), (math.ceil(t), False)):
            if 0 <= r < 2 ** 32:
                c = oracle.e2m1_sr(np.array([v], np.float32), np.array([r], np.uint32))[0]
                assert abs(oracle.e2m1_value(int(c) & 7)) == (hi if up else lo)


def _python_mx_row(y, elem_max, enc):
    """Scales by scanning e; codes by `enc` on fl32(y * 2^-e)."""
    K = y.size // 32
    scales, codes = [], []
    for k in range(K):
        blk = y[32 * k:32 * (k + 1)]
        a = float(np.max(np.abs(blk.astype(np.float64))))
        e = next(e for e in range(-127, 128) if a <= elem_max * 2.0 ** e)
        scales.append(e + 127)
        codes.append(enc((blk * np.float32(2.0 ** -e)).astype(np.float32)))
    return np.array(scales, np.uint8), np.concatenate(codes)


def _pack_e2m1(c):
    c = c.astype(np.uint8)
    return (c[0::2] | (c[1::2] << 4)).astype(np.uint8)


@pytest.mark.parametrize("p", [1.0, 2.0, 4.0, math.inf])
def test_mxfp4_rows_vs_python(p):
    T, D = 6, 256
    x = synthetic.activations(T, D, "outliers", seed=11)
    g = synthetic.gamma(D, seed=11)
    q, s, G = oracle.mxnorm_fwd_ex(x, g, p, fmt="e2m1")
    xf = x.float().numpy()
    gf = g.float().numpy()
    for t in range(T):
        m = np.abs(xf[t].reshape(-1, 32).astype(np.float64)).max(1)
        Gw = np.float32(m.max() if math.isinf(p) else scipy.stats.pmean(m, p))
        assert abs(float(G[t]) - float(Gw)) <= 1e-6 * float(Gw)
        sc = np.float32(1.0) / G[t]
        y = ((xf[t] * sc).astype(np.float32) * gf).astype(np.float32)
        sw, cw = _python_mx_row(y, 6.0, _ml_e2m1_codes)
        assert np.array_equal(s[t], sw)
        assert np.array_equal(q[t], _pack_e2m1(cw))
        # no element saturates: |y| * 2^-e <= 6
        assert np.all(np.abs(y.reshape(-1, 32)) <= 6.0 * 2.0 ** (sw.astype(np.int64) - 127)[:, None])


def test_mxfp4_cast_and_sr_consistency():
    T, D = 4, 128
    x = synthetic.activations(T, D, "student_t", seed=3)
    q, s = oracle.mx_cast(x, fmt="e2m1")
    sw = np.stack([_python_mx_row(x.float().numpy()[t], 6.0, _ml_e2m1_codes)[0] for t in range(T)])
    assert np.array_equal(s, sw)
    # SR codes: each element at one of its two neighbours, words from the Philox layout
    qs, ss = oracle.mx_cast(x, fmt="e2m1", rounding=1, seed=9)
    assert np.array_equal(ss, s)
    xf = x.float().numpy()
    for t in range(T):
        for j in range(D):
            e = int(s[t, j // 32]) - 127
            v = np.float32(xf[t, j] * np.float32(2.0 ** -e))
            r = oracle.sr_words(9, [t * D + j])
            want = oracle.e2m1_sr(np.array([v], np.float32), r)[0]
            got = (qs[t, j // 2] >> (4 * (j & 1))) & 0xF
            assert got == want


def _scale_exp_G(m, p, elem_max):
    e = np.array([next(e for e in range(-127, 128) if a <= elem_max * 2.0 ** e) for a in m])
    r = 2.0 ** e
    return r.max() if math.isinf(p) else scipy.stats.pmean(r, p)


@pytest.mark.parametrize("fmt,elem_max", [("e4m3", 448.0), ("e2m1", 6.0)])
@pytest.mark.parametrize("p", [1.0, 2.0, 4.0, math.inf])
def test_scale_reuse_G_direct_and_bracket(fmt, elem_max, p):
    T, D = 8, 512
    x = synthetic.activations(T, D, "student_t", seed=4)
    _, _, Gs = oracle.mxnorm_fwd_ex(x, None, p, stat="scale_exp", fmt=fmt)
    _, _, Ga = oracle.mxnorm_fwd_ex(x, None, p, fmt=fmt)
    xf = x.float().numpy().astype(np.float64)
    for t in range(T):
        m = np.abs(xf[t]).reshape(-1, 32).max(1)
        want = _scale_exp_G(m, p, elem_max)
        assert abs(float(Gs[t]) - want) <= 1e-6 * want
        # 2^e_k in [m_k / max, 2 m_k / max): the p-mean keeps the bracket
        assert Ga[t] / elem_max * (1 - 1e-6) <= Gs[t] < 2 * Ga[t] / elem_max * (1 + 1e-6)


def test_scale_reuse_exact_powers_and_scaling():
    # blocks whose maxima are 448 * 2^j exactly: G' is the p-mean of 2^j
    D = 32 * 6
    js = np.array([0, -1, -3, 2, 0, -5])
    row = np.zeros(D, np.float32)
    for k, j in enumerate(js):
        row[32 * k] = 448.0 * 2.0 ** j
        row[32 * k + 5] = -1.0 * 2.0 ** j
    x = torch.from_numpy(row[None]).to(torch.bfloat16)
    for p in (1.0, 2.0, 4.0):
        _, _, G = oracle.mxnorm_fwd_ex(x, None, p, stat="scale_exp")
        want = scipy.stats.pmean(2.0 ** js, p)
        assert abs(float(G[0]) - want) <= 1e-7 * want
    # 2^t input scaling: G' scales by 2^t exactly, codes and scales unchanged
    x = synthetic.activations(4, 256, "outliers", seed=8)
    q0, s0, G0 = oracle.mxnorm_fwd_ex(x, None, 2.0, stat="scale_exp")
    for t in (-7, 3, 20):
        q1, s1, G1 = oracle.mxnorm_fwd_ex((x.float() * 2.0 ** t).to(torch.bfloat16), None, 2.0,
                                          stat="scale_exp")
        assert np.array_equal(G1, G0 * np.float32(2.0 ** t))
        assert np.array_equal(q1, q0) and np.array_equal(s1, s0)


def test_default_statistic_and_format_are_the_plain_forward():
    x = synthetic.activations(5, 384, "outliers", seed=6)
    g = synthetic.gamma(384, seed=6)
    for rnd in (0, 1):
        a = oracle.mxnorm_fwd(x, g, 2.0, rounding=rnd, seed=3)
        b = oracle.mxnorm_fwd_ex(x, g, 2.0, rounding=rnd, seed=3)
        assert all(np.array_equal(u, v) for u, v in zip(a, b))


def test_gain_cast_pins():
    T, D = 6, 256
    w = synthetic.gemm_weight(T, D, seed=2)
    ones = torch.ones(D, dtype=torch.bfloat16)
    q0, s0 = oracle.mx_cast(w)
    q1, s1 = oracle.mx_cast(w, ones)
    assert np.array_equal(q0, q1) and np.array_equal(s0, s1)
    assert np.array_equal(q0, oracle.mxfp8_cast(w)[0])
    # power-of-two gains are exact: codes unchanged, scale exponents move by t
    t = np.random.default_rng(1).integers(-3, 4, D)
    g2 = torch.from_numpy((2.0 ** t).astype(np.float32)).to(torch.bfloat16)
    q2, s2 = oracle.mx_cast(w, g2)
    wf = w.float().numpy()
    gf = g2.float().numpy()
    for r in range(T):
        y = (wf[r] * gf).astype(np.float32)
        enc = lambda v: torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        sw, cw = _python_mx_row(y, 448.0, enc)
        assert np.array_equal(s2[r], sw) and np.array_equal(q2[r], cw)
    # a general gain: fl32(w * gamma), then the float8 cast of torch
    g = synthetic.gamma(D, seed=5)
    q3, s3 = oracle.mx_cast(w, g)
    gf = g.float().numpy()
    for r in range(T):
        y = (wf[r] * gf).astype(np.float32)
        enc = lambda v: torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        sw, cw = _python_mx_row(y, 448.0, enc)
        assert np.array_equal(s3[r], sw) and np.array_equal(q3[r], cw)


# ---------------------------------------------------------------- NVFP4

E4M3_POS = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def _brute_nvfp4_scale_code(a):
    ok = np.nonzero(6.0 * E4M3_POS >= a)[0]
    return int(ok[0]) if ok.size else 0x7E


def test_nvfp4_scale_code_vs_e4m3_grid():
    rng = np.random.default_rng(7)
    a = np.concatenate([[0.0, 1e-6, 6 * 2.0 ** -9, 6 * 2.0 ** -9 * 1.0001, 6.0, 6.0001, 2688.0, 2689.0, 1e30],
                        np.exp(rng.uniform(np.log(1e-5), np.log(3000.0), 4000))]).astype(np.float32)
    got = oracle.nvfp4_scale_code(a)
    want = np.array([_brute_nvfp4_scale_code(float(v)) for v in a])
    assert np.array_equal(got, want)
    # every grid value times 6 is its own threshold: a = 6 s gives s exactly
    for c in range(1, 127):
        assert oracle.nvfp4_scale_code([np.float32(6.0 * E4M3_POS[c])])[0] == c


def _python_nvfp4_row(y):
    scales, codes = [], []
    for k in range(y.size // 16):
        blk = y[16 * k:16 * (k + 1)]
        a = float(np.max(np.abs(blk.astype(np.float64))))
        c = _brute_nvfp4_scale_code(a)
        scales.append(c)
        if c == 0:
            codes.append(np.zeros(16, np.uint8))
            continue
        inv = np.float32(1.0) / np.float32(E4M3_POS[c])
        codes.append(_ml_e2m1_codes((blk * inv).astype(np.float32)))
    return np.array(scales, np.uint8), _pack_e2m1(np.concatenate(codes))


@pytest.mark.parametrize("p", [1.0, 2.0, 4.0, math.inf])
def test_nvfp4_rows_vs_python(p):
    T, D = 5, 256
    x = synthetic.activations(T, D, "outliers", seed=12)
    g = synthetic.gamma(D, seed=12)
    q, s, G = oracle.mxnorm_fwd_ex(x, g, p, fmt="nvfp4")
    assert q.shape == (T, D // 2) and s.shape == (T, D // 16)
    xf, gf = x.float().numpy(), g.float().numpy()
    for t in range(T):
        m = np.abs(xf[t].reshape(-1, 16).astype(np.float64)).max(1)       # 16-element blocks
        Gw = np.float32(m.max() if math.isinf(p) else scipy.stats.pmean(m, p))
        assert abs(float(G[t]) - float(Gw)) <= 1e-6 * float(Gw)
        y = ((xf[t] * (np.float32(1.0) / G[t])).astype(np.float32) * gf).astype(np.float32)
        sw, qw = _python_nvfp4_row(y)
        assert np.array_equal(s[t], sw) and np.array_equal(q[t], qw)


def test_nvfp4_invariants_and_zero_blocks():
    x = synthetic.activations(4, 128, "student_t", seed=2)
    q0, s0, G0 = oracle.mxnorm_fwd_ex(x, None, 2.0, fmt="nvfp4")
    for t in (-5, 7):
        q1, s1, G1 = oracle.mxnorm_fwd_ex((x.float() * 2.0 ** t).to(torch.bfloat16), None, 2.0, fmt="nvfp4")
        assert np.array_equal(q1, q0) and np.array_equal(s1, s0)
        assert np.array_equal(G1, G0 * np.float32(2.0 ** t))
    z = x.clone()
    z[1, 16:32] = 0
    q, s, _ = oracle.mxnorm_fwd_ex(z, None, 2.0, fmt="nvfp4")
    assert s[1, 1] == 0 and np.all(q[1, 8:16] == 0)
    # the gain cast in NVFP4 is the python row on fl32(x * gain)
    g = synthetic.gamma(128, seed=4)
    qc, sc = oracle.mx_cast(x, g, fmt="nvfp4")
    for r in range(4):
        y = (x.float().numpy()[r] * g.float().numpy()).astype(np.float32)
        sw, qw = _python_nvfp4_row(y)
        assert np.array_equal(sc[r], sw) and np.array_equal(qc[r], qw)


def test_nvfp4_scale_reuse_statistic():
    x = synthetic.activations(3, 256, "outliers", seed=9)
    _, _, G = oracle.mxnorm_fwd_ex(x, None, 2.0, stat="scale_exp", fmt="nvfp4")
    xf = x.float().numpy().astype(np.float64)
    for t in range(3):
        m = np.abs(xf[t]).reshape(-1, 16).max(1)
        sv = np.array([E4M3_POS[_brute_nvfp4_scale_code(a)] for a in m])
        want = scipy.stats.pmean(sv, 2.0)
        assert abs(float(G[t]) - want) <= 1e-6 * want
