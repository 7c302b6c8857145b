"""Shared comparison helpers for the GPU parity tests and the smoke check.

Tolerances (the numeric contract):
* G: within 1e-6 relative of the oracle's long-double p-mean (exact for
  p = inf, where G is a maximum).
* E8M0 scales and E4M3 / E2M1 codes (nearest-even and stochastic): bit-exact against
  the oracle re-run with the kernel's own G bits (two-stage parity: the kernel
  and the oracle add the p-mean terms in different orders, so the fp32 G may
  differ in its last bits; given the same G every later step is a sequence of
  correctly rounded fp32 operations and exact integer rules).
* Strict (always run): against the oracle's own G.  For p = 1, 2, 4 and
  infinity the kernel's G is the p-mean rounded once to fp32, so E8M0 scales
  and stochastic-rounding codes must equal the oracle's own; a nearest-even
  E4M3 code may differ by one step only where the oracle's pre-rounding value
  lies within 1e-6 relative of the rounding midpoint.  The counts of G bits,
  scales and codes that differ are reported.
* RMSNorm bf16 output: within one bf16 ulp of the double-precision oracle.
* Backward: relative L2 error <= 1e-3 against the float64 oracle rounded to
  the output type (bf16).  The outputs are bf16, whose rounding alone leaves a
  relative L2 error near 2^-7 ln2 / sqrt(12) ~ 1.6e-3 against unrounded values;
  the tolerance bounds the arithmetic, not the output format.
"""
import math

import numpy as np
import torch

import oracle

G_RTOL = 1e-6
BWD_RTOL_L2 = 1e-3


def to_np_u8(t):
    return t.detach().cpu().contiguous().numpy().view(np.uint8)


# p values for which the kernel's G is the definition's p-mean rounded once
# to fp32 (terms and sums exact in double, a correctly rounded root): there
# the scales and codes must equal the oracle's own, not only the oracle's
# re-run from the kernel's G.
EXACT_P = (1.0, 2.0, 4.0, math.inf)


def _e4m3_magnitude(code):
    return oracle.e4m3_value(int(code) & 0x7F)


def _strict_e4m3_boundary(x_cpu, g_cpu, G_own, s_own, q_own, qh, rows_np, bad):
    """The allowance of the numeric contract for an E4M3 code that differs from
    the oracle's own result: the two codes are one grid step apart with the same
    sign, and the oracle's pre-rounding value v = y * 2^-e (y = fl(fl(x * s) *
    gamma), s = fl(1 / G), all fp32, from the oracle's own G) lies within 1e-6
    relative of the rounding midpoint between their grid values."""
    D = x_cpu.shape[1]
    xs = x_cpu.float().numpy()
    gs = None if g_cpu is None else g_cpu.float().numpy()
    for i, c in zip(*np.nonzero(bad)):
        a, b = int(q_own[i, c]), int(qh[i, c])
        assert (a ^ b) & 0x80 == 0, f"code sign differs at row {rows_np[i]} col {c}"
        assert abs((a & 0x7F) - (b & 0x7F)) == 1, f"codes {a:#x} / {b:#x} are more than one step apart"
        G = np.float32(G_own[i])
        sc = np.float32(0.0) if G == 0 else np.float32(1.0) / G
        y = np.float32(np.float32(xs[rows_np[i], c]) * sc)
        if gs is not None:
            y = np.float32(y * np.float32(gs[c]))
        e = int(s_own[i, c // 32]) - 127
        v = abs(float(y)) * 2.0 ** (-e)
        mid = 0.5 * (_e4m3_magnitude(a) + _e4m3_magnitude(b))
        assert abs(v - mid) <= 1e-6 * mid, (
            f"row {rows_np[i]} col {c}: codes differ but v = {v!r} is not within 1e-6 of the midpoint {mid!r}")
    assert D % 32 == 0


def check_mxnorm_fwd(x_dev, g_dev, p, rounding, seed, q, s, G, rows=None,
                     stat="absmax", fmt="e4m3"):
    """Parity of an mxnorm_fwd(_ex) result with the oracle; returns a report dict.

    (i) G within G_RTOL of the oracle's p-mean.  (ii) Two-stage: scales and
    codes bit-exact against the oracle re-run from the kernel's own G bits.
    (iii) Strict: against the oracle's own G.  For p in EXACT_P the scales and
    the stochastic-rounding codes must be equal; a nearest-even code may differ
    only by one step where its pre-rounding value lies within 1e-6 of the
    rounding midpoint (checked for E4M3; FP4 codes must be equal).  For other p
    (fp32 powf in the kernel) scales and codes may differ only in rows whose G
    differs.  The counts are returned."""
    x_cpu = x_dev.cpu()
    g_cpu = None if g_dev is None else g_dev.cpu()
    T = x_cpu.shape[0]
    rows_np = np.arange(T) if rows is None else np.asarray(rows, np.int64)
    p_used = float(np.float32(p))          # the C ABI takes p as fp32
    qh = to_np_u8(q)[rows_np]
    sh = to_np_u8(s)[rows_np]
    Gh = G.detach().cpu().numpy()[rows_np]
    q_own, s_own, G_ref = oracle.mxnorm_fwd_ex(x_cpu, g_cpu, p_used, rows=rows_np, rounding=rounding, seed=seed,
                                               stat=stat, fmt=fmt)
    # stage (i): the statistic
    G_ref64 = G_ref.astype(np.float64)
    if np.isinf(p):
        assert np.array_equal(Gh, G_ref), "G must equal the row max for p = inf"
        g_rel = 0.0
    else:
        rel = np.abs(Gh.astype(np.float64) - G_ref64) / np.where(G_ref64 > 0, G_ref64, 1.0)
        g_rel = float(rel.max()) if rel.size else 0.0
        assert g_rel <= G_RTOL, f"G relative error {g_rel:.3e} > {G_RTOL}"
    # stage (ii): codes and scales from the kernel's G
    q_ref, s_ref, _ = oracle.mxnorm_fwd_ex(x_cpu, g_cpu, p_used, rows=rows_np, G_in=Gh, rounding=rounding,
                                           seed=seed, stat=stat, fmt=fmt)
    bad_s = np.count_nonzero(s_ref != sh)
    bad_q = np.count_nonzero(q_ref != qh)
    assert bad_s == 0, f"{bad_s} E8M0 scales differ"
    assert bad_q == 0, f"{bad_q} {fmt} code bytes differ"
    # stage (iii): against the oracle's own G
    g_bad = Gh.view(np.uint32) != G_ref.astype(np.float32).view(np.uint32)
    s_bad = s_own != sh
    q_bad = q_own != qh
    if p in EXACT_P:
        assert not s_bad.any(), f"{np.count_nonzero(s_bad)} scales differ from the oracle's own"
        if rounding != 0 or fmt != "e4m3":
            assert not q_bad.any(), f"{np.count_nonzero(q_bad)} codes differ from the oracle's own"
        elif q_bad.any():
            _strict_e4m3_boundary(x_cpu, g_cpu, G_ref, s_own, q_own, qh, rows_np, q_bad)
    else:
        assert not (s_bad.any(axis=1) & ~g_bad).any(), "scales differ in a row with equal G"
        assert not (q_bad.any(axis=1) & ~g_bad).any(), "codes differ in a row with equal G"
    return {"rows": int(rows_np.size), "G_max_rel": g_rel,
            "strict_G_bit_mismatch_rows": int(np.count_nonzero(g_bad)),
            "strict_scale_mismatch": int(np.count_nonzero(s_bad)),
            "strict_code_mismatch": int(np.count_nonzero(q_bad))}


def check_cast(x_dev, rounding, seed, q, s, gain_dev=None, fmt="e4m3"):
    g = None if gain_dev is None else gain_dev.cpu()
    q_ref, s_ref = oracle.mx_cast(x_dev.cpu(), g, rounding=rounding, seed=seed, fmt=fmt)
    assert np.array_equal(to_np_u8(s), s_ref), "E8M0 scales differ"
    assert np.array_equal(to_np_u8(q), q_ref), f"{fmt} codes differ"


def bf16_ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 steps between two arrays of bf16 bit patterns."""
    def ordered(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    return np.abs(ordered(a_bits) - ordered(b_bits))


def round_bf16(a):
    """float64 array -> float64 values of the nearest bf16 (for tolerance metrics)."""
    return torch.from_numpy(np.ascontiguousarray(a, np.float64)).to(torch.bfloat16).double().numpy()


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def bf16_bits(a):
    """float64 values -> bit patterns (uint16) of their nearest bf16."""
    t = torch.from_numpy(np.ascontiguousarray(a, np.float64)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def check_bwd_elementwise(out_bf16, ref64, axis_scale):
    """Element-wise bound for a bf16 backward output against the float64 oracle:
    each element is within one bf16 step of the oracle rounded to bf16, or (where
    the fp32 sum g - x (x.g)/(x.x) cancels to a value far below its row's size)
    within 2^-16 of the row's root-mean-square of the oracle's values.  fp32
    arithmetic errs by ~2^-24 of the operands, so 2^-16 leaves a factor of 256.
    axis_scale: the axis over which the root-mean-square is taken (1: per row of
    dx; None: over all of dgamma).  Returns (max bf16 steps, elements that
    needed the absolute bound)."""
    got = out_bf16.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    ref = np.asarray(ref64, np.float64)
    steps = bf16_ulp_distance(got, bf16_bits(ref))
    if axis_scale is None:
        rms = np.sqrt(np.mean(ref * ref))
    else:
        rms = np.sqrt(np.mean(ref * ref, axis=axis_scale, keepdims=True))
    gotf = out_bf16.detach().cpu().double().numpy()
    small = np.abs(gotf - ref) <= 2.0 ** -16 * rms
    bad = (steps > 1) & ~small
    assert not bad.any(), (f"{np.count_nonzero(bad)} elements beyond one bf16 step and 2^-16 of the rms; "
                           f"worst {steps[bad].max()} steps")
    return int(steps.max()) if steps.size else 0, int(np.count_nonzero((steps > 1) & small))


def mma_scale_offset(row, k, kp4):
    """Byte offset of scale (row, k) in the tcgen05 128x4 block-scale layout."""
    return ((row // 128) * (kp4 // 4) + k // 4) * 512 + (row % 32) * 16 + ((row % 128) // 32) * 4 + (k % 4)
