"""Shared comparison helpers for the GPU parity tests and the smoke check.

Tolerances (the numeric contract):
* G: within 1e-6 relative of the oracle's long-double p-mean (exact for
  p = inf, where G is a maximum).
* E8M0 scales and E4M3 / E2M1 codes (nearest-even and stochastic): bit-exact against
  the oracle re-run with the kernel's own G bits (two-stage parity: the kernel
  and the oracle add the p-mean terms in different orders, so the fp32 G may
  differ in its last bits; given the same G every later step is a sequence of
  correctly rounded fp32 operations and exact integer rules).
* The strict report also compares with the oracle's own G and counts codes
  that differ; each such code must be one step away and its pre-rounding
  value within 1e-6 relative of a rounding boundary.
* RMSNorm bf16 output: within one bf16 ulp of the double-precision oracle.
* Backward: relative L2 error <= 1e-3 against the float64 oracle rounded to
  the output type (bf16).  The outputs are bf16, whose rounding alone leaves a
  relative L2 error near 2^-7 ln2 / sqrt(12) ~ 1.6e-3 against unrounded values;
  the tolerance bounds the arithmetic, not the output format.
"""
import numpy as np
import torch

import oracle

G_RTOL = 1e-6
BWD_RTOL_L2 = 1e-3


def to_np_u8(t):
    return t.detach().cpu().contiguous().numpy().view(np.uint8)


def check_mxnorm_fwd(x_dev, g_dev, p, rounding, seed, q, s, G, rows=None, strict=True,
                     stat="absmax", fmt="e4m3"):
    """Two-stage parity of an mxnorm_fwd(_ex) result; returns a small report dict."""
    x_cpu = x_dev.cpu()
    g_cpu = None if g_dev is None else g_dev.cpu()
    T = x_cpu.shape[0]
    rows_np = np.arange(T) if rows is None else np.asarray(rows, np.int64)
    qh = to_np_u8(q)[rows_np]
    sh = to_np_u8(s)[rows_np]
    Gh = G.detach().cpu().numpy()[rows_np]
    q_own, s_own, G_ref = oracle.mxnorm_fwd_ex(x_cpu, g_cpu, p, rows=rows_np, rounding=rounding, seed=seed,
                                               stat=stat, fmt=fmt)
    # stage (i): the statistic
    G_ref64 = G_ref.astype(np.float64)
    if np.isinf(p):
        assert np.array_equal(Gh, G_ref), "G must equal the row max for p = inf"
    else:
        rel = np.abs(Gh.astype(np.float64) - G_ref64) / np.where(G_ref64 > 0, G_ref64, 1.0)
        assert rel.max() <= G_RTOL, f"G relative error {rel.max():.3e} > {G_RTOL}"
    # stage (ii): codes and scales from the kernel's G
    q_ref, s_ref, _ = oracle.mxnorm_fwd_ex(x_cpu, g_cpu, p, rows=rows_np, G_in=Gh, rounding=rounding,
                                           seed=seed, stat=stat, fmt=fmt)
    bad_s = np.count_nonzero(s_ref != sh)
    bad_q = np.count_nonzero(q_ref != qh)
    assert bad_s == 0, f"{bad_s} E8M0 scales differ"
    assert bad_q == 0, f"{bad_q} {fmt} code bytes differ"
    report = {"rows": int(rows_np.size), "G_max_rel": 0.0 if np.isinf(p) else float(rel.max())}
    if strict:
        report["strict_scale_mismatch"] = int(np.count_nonzero(s_own != sh))
        report["strict_code_mismatch"] = int(np.count_nonzero(q_own != qh))
    return report


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


def mma_scale_offset(row, k, kp4):
    """Byte offset of scale (row, k) in the tcgen05 128x4 block-scale layout."""
    return ((row // 128) * (kp4 // 4) + k // 4) * 512 + (row % 32) * 16 + ((row % 128) // 32) * 4 + (k % 4)
