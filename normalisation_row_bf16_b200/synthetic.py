"""Seeded synthetic inputs shared by the CUDA path, the oracle and the benchmark.

This module only draws random numbers; it holds none of the method's
arithmetic, so both sides of a parity check can take their inputs from it.

The shapes and distributions stand in for the Llama-3 activations the MXNorm
pages train on (gist.science "MXNorm: Reusing MXFP block scales for efficient
tensor normalisation", technical summary section 3): no dataset is read.

Recipes (every tensor is bf16 unless stated, drawn with a torch.Generator
seeded from (seed, tensor tag) so that one tensor does not depend on the size of
another):

* ``normal``      x ~ N(0, 1)
* ``outliers``    x ~ N(0, 1) with round(0.01 * D) channels, picked by a seeded
                  permutation, multiplied by 50 (outlier channels, as the FP8
                  trillion-token article on aibr.jp describes for SwiGLU outputs)
* ``student_t``   x = 0.5 * t(nu = 3), t = Z / sqrt(chi2_3 / 3)
* gamma           bf16(1 + 0.1 * N(0, 1))
* upstream grad   dy ~ N(0, 1e-2) read as standard deviation 0.01
* GEMM weight     W ~ N(0, 0.02) stored as [N, K] (each output column's weights
                  contiguous along the reduction dimension)
"""
from __future__ import annotations

import math

import torch

_TAGS = {"x": 1, "gamma": 2, "dy": 3, "perm": 4, "w": 5, "chi": 6}


def _gen(seed: int, tag: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + _TAGS[tag] * 7_919) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _randn(shape, seed, tag, device, dtype=torch.float32):
    return torch.randn(*shape, generator=_gen(seed, tag, device), device=device, dtype=dtype)


def activations(T: int, D: int, kind: str = "normal", seed: int = 0, device="cpu") -> torch.Tensor:
    """x bf16 [T, D] (row-major, contiguous)."""
    if kind == "normal":
        x = _randn((T, D), seed, "x", device)
    elif kind == "outliers":
        x = _randn((T, D), seed, "x", device)
        n_out = int(round(0.01 * D))
        if n_out > 0:
            perm = torch.randperm(D, generator=_gen(seed, "perm", "cpu"))[:n_out].to(device)
            x[:, perm] *= 50.0
    elif kind == "student_t":
        z = _randn((T, D), seed, "x", device)
        g = _gen(seed, "chi", device)
        chi2 = torch.zeros(T, D, device=device)
        for _ in range(3):
            c = torch.randn(T, D, generator=g, device=device)
            chi2.addcmul_(c, c)
        x = 0.5 * z / torch.sqrt(chi2 / 3.0)
        del z, chi2
    else:
        raise ValueError(f"unknown activation kind {kind!r}")
    return x.to(torch.bfloat16)


def gamma(D: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """gamma bf16 [D] = bf16(1 + 0.1 N(0,1))."""
    return (1.0 + 0.1 * _randn((D,), seed, "gamma", device)).to(torch.bfloat16)


def upstream_grad(T: int, D: int, seed: int = 0, std: float = 1e-2, device="cpu") -> torch.Tensor:
    """dy bf16 [T, D] ~ N(0, std^2)."""
    return (std * _randn((T, D), seed, "dy", device)).to(torch.bfloat16)


def gemm_weight(N: int, K: int, seed: int = 0, std: float = 0.02, device="cpu") -> torch.Tensor:
    """W bf16 stored [N, K]: row n holds the K weights of output column n."""
    return (std * _randn((N, K), seed, "w", device)).to(torch.bfloat16)


# The workloads, by what they are.  Each entry: (T, D, activation kind, p).
WORKLOADS = {
    "tiny_256x1024_normal_p2": dict(T=256, D=1024, kind="normal", p=2.0),
    "llama8b_8192x4096_outliers_p2": dict(T=8192, D=4096, kind="outliers", p=2.0),
    "sweep_16384x2048_student_t": dict(T=16384, D=2048, kind="student_t"),
    "sweep_16384x4096_student_t": dict(T=16384, D=4096, kind="student_t"),
    "sweep_16384x8192_student_t": dict(T=16384, D=8192, kind="student_t"),
    "sweep_16384x16384_student_t": dict(T=16384, D=16384, kind="student_t"),
    "bwd_8192x4096_normal_p2": dict(T=8192, D=4096, kind="normal", p=2.0),
    "gemm_8192x4096x6144_normal_p2": dict(T=8192, D=4096, kind="normal", p=2.0, N=6144),
}

SWEEP_P = (1.0, 2.0, 4.0, math.inf)
