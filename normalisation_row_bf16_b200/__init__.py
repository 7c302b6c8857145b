"""B200-native MXNorm: fused block-absmax p-mean normalisation with MXFP8 cast.

The compute path is the C-ABI library ``libmxnorm_b200.so`` (hand-written
sm_100a CUDA).  ``normalisation_row_bf16_b200.ops`` is the thin binding over it;
it loads the library on first use and raises if the library is missing.  There
is no CPU fallback.
"""

__all__ = ["ops", "synthetic"]
