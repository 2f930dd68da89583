"""Fit of the cubic behind the FMA-pipe 2^x of the bf16 prefill kernel.

The prefill kernel computes one exponent pair in sixteen on the FMA pipe
instead of the SFU (device_common.cuh, exp2_poly_pair): x = n + f with
n = round(x) and f in [-1/2, 1/2], 2^x = 2^n * p(f), where p is a cubic
minimising the squared *relative* error (p(f) - 2^f) / 2^f over the 64
Chebyshev nodes f_k = cos((2k + 1) pi / 128) / 2 of [-1/2, 1/2] (ordinary
weighted least squares, weights 2^-f_k).  Running this file prints the four
coefficients (constant term first) as float32 values and the cubic's maximum
relative error on [-1/2, 1/2]; tests/test_exp2_cubic.py checks that they are
the ones in the kernel source and that the bound holds.
"""
from __future__ import annotations

import numpy as np

NODES = 64


def fit() -> np.ndarray:
    """Coefficients c0..c3 (float64) of the relative-error least-squares cubic."""
    k = np.arange(NODES)
    f = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * NODES))
    w = 2.0 ** -f
    a = np.vander(f, 4, increasing=True) * w[:, None]
    c, *_ = np.linalg.lstsq(a, (2.0 ** f) * w, rcond=None)
    return c


def max_rel_error(c: np.ndarray, n: int = 200001) -> float:
    """Maximum of |p(f) / 2^f - 1| over a fine grid of [-1/2, 1/2], p evaluated in fp64."""
    f = np.linspace(-0.5, 0.5, n)
    p = c[0] + f * (c[1] + f * (c[2] + f * c[3]))
    return float(np.max(np.abs(p / 2.0 ** f - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("coefficients (c0 + c1 f + c2 f^2 + c3 f^3), float32:", [repr(float(np.float32(x))) for x in c])
    print("max relative error on [-1/2, 1/2]: %.3g" % max_rel_error(c.astype(np.float32).astype(np.float64)))
