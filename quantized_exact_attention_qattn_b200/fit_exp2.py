"""Coefficients of the FMA-pipe exp2 polynomial used by the attention kernel.

2^x = 2^n * 2^f with n = round(x), f = x - n in [-1/2, 1/2]; 2^f is a
polynomial of degree DEG in f evaluated by Horner's rule in FP32.  The
coefficients minimise the maximum RELATIVE error on [-1/2, 1/2] (Lawson's
re-weighted least squares on Chebyshev nodes, float64), then are rounded to
FP32.  Running this module prints the C initialisers and the
measured FP32 error; the kernel's constants were produced by it.

    python -m quantized_exact_attention_qattn_b200.fit_exp2 [DEG]
"""
from __future__ import annotations

import sys

import numpy as np


def fit(deg: int, iters: int = 400):
    """Relative-minimax fit of 2^f on [-1/2, 1/2] (float64) by Lawson's
    iteratively re-weighted least squares, which converges to the minimax
    solution of a linear approximation problem."""
    x = 0.5 * np.cos(np.pi * (np.arange(4001) + 0.5) / 4001)      # Chebyshev nodes
    y = np.exp2(x)
    V = np.vander(x, deg + 1, increasing=True) / y[:, None]        # relative residual
    w = np.full(x.size, 1.0 / x.size)
    coef = None
    for _ in range(iters):
        sw = np.sqrt(w)
        coef, *_ = np.linalg.lstsq(V * sw[:, None], sw, rcond=None)
        err = np.abs(V @ coef - 1.0)
        w = w * err
        w /= w.sum()
    return coef


def fp32_error(c32: np.ndarray) -> float:
    """Max relative error of FP32 Horner evaluation against float64 2^f."""
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    acc = np.full_like(f, c32[-1])
    for cj in c32[-2::-1]:
        acc = (acc * f + cj).astype(np.float32)   # FMA rounding is at least this good
    return float(np.max(np.abs(acc.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


def main(argv):
    deg = int(argv[1]) if len(argv) > 1 else 4
    c = fit(deg)
    c32 = c.astype(np.float32)
    print(f"// degree {deg}, max relative error in FP32: {fp32_error(c32):.3e}")
    print("{" + ", ".join(f"{float(v):.9e}f" for v in c32) + "}")


if __name__ == "__main__":
    main(sys.argv)
