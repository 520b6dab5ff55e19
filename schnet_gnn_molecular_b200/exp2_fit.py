"""Coefficients of the polynomial 2^f, f in [-1/2, 1/2], used by ``ex2_fma2`` in
``csrc/common.cuh`` (the exponentials of the forward softplus that run on the FMA
pipe instead of the MUFU).

Method: reweighted least squares (Lawson's iteration) on Chebyshev nodes for
the relative error, which converges towards the minimax polynomial of the
given degree; the result is rounded to float32 and checked by evaluating the
Horner form in float32 on a dense grid.

    python -m schnet_gnn_molecular_b200.exp2_fit      # prints the coefficients and the bound
"""
from __future__ import annotations

import numpy as np

DEGREE = 5


def fit(degree: int = DEGREE, nodes: int = 4000, iterations: int = 200) -> np.ndarray:
    """float32 coefficients c_0 .. c_degree of 2^f ~ sum_j c_j f^j on [-1/2, 1/2]."""
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)
    A = np.vander(f, degree + 1, increasing=True) / np.exp2(f)[:, None]   # relative error rows
    w = np.ones(nodes)
    c = np.zeros(degree + 1)
    for _ in range(iterations):
        c = np.linalg.lstsq(A * w[:, None], w, rcond=None)[0]
        err = np.abs(A @ c - 1.0)
        w = w * (err / err.max()) ** 0.3 + 1e-12
        w /= w.max()
    return c.astype(np.float32)


def horner_f32(c: np.ndarray, f: np.ndarray) -> np.ndarray:
    """The polynomial evaluated as the device does: float32 fused multiply-adds."""
    f = f.astype(np.float32)
    acc = np.full_like(f, c[-1])
    for cj in c[-2::-1]:
        acc = (acc.astype(np.float64) * f + np.float64(cj)).astype(np.float32)
    return acc


def max_rel_error(c: np.ndarray, samples: int = 2_000_001) -> float:
    f = np.linspace(-0.5, 0.5, samples).astype(np.float32)
    return float(np.max(np.abs(horner_f32(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("coefficients c0..c5:", ", ".join(repr(float(x)) for x in c))
    print(f"max relative error (float32 Horner): {max_rel_error(c):.3e}")
