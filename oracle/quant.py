"""Channel-wise 16-bit weight storage, as the oracle reads it -- TEST INFRASTRUCTURE.

FlashSchNet (paper-curation summary), How: the filter-network weights are
stored in 16 bits with a per-channel scale.  Reading taken here: for each
output channel o of a dense weight W[in][out], s_o = max_i |W[i][o]| (1 if the
column is zero), the stored value is round-to-nearest-even(W / s_o) in fp16 or
bf16, and the effective ("dequantized") weight is s_o * stored, in float64.
"""
from __future__ import annotations

import numpy as np


def _round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (8 significant bits), ties to even."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                   # x = m 2^e, 0.5 <= |m| < 1
    q = np.rint(m * 256.0) / 256.0       # 8 significant bits; rint is half-to-even
    return np.ldexp(q, e)


def _round_fp16(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def dequantize(W: np.ndarray, dtype: str) -> np.ndarray:
    """W [..., in, out] -> s_o * RN16(W / s_o), float64."""
    W = np.asarray(W, dtype=np.float64)
    s = np.abs(W).max(axis=-2, keepdims=True)
    s = np.where(s > 0, s, 1.0)
    r = _round_fp16(W / s) if dtype == "fp16" else _round_bf16(W / s)
    return r * s


def dequantized_weights(weights: dict, dtype: str) -> dict:
    """Copy of a weight dict with the filter network's W1 and W2 dequantized."""
    out = dict(weights)
    for k in ("W1", "W2"):
        out[k] = dequantize(weights[k], dtype)
    return out
