"""Shared helpers for the parity tests: oracle models built from the same seeded
inputs the CUDA path gets, and the error measures the tolerances refer to."""
from __future__ import annotations

import numpy as np

import oracle
from oracle import quant
from schnet_gnn_molecular_b200 import workloads

ENERGY_RTOL = 1e-5          # float32 / tensor-core path vs float64 oracle, per replica
FORCE_RTOL = 1e-4           # relative Frobenius error of all forces
FORCE_RTOL_16BIT = 2e-3     # 16-bit filter weights vs the fp32 oracle
FORCE_RTOL_DEQUANT = 1e-4   # 16-bit filter weights vs the oracle on the same dequantized weights
ENERGY_RTOL_16BIT = 2e-3    # fp16 fast mode (16-bit weights and filter activations) vs the fp32 oracle


def oracle_model(w: workloads.Workload, weights: dict, dequant: str | None = None) -> oracle.Model:
    ww = quant.dequantized_weights(weights, dequant) if dequant else weights
    return oracle.Model(n_types=w.n_types, F=w.F, K=w.K, L=w.L, rbf_min=w.rbf_min, rbf_max=w.rbf_max,
                        rbf_sigma=w.rbf_sigma, cutoff=w.cutoff, weights=ww, periodic=w.periodic,
                        box=(w.box,) * 3 if w.periodic else (0.0, 0.0, 0.0))


def rel_frobenius(a, b) -> float:
    a = np.asarray(a, dtype=np.float64); b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def energy_rel(e_gpu, e_ref, eps_ref=None, replica_offsets=None) -> float:
    """max over replicas of |dE_r| / scale_r with scale_r = max(|E_r|, sum_{i in r} |eps_i|).

    A replica energy is a sum of per-atom terms of both signs; when they cancel,
    |E_r| says nothing about the precision of the sum, so the summands'
    magnitude is the floor of the scale (without eps_ref the scale is |E_r|)."""
    e_gpu = np.asarray(e_gpu, dtype=np.float64); e_ref = np.asarray(e_ref, dtype=np.float64)
    scale = np.abs(e_ref)
    if eps_ref is not None:
        eps_ref = np.abs(np.asarray(eps_ref, dtype=np.float64))
        ro = np.asarray(replica_offsets if replica_offsets is not None else [0, len(eps_ref)])
        mag = np.array([eps_ref[ro[r]:ro[r + 1]].sum() for r in range(len(ro) - 1)])
        scale = np.maximum(scale, mag)
    return float(np.max(np.abs(e_gpu - e_ref) / np.maximum(scale, 1e-12)))


def sorted_rows(row_ptr, col):
    return [np.sort(col[row_ptr[i]:row_ptr[i + 1]]) for i in range(len(row_ptr) - 1)]
