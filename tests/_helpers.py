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


def _replica_scales(e_ref, eps_ref, replica_offsets):
    """(|E_r|, sum_{i in r} |eps_i|) per replica."""
    e_ref = np.asarray(e_ref, dtype=np.float64)
    eps_ref = np.abs(np.asarray(eps_ref, dtype=np.float64))
    ro = np.asarray(replica_offsets if replica_offsets is not None else [0, len(eps_ref)])
    mag = np.array([eps_ref[ro[r]:ro[r + 1]].sum() for r in range(len(ro) - 1)])
    return np.abs(e_ref), mag


def energy_rel(e_gpu, e_ref, eps_ref=None, replica_offsets=None) -> float:
    """max over replicas of |dE_r| / scale_r with scale_r = max(|E_r|, sum_{i in r} |eps_i|).

    A replica energy is a sum of per-atom terms of both signs; when they cancel,
    |E_r| says nothing about the precision of the sum, so the summands'
    magnitude is the floor of the scale (without eps_ref the scale is |E_r|)."""
    e_gpu = np.asarray(e_gpu, dtype=np.float64); e_ref = np.asarray(e_ref, dtype=np.float64)
    scale = np.abs(e_ref)
    if eps_ref is not None:
        scale = np.maximum(*_replica_scales(e_ref, eps_ref, replica_offsets))
    return float(np.max(np.abs(e_gpu - e_ref) / np.maximum(scale, 1e-12)))


def energy_rel_plain(e_gpu, e_ref, eps_ref, replica_offsets=None, cancel=0.1) -> tuple[float, int]:
    """Plain |dE_r| / |E_r|, maximised over the replicas whose energy is not a cancelling sum
    (|E_r| >= cancel * sum |eps_i|); returns (that maximum, how many replicas it covers)."""
    e_gpu = np.asarray(e_gpu, dtype=np.float64); e_ref = np.asarray(e_ref, dtype=np.float64)
    absE, mag = _replica_scales(e_ref, eps_ref, replica_offsets)
    keep = (absE >= cancel * mag) & (absE > 0)
    if not np.any(keep):
        return 0.0, 0
    return float(np.max(np.abs(e_gpu - e_ref)[keep] / absE[keep])), int(keep.sum())


def check_energies(e_gpu, e_ref, eps_ref, replica_offsets=None, rtol=ENERGY_RTOL, label=""):
    """The energy bound: relative rtol per replica against max(|E_r|, sum |eps_i|), and the plain
    relative error |dE_r| / |E_r| within rtol as well wherever |E_r| >= 0.1 sum |eps_i| (the floor
    then matters only for replicas whose per-atom terms cancel).  Prints both measures."""
    floor = energy_rel(e_gpu, e_ref, eps_ref, replica_offsets)
    plain, n = energy_rel_plain(e_gpu, e_ref, eps_ref, replica_offsets)
    n_rep = len(np.atleast_1d(e_ref))
    print(f"[energy {label}] floored {floor:.3e}, plain {plain:.3e} over {n}/{n_rep} replicas")
    assert floor <= rtol, (floor, rtol)
    assert plain <= rtol, (plain, rtol)
    return floor, plain


def sorted_rows(row_ptr, col):
    return [np.sort(col[row_ptr[i]:row_ptr[i + 1]]) for i in range(len(row_ptr) - 1)]


# ---------------------------------------------------------------------------
# neighbour-list edge cases: cell grids at the rounding edge
# ---------------------------------------------------------------------------
CELL_MARGIN = 1.0 + 2.0 ** -20   # the library's documented cell-width margin over r_c + skin


def fp32_above(x: float) -> float:
    """Smallest float32 value >= x."""
    f = np.float32(x)
    return float(f) if float(f) >= x else float(np.nextafter(f, np.float32(np.inf)))


def face_straddling_pairs(extent, n_cells, rl, rng, periodic, origin=(0.0, 0.0, 0.0)):
    """float32 positions of pairs at distance ~ rl (just inside, just outside) that straddle
    every cell face of a grid of n_cells[a] equal cells over [origin, origin + extent) per axis,
    the periodic wrap face included (both unwrapped and wrapped copies), plus pairs crossing
    three faces at a grid corner.  The coordinates not along the pair are random."""
    extent = np.asarray(extent, dtype=np.float64)
    origin = np.asarray(origin, dtype=np.float64)
    pts = []
    gaps = [rl - 1e-3, rl - 1e-5, rl + 1e-5, rl - 0.25]
    splits = [0.5, 0.1, 0.9, 1e-4, 1 - 1e-4]
    for a in range(3):
        w = extent[a] / n_cells[a]
        faces = range(0 if periodic else 1, n_cells[a])
        for k in faces:
            for D in gaps:
                for s in splits:
                    p = origin + rng.uniform(0.0, 1.0, size=3) * extent
                    q = p.copy()
                    f = origin[a] + k * w
                    p[a] = f - s * D
                    q[a] = f + (1 - s) * D
                    pts += [p, q]
                    if periodic and k == 0:          # the same pair wrapped into the box
                        p2 = p.copy(); p2[a] += extent[a]
                        pts += [p2, q]
    diag = np.ones(3) / np.sqrt(3.0)
    for k in range(1, min(n_cells)) if not periodic else range(min(n_cells)):
        corner = origin + k * extent / np.asarray(n_cells)
        for D in gaps:
            for s in splits:
                pts += [corner - s * D * diag, corner + (1 - s) * D * diag]
    return np.asarray(pts, dtype=np.float32)


def random_box_positions(n, box, rng, min_dist=3.0):
    """n float32 points uniform in an orthorhombic box with a minimum-image rejection distance."""
    box = np.asarray(box, dtype=np.float64)
    out = []
    while len(out) < n:
        p = rng.uniform(0.0, 1.0, size=3) * box
        ok = True
        for q in out:
            d = p - q
            d -= box * np.rint(d / box)
            if d @ d < min_dist * min_dist:
                ok = False
                break
        if ok:
            out.append(p)
    return np.asarray(out, dtype=np.float32)
