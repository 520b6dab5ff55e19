"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle's tests.

This module draws geometries, bead types, weights and raw normal deviates.  It
holds none of the method's arithmetic (no distances-to-energies, no filters, no
integrator): every number it returns is an *input* to the path.

Geometry recipes (coarse-grained beads, Angstrom):
  * ``chain``         -- 3D random walk, fixed bond length, a step is rejected if
                         the new bead comes closer than ``min_dist`` to any bead.
  * ``compact_chain`` -- the same walk confined to a sphere of radius R, with
                         backtracking when stuck; kept only if its radius of
                         gyration falls in ``rg_range`` (a uniform sphere has
                         R_g = sqrt(3/5) R).
  * ``periodic_box``  -- random sequential addition in a cubic box with a
                         minimum pair distance under the minimum image.
Weights are Xavier-uniform U(+-sqrt(6 / (fan_in + fan_out))) in float32.
"""
from __future__ import annotations

import math

import numpy as np


def _unit_vectors(rng: np.random.Generator, m: int) -> np.ndarray:
    v = rng.normal(size=(m, 3))
    v /= np.linalg.norm(v, axis=1, keepdims=True)
    return v


def chain(n: int, rng: np.random.Generator, bond: float = 3.8, min_dist: float = 3.0,
          confine_radius: float | None = None, batch: int = 64) -> np.ndarray:
    """Self-avoiding random walk of n beads (float64 [n,3]); optional confinement.

    The clash test of a candidate against beads 0..t-2 only visits beads in grid
    cells (edge min_dist) near bead t-1; beads outside are farther than min_dist
    from every candidate, so the accepted walk is the same as an all-pairs test."""
    pos = np.zeros((n, 3))
    if n == 0:
        return pos
    md2 = min_dist * min_dist
    cell = min_dist
    grid: dict = {}

    def add(k):
        key = tuple(np.floor(pos[k] / cell).astype(np.int64))
        grid.setdefault(key, []).append(k)

    reach = int(math.ceil((bond + min_dist) / cell)) + 1
    offs = np.arange(-reach, reach + 1)
    add(0)
    t = 1
    stuck = 0
    while t < n:
        cand = pos[t - 1] + bond * _unit_vectors(rng, batch)
        ok = np.ones(batch, dtype=bool)
        if confine_radius is not None:
            ok &= (cand * cand).sum(1) <= confine_radius * confine_radius
        if t > 1:
            c0 = np.floor(pos[t - 1] / cell).astype(np.int64)
            near = []
            for dx in offs:
                for dy in offs:
                    for dz in offs:
                        near.extend(grid.get((c0[0] + dx, c0[1] + dy, c0[2] + dz), ()))
            if near:
                idx = np.unique(np.asarray(near, dtype=np.int64))
                idx = idx[idx < t - 1]
                if idx.size:
                    d2 = ((cand[:, None, :] - pos[None, idx, :]) ** 2).sum(-1)
                    ok &= (d2 >= md2).all(1)
        acc = np.flatnonzero(ok)
        if acc.size:
            pos[t] = cand[acc[0]]
            add(t)
            t += 1
            stuck = 0
        else:
            stuck += 1
            if stuck >= 8:                      # back off a few beads and retry
                t = max(1, t - 1 - int(rng.integers(1, 6)))
                stuck = 0
    return pos


def radius_of_gyration(pos: np.ndarray) -> float:
    c = pos - pos.mean(0)
    return float(np.sqrt((c * c).sum(1).mean()))


def compact_chain(n: int, rng: np.random.Generator, rg_target: float = 12.0, rg_tol: float = 0.5,
                  bond: float = 3.8, min_dist: float = 3.0, radius: float | None = None,
                  max_tries: int = 200) -> np.ndarray:
    """Walk confined to a sphere sized so that a uniform fill has R_g = rg_target.

    The sphere radius is sqrt(5/3) * rg_target (for n beads built "the same way"
    at other sizes pass ``radius`` scaled by (n/n_ref)^(1/3)).  Retries until
    R_g lies in [rg_target - rg_tol, rg_target + rg_tol]."""
    R = math.sqrt(5.0 / 3.0) * rg_target if radius is None else radius
    for _ in range(max_tries):
        p = chain(n, rng, bond, min_dist, confine_radius=R)
        rg = radius_of_gyration(p)
        if abs(rg - rg_target) <= rg_tol:
            return p - p.mean(0)
    raise RuntimeError("compact_chain: radius-of-gyration window not reached")


def periodic_box(n: int, box: float, rng: np.random.Generator, min_dist: float = 3.0) -> np.ndarray:
    """Random sequential addition of n points in [0, box)^3 with a minimum-image
    minimum pair distance (batched: candidates clashing with accepted points or
    with earlier candidates of the same batch are dropped)."""
    from scipy.spatial import cKDTree

    acc = np.zeros((0, 3))
    while acc.shape[0] < n:
        need = n - acc.shape[0]
        cand = rng.uniform(0.0, box, size=(int(need * 1.3) + 64, 3))
        if acc.shape[0]:
            tree = cKDTree(acc, boxsize=box)
            dd, _ = tree.query(cand, k=1, distance_upper_bound=min_dist)
            cand = cand[~np.isfinite(dd) | (dd >= min_dist)]
        if cand.shape[0] == 0:
            continue
        ct = cKDTree(cand, boxsize=box)
        pairs = ct.query_pairs(min_dist, output_type="ndarray")
        bad = np.zeros(cand.shape[0], dtype=bool)
        if pairs.size:
            # sequential order: drop the later member of each clashing pair
            bad[np.maximum(pairs[:, 0], pairs[:, 1])] = True
        cand = cand[~bad]
        acc = np.concatenate([acc, cand[:need]], axis=0)
    return acc[:n]


def bead_types(n: int, n_types: int, rng: np.random.Generator) -> np.ndarray:
    return rng.integers(0, n_types, size=n).astype(np.int32)


def xavier(rng: np.random.Generator, fan_in: int, fan_out: int, shape=None) -> np.ndarray:
    a = math.sqrt(6.0 / (fan_in + fan_out))
    shape = (fan_in, fan_out) if shape is None else shape
    return rng.uniform(-a, a, size=shape).astype(np.float32)


def schnet_weights(rng: np.random.Generator, n_types: int, F: int, K: int, L: int,
                   bias_scale: float = 0.0) -> dict:
    """Xavier-uniform float32 weights, dense layers [in, out]; biases zero unless
    bias_scale > 0 (then U(-bias_scale, bias_scale), used by tests to exercise
    the bias paths)."""
    H = F // 2

    def bias(*shape):
        if bias_scale > 0:
            return rng.uniform(-bias_scale, bias_scale, size=shape).astype(np.float32)
        return np.zeros(shape, np.float32)

    w = {
        "emb": xavier(rng, n_types, F),
        "W_in": np.stack([xavier(rng, F, F) for _ in range(L)]),
        "W1": np.stack([xavier(rng, K, F) for _ in range(L)]),
        "b1": bias(L, F),
        "W2": np.stack([xavier(rng, F, F) for _ in range(L)]),
        "b2": bias(L, F),
        "Wo1": np.stack([xavier(rng, F, F) for _ in range(L)]),
        "bo1": bias(L, F),
        "Wo2": np.stack([xavier(rng, F, F) for _ in range(L)]),
        "bo2": bias(L, F),
        "R1": xavier(rng, F, H),
        "c1": bias(H),
        "R2": xavier(rng, H, 1).reshape(H),
        "c2": float(bias(1)[0]),
    }
    return w


def standard_normals(n: int, rng: np.random.Generator) -> np.ndarray:
    """Raw N(0,1) deviates [n,3] (callers scale them into velocities)."""
    return rng.normal(size=(n, 3))


def random_rotation(rng: np.random.Generator) -> np.ndarray:
    """Uniformly distributed 3x3 rotation matrix (QR of a Gaussian matrix with the
    sign convention that makes the factorisation unique, then det fixed to +1)."""
    q, r = np.linalg.qr(rng.normal(size=(3, 3)))
    q = q * np.sign(np.diag(r))
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q
