"""CPU: the seeded synthetic inputs follow the recipe the workloads state
(self-avoiding chains with 3.8 A bonds and 3.0 A clash distance; compact chains
confined to the sphere of a uniform fill with R_g = 12 A and accepted inside the
R_g window; random sequential addition in a periodic box with a 3.0 A
minimum-image distance; Xavier-uniform weights; uniform bead types)."""
import math

import numpy as np
from scipy.spatial import cKDTree

from schnet_gnn_molecular_b200 import inputs, workloads


def _min_nonbonded(p):
    d = np.sqrt(((p[:, None, :] - p[None, :, :]) ** 2).sum(-1))
    n = len(p)
    mask = np.abs(np.arange(n)[:, None] - np.arange(n)[None, :]) > 1
    return d[mask].min()


def test_chain_bonds_and_clash_distance():
    p = inputs.chain(200, np.random.default_rng(0))
    bonds = np.linalg.norm(np.diff(p, axis=0), axis=1)
    assert np.allclose(bonds, 3.8, atol=1e-9)
    assert _min_nonbonded(p) >= 3.0


def test_compact_chain_window_and_confinement():
    rng = np.random.default_rng(1000)
    p = inputs.compact_chain(269, rng)
    rg = inputs.radius_of_gyration(p)
    assert 11.5 <= rg <= 12.5
    assert np.allclose(np.linalg.norm(np.diff(p, axis=0), axis=1), 3.8, atol=1e-9)
    assert _min_nonbonded(p) >= 3.0
    # centred on its mean; the walk stayed inside the sphere of radius sqrt(5/3) * 12 about its origin,
    # so every bead lies within twice that radius of the centroid
    assert np.allclose(p.mean(0), 0.0, atol=1e-9)
    assert np.max(np.linalg.norm(p, axis=1)) <= 2 * math.sqrt(5.0 / 3.0) * 12.0


def test_bench_workload_replicas_are_compact_chains():
    w = workloads.PROTEIN64.with_(n_replicas=3)
    pos = workloads.positions(w).astype(np.float64)
    for r in range(3):
        p = pos[r * w.beads:(r + 1) * w.beads]
        assert 11.5 <= inputs.radius_of_gyration(p) <= 12.5


def test_periodic_box_minimum_image_distance():
    box = 40.0
    p = inputs.periodic_box(600, box, np.random.default_rng(4), min_dist=3.0)
    assert p.shape == (600, 3) and np.all(p >= 0.0) and np.all(p < box)
    dd, _ = cKDTree(p, boxsize=box).query(p, k=2)
    assert dd[:, 1].min() >= 3.0


def test_box_workload_density():
    w = workloads.BOX1M
    assert abs(w.n_atoms / w.box ** 3 - 0.01) < 1e-9


def test_xavier_bounds_and_types():
    rng = np.random.default_rng(7)
    W = inputs.xavier(rng, 128, 64)
    a = math.sqrt(6.0 / (128 + 64))
    assert W.dtype == np.float32 and np.abs(W).max() <= a and np.abs(W).max() > 0.9 * a
    assert abs(float(W.mean())) < 0.01 and abs(float(W.var()) - a * a / 3) < 0.05 * a * a
    t = inputs.bead_types(100_000, 25, rng)
    assert t.dtype == np.int32 and t.min() == 0 and t.max() == 24
    counts = np.bincount(t, minlength=25)
    assert np.all(np.abs(counts - 4000) < 5 * math.sqrt(4000))
