"""Cell-list edge cases of the neighbour build, bit-exact against the brute-force
float64 definition (neighbour inclusion d^2 < (r_c + skin)^2; Tessera abstract,
"conservative neighbour skin").

* Grids at the rounding edge: boxes (periodic) and replica extents (open
  boundaries) whose cells are exactly r_c + skin wide, or the smallest float32
  width above the library's (r_c + skin)(1 + 2^-20) threshold, with pairs at
  distances just inside and just outside r_c + skin straddling every cell face,
  the periodic wrap included.  A pair binned two cells apart would be missing.
* Periodic grids of one, two and three cells along an axis (boxes between
  2 (r_c + skin) and 4 (r_c + skin)), where the 27-cell stencil must visit each
  cell once by its absolute index.
Energies and forces on the small periodic boxes are checked against the oracle
too, so the minimum image is exercised with so few cells."""
import zlib

import numpy as np
import pytest
import torch

import oracle
from _helpers import (CELL_MARGIN, FORCE_RTOL, check_energies, face_straddling_pairs, fp32_above, oracle_model,
                      random_box_positions, rel_frobenius)
from schnet_gnn_molecular_b200 import api, workloads

pytestmark = pytest.mark.gpu

BOXW = workloads.BOX1M      # r_c = 12, skin = 2, F = 128, K = 50, L = 3, 10 types
RL = BOXW.cutoff + BOXW.skin


def _model(n, box3, periodic=True, ro=None, bias_scale=0.0):
    weights = workloads.weights(BOXW, bias_scale=bias_scale)
    ro = [0, n] if ro is None else ro
    m = api.SchNet(n_types=BOXW.n_types, F=BOXW.F, K=BOXW.K, L=BOXW.L, rbf_min=BOXW.rbf_min,
                   rbf_max=BOXW.rbf_max, rbf_sigma=BOXW.rbf_sigma, cutoff=BOXW.cutoff, skin=BOXW.skin,
                   replica_offsets=ro, weights=weights, periodic=periodic,
                   box=box3 if periodic else (0.0, 0.0, 0.0))
    return m, weights


def _check_list(pos, box3, periodic=True, ro=None):
    n = len(pos)
    model, _ = _model(n, box3, periodic, ro)
    model.build_neighbors(torch.as_tensor(pos, device="cuda"))
    rp, col, rev = model.neighbors()
    assert model.status() == 0
    model.close()
    rp_o, col_o = oracle.neighbors(pos, BOXW.cutoff, BOXW.skin, ro, periodic, box3)
    assert np.array_equal(rp, rp_o)
    assert np.array_equal(col, col_o)
    rows = np.repeat(np.arange(n), np.diff(rp))
    assert np.all(rev >= 0) and np.array_equal(col[rev], rows) and np.array_equal(rev[rev], np.arange(len(col)))
    return len(col)


def _periodic_edge_cases():
    at = fp32_above(4 * RL * CELL_MARGIN)          # 4 cells, each just wider than the threshold
    cases = {
        "cells_just_above_threshold": ((at,) * 3, [(4, 4, 4)]),
        "box_exactly_4rl": ((4 * RL,) * 3, [(4, 4, 4), (3, 3, 3)]),   # 3 cells now; 4 exact ones before
        "box_exactly_2rl": ((2 * RL,) * 3, [(2, 2, 2), (1, 1, 1)]),   # one cell per axis
        "two_cells_per_axis": ((2.5 * RL,) * 3, [(2, 2, 2)]),
        "one_two_three_cells": ((2 * RL, 2.5 * RL, 3.25 * RL), [(1, 2, 3), (2, 3, 4)]),
        "mixed_exact": ((3 * RL, fp32_above(3 * RL * CELL_MARGIN), 5 * RL), [(3, 3, 5), (2, 3, 4)]),
    }
    return cases


@pytest.mark.parametrize("name", list(_periodic_edge_cases()))
def test_periodic_grid_edges_bit_exact(name):
    box3, grids = _periodic_edge_cases()[name]
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    parts = [face_straddling_pairs(box3, g, RL, rng, periodic=True) for g in grids]
    parts.append(random_box_positions(150, box3, rng, min_dist=2.0))
    pos = np.concatenate(parts)
    E = _check_list(pos, box3)
    assert E > 0


@pytest.mark.parametrize("extent_kind", ["exact_3rl", "just_above_threshold", "exact_2rl", "seven_cells"])
def test_open_boundary_grid_edges_bit_exact(extent_kind):
    # the faces of the grid the extent suggests (cells exactly r_c + skin wide, or just wider)
    ext = {"exact_3rl": 3 * RL, "just_above_threshold": fp32_above(3 * RL * CELL_MARGIN), "exact_2rl": 2 * RL,
           "seven_cells": fp32_above(7 * RL * CELL_MARGIN)}[extent_kind]
    ncell = {"exact_3rl": 3, "just_above_threshold": 3, "exact_2rl": 2, "seven_cells": 7}[extent_kind]
    rng = np.random.default_rng(17 + ncell)
    reps = []
    for r in range(3):   # three replicas (edges never cross replicas), bounding boxes [-ext/2, ext/2]
        org = np.array([-0.5 * ext, 0.25 * r, -0.5 * ext])   # x and z extents exactly ext in float32
        extent = (ext, ext * 0.5 + 1.0, ext)
        grid = (ncell, max(1, ncell // 2), ncell)
        p = face_straddling_pairs(extent, grid, RL, rng, periodic=False, origin=org)
        anchors = np.array([org, org + np.asarray(extent)], dtype=np.float32)   # pin the bounding box
        reps.append(np.concatenate([anchors, p]))
    ro = np.concatenate([[0], np.cumsum([len(p) for p in reps])]).astype(np.int32)
    pos = np.concatenate(reps)
    assert float(pos[1, 0]) - float(pos[0, 0]) == float(np.float32(ext))
    assert float(pos[1, 2]) - float(pos[0, 2]) == float(np.float32(ext))
    E = _check_list(pos, (0.0, 0.0, 0.0), periodic=False, ro=ro)
    assert E > 0


@pytest.mark.parametrize("box3", [(2 * RL,) * 3, (2.5 * RL,) * 3, (2 * RL, 2.5 * RL, 3.25 * RL)],
                         ids=["one_cell", "two_cells", "one_two_three"])
def test_energy_forces_small_periodic_boxes(box3):
    rng = np.random.default_rng(7)
    n = int(0.01 * np.prod(box3))
    pos = random_box_positions(n, box3, rng)
    types = rng.integers(0, BOXW.n_types, size=n).astype(np.int32)
    model, weights = _model(n, box3, bias_scale=0.1)
    p, t = torch.as_tensor(pos, device="cuda"), torch.as_tensor(types, device="cuda")
    model.build_neighbors(p)
    E, F = model.energy_forces(p, t)
    torch.cuda.synchronize()
    assert model.status() == 0
    model.close()
    m = oracle.Model(n_types=BOXW.n_types, F=BOXW.F, K=BOXW.K, L=BOXW.L, rbf_min=BOXW.rbf_min,
                     rbf_max=BOXW.rbf_max, rbf_sigma=BOXW.rbf_sigma, cutoff=BOXW.cutoff, weights=weights,
                     periodic=True, box=box3)
    Eo, eps_o, Fo = oracle.energy_forces(m, pos.astype(np.float64), types)
    check_energies(E.cpu().numpy(), Eo, eps_o, label=f"periodic box {box3}")
    assert rel_frobenius(F.cpu().numpy(), Fo) <= FORCE_RTOL
