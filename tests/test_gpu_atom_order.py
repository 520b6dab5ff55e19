"""GPU: the library holds atoms in cell order between neighbour builds, but every
result it returns is in the caller's order and does not depend on that order.

* Relabelling the atoms inside each replica permutes forces and per-atom
  energies and leaves replica energies unchanged (up to summation order).
* A velocity-Verlet trajectory that rebuilds the list (and so the internal
  order) every other step follows the float64 oracle's trajectory.
"""
import numpy as np
import pytest
import torch

import oracle
from _helpers import ENERGY_RTOL, energy_rel, oracle_model, rel_frobenius
from schnet_gnn_molecular_b200 import api, workloads

pytestmark = pytest.mark.gpu

# 64 cells of >= 14 A: the cell order differs from the input order
PERIODIC_SMALL = workloads.BOX1M.with_(name="periodic_box_3000", beads=3000, box=(3000 / 0.01) ** (1 / 3),
                                       seed=4000)
# 4 replicas of a 2048-bead globule (the others rotated copies of the first): per-replica grids
# of several cells each
GLOBULES = workloads.globule(2048).with_(name="cg_globule_4x2048", n_replicas=4, pool=1)


def _dev(a, dtype=None):
    return torch.as_tensor(np.ascontiguousarray(a), dtype=dtype).cuda()


def _within_replica_permutation(w, rng):
    ro = w.replica_offsets()
    return np.concatenate([ro[r] + rng.permutation(ro[r + 1] - ro[r]) for r in range(w.n_replicas)])


def _eval(model, pos, types):
    p, t = _dev(pos, torch.float32), _dev(types, torch.int32)
    model.build_neighbors(p)
    E, F = model.energy_forces(p, t)
    eps = model.atom_energies()
    rp, col, rev = model.neighbors()
    torch.cuda.synchronize()
    assert model.status() == 0
    return E.cpu().numpy(), F.cpu().numpy(), eps.cpu().numpy(), (rp, col, rev)


@pytest.mark.parametrize("w", [PERIODIC_SMALL, GLOBULES], ids=lambda w: w.name)
def test_relabelling_atoms_permutes_results(w):
    pos, types = workloads.positions(w), workloads.types(w)
    weights = workloads.weights(w, bias_scale=0.1)
    model = api.from_workload(w, weights)
    E0, F0, eps0, (rp0, col0, _) = _eval(model, pos, types)
    perm = _within_replica_permutation(w, np.random.default_rng(11))   # new atom k = old atom perm[k]
    E1, F1, eps1, (rp1, col1, rev1) = _eval(model, pos[perm], types[perm])
    model.close()
    assert rel_frobenius(F1, F0[perm]) <= 1e-6
    assert energy_rel(E1, E0, eps0, w.replica_offsets()) <= 1e-6
    # per-atom energies: the energy tolerance, on the largest per-atom magnitude (float32 sums taken in
    # another order differ by a few 1e-7 of it)
    assert np.max(np.abs(eps1 - eps0[perm])) <= ENERGY_RTOL * np.max(np.abs(eps0))
    # the list of the relabelled system is the relabelled list (rows ascending in the caller's labels)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(len(perm))
    for k in range(0, w.n_atoms, max(1, w.n_atoms // 200)):
        i = perm[k]
        assert np.array_equal(col1[rp1[k]:rp1[k + 1]], np.sort(inv[col0[rp0[i]:rp0[i + 1]]]))
    rows1 = np.repeat(np.arange(w.n_atoms), np.diff(rp1))
    assert np.array_equal(col1[rev1], rows1) and np.array_equal(rows1[rev1], col1)


def test_velocity_verlet_with_rebuilds_follows_the_oracle():
    w = PERIODIC_SMALL
    pos, types = workloads.positions(w), workloads.types(w)
    weights = workloads.weights(w, bias_scale=0.1)
    mass = workloads.masses(w)
    vel = (workloads.velocity_normals(w) * np.sqrt(0.0019872041 * 300 * 4.184e-4 / w.mass)).astype(np.float32)
    model = api.from_workload(w, weights)
    p, v = _dev(pos, torch.float32), _dev(vel, torch.float32)
    n_steps = 6
    epot, ekin, st = model.step(p, v, _dev(types, torch.int32), _dev(mass, torch.float32), n_steps, dt=w.dt_fs,
                                gamma=0.0, n_rebuild=2, seed=5)
    torch.cuda.synchronize()
    model.close()
    m = oracle_model(w, weights)
    x, vo = pos.astype(np.float64), vel.astype(np.float64)
    _, _, Fo = oracle.energy_forces(m, x, types)
    for s in range(n_steps):
        x, vo, Fo, epo, eko = oracle.md_step(m, x, vo, types, mass.astype(np.float64), Fo, w.dt_fs, 0.0, 300.0,
                                             5, s)
    assert np.max(np.abs(p.cpu().numpy() - x)) < 1e-4
    assert rel_frobenius(v.cpu().numpy(), vo) < 1e-4
    assert energy_rel(epot.cpu().numpy(), epo) <= ENERGY_RTOL
    assert abs(ekin.cpu().numpy()[0] / eko[0] - 1) < 1e-4
