"""Full-size periodic workload (10^6 beads, minimum image, cell list): the GPU
evaluates the whole box; the oracle checks sampled atoms exactly on a local
cluster.  The force on atom c depends only on atoms within 2 L r_c of c (an
atom k within L r_c of c needs its own L r_c ball), and its energy eps_c on
atoms within L r_c, so the oracle runs non-periodically on the ball of radius
2 L r_c around c, unwrapped by the minimum image."""
import numpy as np
import pytest
import torch

import oracle
from _helpers import oracle_model
from schnet_gnn_molecular_b200 import api, workloads

pytestmark = pytest.mark.gpu

W = workloads.BOX1M


@pytest.fixture(scope="module")
def box_run():
    pos = workloads.positions(W)
    types = workloads.types(W)
    weights = workloads.weights(W, bias_scale=0.05)
    model = api.from_workload(W, weights)
    p = torch.as_tensor(pos, device="cuda")
    t = torch.as_tensor(types, device="cuda")
    model.build_neighbors(p)
    E, F = model.energy_forces(p, t)
    eps = model.atom_energies()
    torch.cuda.synchronize()
    assert model.status() == 0
    rp, col, _ = model.neighbors()
    out = dict(pos=pos, types=types, weights=weights, E=E.cpu().numpy(), F=F.cpu().numpy(),
               eps=eps.cpu().numpy(), E_list=len(col), row_ptr=rp, col=col)
    model.close()
    return out


def _cluster(pos, c, radius):
    d = pos.astype(np.float64) - pos[c].astype(np.float64)
    d -= W.box * np.rint(d / W.box)
    sel = np.flatnonzero((d * d).sum(1) < radius * radius)
    local = np.concatenate([[c], sel[sel != c]])
    return local, pos[c].astype(np.float64) + d[local]


def test_sampled_rows_bit_exact(box_run):
    # 1,000 seeded atoms: each one's row of the full 10^6-bead list against the brute-force
    # definition on the atoms of its (r_c + skin + 1 A) ball, kept in their original (unwrapped)
    # coordinates so the oracle's periodic pair test is the very one the full list uses.  The
    # balls go to the oracle as separate replicas of one call (edges never cross replicas).
    from scipy.spatial import cKDTree
    pos = box_run["pos"]
    rl = W.cutoff + W.skin
    rng = np.random.default_rng(99)
    centres = rng.choice(W.n_atoms, size=1000, replace=False)
    wrapped = np.mod(pos.astype(np.float64), W.box)
    wrapped[wrapped >= W.box] = 0.0
    tree = cKDTree(wrapped, boxsize=W.box)
    balls = [np.asarray(sorted(tree.query_ball_point(wrapped[c], rl + 1.0)), dtype=np.int64) for c in centres]
    balls = [np.concatenate([[c], b[b != c]]) for c, b in zip(centres, balls)]
    ro = np.concatenate([[0], np.cumsum([len(b) for b in balls])]).astype(np.int32)
    sub = pos[np.concatenate(balls)]
    rp_o, col_o = oracle.neighbors(sub, W.cutoff, W.skin, ro, True, (W.box,) * 3)
    rp, col = box_run["row_ptr"], box_run["col"]
    n_checked = 0
    for k, (c, b) in enumerate(zip(centres, balls)):
        first = ro[k]                      # atom c is its ball's first atom
        local = col_o[rp_o[first]:rp_o[first + 1]] - first
        expect = np.sort(b[local])
        got = col[rp[c]:rp[c + 1]]
        assert np.array_equal(got, expect), f"row {c}"
        n_checked += len(got)
    assert n_checked > 1000 * 100


def test_edge_count_matches_density(box_run):
    # listed directed edges: N * rho * 4/3 pi (r_c + skin)^3 within a few percent
    expect = W.n_atoms * 0.01 * 4.0 / 3.0 * np.pi * (W.cutoff + W.skin) ** 3
    assert abs(box_run["E_list"] / expect - 1.0) < 0.05


def test_net_force_vanishes(box_run):
    F = box_run["F"].astype(np.float64)
    assert np.abs(F.sum(0)).max() <= 1e-5 * np.abs(F).sum(0).max()


@pytest.mark.parametrize("c", [0, 777_777])
def test_sampled_atoms_against_oracle(box_run, c):
    m = oracle_model(W.with_(periodic=False), box_run["weights"])
    local, x = _cluster(box_run["pos"], c, 2 * W.L * W.cutoff)
    _, eps_o, F_o = oracle.energy_forces(m, x, box_run["types"][local])
    F_gpu = box_run["F"][c].astype(np.float64)
    assert np.linalg.norm(F_gpu - F_o[0]) <= 1e-4 * np.linalg.norm(F_o[0]) + 1e-6
    assert abs(box_run["eps"][c] - eps_o[0]) <= 1e-5 * max(abs(eps_o[0]), 1e-2)
