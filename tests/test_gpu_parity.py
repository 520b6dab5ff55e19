"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on the
same seeded inputs.  Tolerances: neighbour lists bit-exact; energies relative
1e-5 per replica; forces relative Frobenius 1e-4 (16-bit filter weights: 2e-3
against the fp32 oracle, 1e-4 against the oracle on the dequantized weights)."""
import numpy as np
import pytest
import torch

import oracle
from _helpers import (ENERGY_RTOL, ENERGY_RTOL_16BIT, FORCE_RTOL, FORCE_RTOL_16BIT, FORCE_RTOL_DEQUANT,
                      check_energies, energy_rel, oracle_model,
                      rel_frobenius)
from schnet_gnn_molecular_b200 import api, inputs, workloads

pytestmark = pytest.mark.gpu

SMALL_PROTEIN = workloads.PROTEIN64.with_(name="cg_protein_6x269", n_replicas=6, seed=1000)
PERIODIC_SMALL = workloads.BOX1M.with_(name="periodic_box_3000", beads=3000, box=(3000 / 0.01) ** (1 / 3),
                                       seed=4000)
PERIODIC_20K = workloads.BOX1M.with_(name="periodic_box_20000", beads=20000, box=(20000 / 0.01) ** (1 / 3),
                                     seed=4000)


def _dev(a, dtype=None):
    return torch.as_tensor(np.ascontiguousarray(a), dtype=dtype).cuda()


def _setup(w, bias_scale=0.0, weight_dtype=None, seed_offset=0):
    pos = workloads.positions(w)
    types = workloads.types(w)
    weights = workloads.weights(w, bias_scale=bias_scale, seed_offset=seed_offset)
    model = api.from_workload(w, weights, weight_dtype=weight_dtype)
    return pos, types, weights, model


def _gpu_eval(model, pos, types):
    p = _dev(pos, torch.float32)
    t = _dev(types, torch.int32)
    model.build_neighbors(p)
    E, F = model.energy_forces(p, t)
    torch.cuda.synchronize()
    assert model.status() == 0
    return E.cpu().numpy(), F.cpu().numpy()


# ---------------------------------------------------------------------------
# neighbour lists: bit-exact against the brute-force float64 definition
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("w", [workloads.TINY, SMALL_PROTEIN, PERIODIC_SMALL, workloads.PROTEIN64, PERIODIC_20K],
                         ids=lambda w: w.name)
def test_neighbor_list_bit_exact(w):
    pos, types, weights, model = _setup(w)
    model.build_neighbors(_dev(pos, torch.float32))
    rp, col, rev = model.neighbors()
    rp_o, col_o = oracle.neighbors(pos, w.cutoff, w.skin, w.replica_offsets(), w.periodic, (w.box,) * 3)
    assert np.array_equal(rp, rp_o)
    assert np.array_equal(col, col_o)
    rows = np.repeat(np.arange(w.n_atoms), np.diff(rp))
    assert np.all(rev >= 0)
    assert np.array_equal(col[rev], rows) and np.array_equal(rows[rev], col)
    assert np.array_equal(rev[rev], np.arange(len(col)))


# ---------------------------------------------------------------------------
# energies and forces
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("bias_scale", [0.0, 0.2])
def test_energy_forces_tiny_chain(bias_scale):
    w = workloads.TINY
    pos, types, weights, model = _setup(w, bias_scale=bias_scale)
    E, F = _gpu_eval(model, pos, types)
    Eo, eps_o, Fo = oracle.energy_forces(oracle_model(w, weights), pos.astype(np.float64), types)
    check_energies(E, Eo, eps_o, label=f"tiny chain, bias {bias_scale}")
    assert rel_frobenius(F, Fo) <= FORCE_RTOL
    eps = model.atom_energies().cpu().numpy()
    assert np.max(np.abs(eps - eps_o)) <= 1e-5 * np.max(np.abs(eps_o))


def test_energy_forces_multi_replica():
    w = SMALL_PROTEIN
    pos, types, weights, model = _setup(w, bias_scale=0.1)
    E, F = _gpu_eval(model, pos, types)
    ro = w.replica_offsets()
    Eo, eps_o, Fo = oracle.energy_forces(oracle_model(w, weights), pos.astype(np.float64), types, ro)
    check_energies(E, Eo, eps_o, ro, label="6 x 269")
    assert rel_frobenius(F, Fo) <= FORCE_RTOL
    # no net force inside any (isolated) replica
    for r in range(w.n_replicas):
        Fr = F[r * w.beads:(r + 1) * w.beads]
        assert np.abs(Fr.sum(0)).max() <= 1e-4 * np.abs(Fr).max() * np.sqrt(w.beads)


def test_energy_forces_periodic():
    w = PERIODIC_SMALL
    pos, types, weights, model = _setup(w)
    E, F = _gpu_eval(model, pos, types)
    Eo, eps_o, Fo = oracle.energy_forces(oracle_model(w, weights), pos.astype(np.float64), types)
    check_energies(E, Eo, eps_o, label="periodic 3000")
    assert rel_frobenius(F, Fo) <= FORCE_RTOL


def test_energy_only_evaluation():
    # d_forces = NULL runs no backward pass; the energies are those of the full evaluation
    w = SMALL_PROTEIN
    pos, types, weights, model = _setup(w, bias_scale=0.1)
    p, t = _dev(pos, torch.float32), _dev(types, torch.int32)
    model.build_neighbors(p)
    E1, F1 = model.energy_forces(p, t)
    E0, F0 = model.energy_forces(p, t, forces=False)
    E2, F2 = model.energy_forces(p, t)
    torch.cuda.synchronize()
    assert F0 is None and model.status() == 0
    assert torch.equal(E0, E1) and torch.equal(E2, E1) and torch.equal(F2, F1)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_sixteen_bit_filter_weights(dtype):
    w = SMALL_PROTEIN.with_(weight_dtype=dtype)
    pos, types, weights, model = _setup(w)
    E, F = _gpu_eval(model, pos, types)
    x64 = pos.astype(np.float64)
    ro = w.replica_offsets()
    Eq, eps_q, Fq = oracle.energy_forces(oracle_model(w, weights, dequant=dtype), x64, types, ro)
    E32, eps32, F32 = oracle.energy_forces(oracle_model(w, weights), x64, types, w.replica_offsets())
    print(f"[errors {dtype}] energy vs dequantized {energy_rel(E, Eq, eps_q, ro):.3e}, forces vs dequantized "
          f"{rel_frobenius(F, Fq):.3e}, energy vs fp32 weights {energy_rel(E, E32, eps32, ro):.3e}, forces vs "
          f"fp32 weights {rel_frobenius(F, F32):.3e}")
    check_energies(E, Eq, eps_q, ro, label=f"{dtype} vs dequantized")
    assert rel_frobenius(F, Fq) <= FORCE_RTOL_DEQUANT
    assert rel_frobenius(F, F32) <= FORCE_RTOL_16BIT


def test_fp16_fast_mode():
    # fp16 weights and fp16 filter activations (one tensor-core product per K-step):
    # held to the 16-bit force bound against the fp32 oracle, and compared with the
    # oracle on the same dequantized weights (the difference is the activation rounding)
    w = SMALL_PROTEIN.with_(weight_dtype="fp16fast")
    pos, types, weights, model = _setup(w, bias_scale=0.1)
    E, F = _gpu_eval(model, pos, types)
    x64 = pos.astype(np.float64)
    ro = w.replica_offsets()
    Eq, eps_q, Fq = oracle.energy_forces(oracle_model(w, weights, dequant="fp16"), x64, types, ro)
    E32, eps32, F32 = oracle.energy_forces(oracle_model(w, weights), x64, types, ro)
    print(f"[errors fp16fast] energy vs dequantized {energy_rel(E, Eq, eps_q, ro):.3e}, forces vs dequantized "
          f"{rel_frobenius(F, Fq):.3e}, energy vs fp32 weights {energy_rel(E, E32, eps32, ro):.3e}, forces vs "
          f"fp32 weights {rel_frobenius(F, F32):.3e}")
    assert rel_frobenius(F, F32) <= FORCE_RTOL_16BIT
    assert rel_frobenius(F, Fq) <= FORCE_RTOL_16BIT
    check_energies(E, E32, eps32, ro, rtol=ENERGY_RTOL_16BIT, label="fp16fast vs fp32 weights")


@pytest.mark.parametrize("ro", [[0, 1, 3, 13], [0, 0, 1, 3, 13], [0, 1, 1, 3, 13, 13]],
                         ids=["three", "empty_first", "empty_inner_and_last"])
def test_isolated_atoms_and_empty_rows(ro):
    # replicas: a lone bead, two far-apart beads, a short chain, and replicas without atoms
    w = workloads.TINY.with_(n_replicas=len(ro) - 1, beads=1)
    rng = np.random.default_rng(5)
    chain = inputs.chain(10, rng)
    pos = np.concatenate([[[0.0, 0, 0]], [[0.0, 0, 0], [50.0, 0, 0]], chain]).astype(np.float32)
    types = inputs.bead_types(13, w.n_types, rng)
    weights = workloads.weights(workloads.TINY, bias_scale=0.3)
    model = api.SchNet(n_types=w.n_types, F=w.F, K=w.K, L=w.L, rbf_min=w.rbf_min, rbf_max=w.rbf_max,
                       rbf_sigma=w.rbf_sigma, cutoff=w.cutoff, skin=w.skin, replica_offsets=ro, weights=weights)
    E, F = _gpu_eval(model, pos, types)
    m = oracle_model(workloads.TINY, weights)
    Eo, eps_o, Fo = oracle.energy_forces(m, pos.astype(np.float64), types, ro)
    check_energies(E, Eo, eps_o, ro, label="isolated atoms")
    assert np.all(E[np.diff(ro) == 0] == 0.0)
    assert np.all(F[:3] == 0.0)
    assert rel_frobenius(F, Fo) <= FORCE_RTOL


# ---------------------------------------------------------------------------
# integrator
# ---------------------------------------------------------------------------
def test_one_langevin_step_matches_oracle():
    w = workloads.TINY
    pos, types, weights, model = _setup(w)
    mass = workloads.masses(w)
    vel = (workloads.velocity_normals(w) * np.sqrt(0.0019872041 * 300 * 4.184e-4 / w.mass)).astype(np.float32)
    p, v = _dev(pos, torch.float32), _dev(vel, torch.float32)
    epot, ekin, st = model.step(p, v, _dev(types, torch.int32), _dev(mass, torch.float32), 1, dt=w.dt_fs,
                                gamma=w.gamma_per_ps, temperature=w.temperature, n_rebuild=w.n_rebuild, seed=77,
                                step0=5)
    torch.cuda.synchronize()
    m = oracle_model(w, weights)
    x64 = pos.astype(np.float64)
    _, _, F0 = oracle.energy_forces(m, x64, types)
    po, vo, Fo, epo, eko = oracle.md_step(m, x64, vel.astype(np.float64), types, mass.astype(np.float64), F0,
                                          w.dt_fs, w.gamma_per_ps, w.temperature, 77, 5)
    assert np.max(np.abs(p.cpu().numpy() - po)) < 1e-4
    assert rel_frobenius(v.cpu().numpy(), vo) < 1e-4
    assert energy_rel(epot.cpu().numpy(), epo) <= ENERGY_RTOL
    assert abs(ekin.cpu().numpy()[0] / eko[0] - 1) < 1e-4


def test_graph_replay_equals_eager():
    w = SMALL_PROTEIN
    pos, types, weights, model = _setup(w)
    mass = _dev(workloads.masses(w), torch.float32)
    vel0 = (workloads.velocity_normals(w) * 0.005).astype(np.float32)
    t = _dev(types, torch.int32)
    outs = []
    for use_graph in (False, True):
        p, v = _dev(pos, torch.float32), _dev(vel0, torch.float32)
        ep, ek, st = model.step(p, v, t, mass, 40, n_rebuild=10, seed=3, use_graph=use_graph)
        outs.append((p.cpu().numpy(), v.cpu().numpy(), ep.cpu().numpy()))
    assert np.array_equal(outs[0][0], outs[1][0])
    assert np.array_equal(outs[0][1], outs[1][1])
    assert np.array_equal(outs[0][2], outs[1][2])


# ---------------------------------------------------------------------------
# full-size workload, sampled: 64 x 269 replicas on the GPU, whole replicas in the oracle
# ---------------------------------------------------------------------------
def test_protein64_sampled_replicas():
    w = workloads.PROTEIN64
    pos, types, weights, model = _setup(w)
    E, F = _gpu_eval(model, pos, types)
    m = oracle_model(w, weights)
    for r in (0, 37, 63):
        sl = slice(r * w.beads, (r + 1) * w.beads)
        Eo, eps_o, Fo = oracle.energy_forces(m, pos[sl].astype(np.float64), types[sl])
        print(f"[errors fp32 replica {r}] forces {rel_frobenius(F[sl], Fo):.3e}")
        check_energies(E[r:r + 1], Eo, eps_o, label=f"64 x 269 replica {r}")
        assert rel_frobenius(F[sl], Fo) <= FORCE_RTOL


# ---------------------------------------------------------------------------
# Gaussian counts: K = 13 (the last group of 8 partly past K, the groups after it
# zero), K = 64 (no padding at all) and K = 8 (one group)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("K", [8, 13, 64])
def test_energy_forces_gaussian_counts(K):
    w = SMALL_PROTEIN.with_(name=f"cg_protein_6x269_K{K}", K=K)
    pos, types, weights, model = _setup(w, bias_scale=0.1)
    E, F = _gpu_eval(model, pos, types)
    ro = w.replica_offsets()
    Eo, eps_o, Fo = oracle.energy_forces(oracle_model(w, weights), pos.astype(np.float64), types, ro)
    check_energies(E, Eo, eps_o, ro, label=f"6 x 269, K = {K}")
    err = rel_frobenius(F, Fo)
    print(f"[errors K={K}] forces {err:.3e}")
    assert err <= FORCE_RTOL


# ---------------------------------------------------------------------------
# depth: one interaction (its single pair-derivative launch over the half list
# starts the per-edge sums afresh) and four (three launches add to them)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("L", [1, 4])
def test_energy_forces_other_depths(L):
    w = SMALL_PROTEIN.with_(name=f"cg_protein_6x269_L{L}", L=L)
    pos, types, weights, model = _setup(w, bias_scale=0.1)
    E, F = _gpu_eval(model, pos, types)
    ro = w.replica_offsets()
    Eo, eps_o, Fo = oracle.energy_forces(oracle_model(w, weights), pos.astype(np.float64), types, ro)
    check_energies(E, Eo, eps_o, ro, label=f"6 x 269, {L} interactions")
    err = rel_frobenius(F, Fo)
    print(f"[errors L={L}] forces {err:.3e}")
    assert err <= FORCE_RTOL
    # a second evaluation after a few MD steps (the pair sums restart every evaluation)
    mass = _dev(workloads.masses(w), torch.float32)
    p, v = _dev(pos, torch.float32), _dev(workloads.velocity_normals(w) * 0.003, torch.float32)
    t = _dev(types, torch.int32)
    model.step(p, v, t, mass, 5, n_rebuild=5, seed=9)
    x = p.cpu().numpy()
    model.build_neighbors(p)
    E2, F2 = model.energy_forces(p, t)
    torch.cuda.synchronize()
    Eo2, eps_o2, Fo2 = oracle.energy_forces(oracle_model(w, weights), x.astype(np.float64), types, ro)
    check_energies(E2.cpu().numpy(), Eo2, eps_o2, ro, label=f"6 x 269, {L} interactions, after 5 steps")
    assert rel_frobenius(F2.cpu().numpy(), Fo2) <= FORCE_RTOL
