"""Pins for the float64 oracle: closed forms, hand-computed special cases,
invariances, finite differences, aggregation, neighbour semantics, RNG and
integrator.  None of these re-types the oracle's formulas: each checks the
oracle against something the mathematics (or a library routine) fixes.
"""
import math

import numpy as np
import pytest
from scipy.special import expit

import oracle
from schnet_gnn_molecular_b200 import inputs

LN2 = math.log(2.0)


# ---------------------------------------------------------------------------
# scalar building blocks
# ---------------------------------------------------------------------------

def test_ssp_closed_forms():
    assert oracle.ssp(0.0) == 0.0
    assert oracle.dssp(0.0) == 0.5
    # ssp(ln 3) = ln 2, ssp(ln 2) = ln(3/2): ln((1+e^x)/2)
    assert abs(oracle.ssp(math.log(3.0)) - LN2) < 1e-15
    assert abs(oracle.ssp(LN2) - math.log(1.5)) < 1e-15
    # asymptotes: ssp(x) - x -> -ln 2 (x -> +inf), ssp(x) -> -ln 2 (x -> -inf)
    assert abs(oracle.ssp(60.0) - 60.0 + LN2) < 1e-12
    assert abs(oracle.ssp(-60.0) + LN2) < 1e-12
    xs = np.linspace(-30, 30, 241)
    ref = np.logaddexp(0.0, xs) - LN2            # library routine
    got = np.array([oracle.ssp(x) for x in xs])
    assert np.max(np.abs(got - ref)) < 1e-14
    dref = expit(xs)                             # library logistic
    dgot = np.array([oracle.dssp(x) for x in xs])
    assert np.max(np.abs(dgot - dref)) < 1e-15


def test_cosine_cutoff_closed_forms():
    rc = 15.0
    assert oracle.fc(0.0, rc) == 1.0
    assert abs(oracle.fc(rc / 2, rc) - 0.5) < 1e-15
    assert abs(oracle.fc(rc / 3, rc) - 0.75) < 1e-15
    assert oracle.fc(rc, rc) == 0.0 and oracle.fc(rc + 1.0, rc) == 0.0
    assert abs(oracle.dfc(rc / 2, rc) + math.pi / (2 * rc)) < 1e-15
    assert oracle.dfc(rc, rc) == 0.0
    assert abs(oracle.dfc(rc * (1 - 1e-9), rc)) < 1e-8     # f_c'(r_c^-) -> 0
    for d in [0.3, 4.1, 9.9, 14.2]:
        h = 1e-6
        fd = (oracle.fc(d + h, rc) - oracle.fc(d - h, rc)) / (2 * h)
        assert abs(fd - oracle.dfc(d, rc)) < 1e-9


def test_gaussian_basis_closed_forms():
    K, rmin, rmax, s = 50, 0.0, 15.0, 0.3
    mus = np.array([oracle.rbf_center(k, K, rmin, rmax) for k in range(K)])
    assert np.allclose(mus, np.linspace(rmin, rmax, K), rtol=0, atol=1e-14)
    for k in [0, 7, 49]:
        e, _ = oracle.rbf(mus[k], K, rmin, rmax, s)
        assert e[k] == 1.0
        e, _ = oracle.rbf(mus[k] + s, K, rmin, rmax, s)
        assert abs(e[k] - math.exp(-0.5)) < 1e-14   # (mu+s)-mu rounds
        e, _ = oracle.rbf(mus[k] - s, K, rmin, rmax, s)
        assert abs(e[k] - math.exp(-0.5)) < 1e-14   # (mu+s)-mu rounds
    d, h = 6.123, 1e-6
    _, de = oracle.rbf(d, K, rmin, rmax, s)
    ep, _ = oracle.rbf(d + h, K, rmin, rmax, s)
    em, _ = oracle.rbf(d - h, K, rmin, rmax, s)
    assert np.max(np.abs((ep - em) / (2 * h) - de)) < 1e-8


# ---------------------------------------------------------------------------
# hand-computed special cases (F = 2, H = 1, T = 1; two atoms at d = r_c / 2)
# ---------------------------------------------------------------------------

def _zeros_model(F=2, K=1, L=1, rmin=0.0, rmax=10.0, sigma=0.3, rc=10.0, T=1):
    H = F // 2
    w = {k: np.zeros(s) for k, s in
         {"emb": (T, F), "W_in": (L, F, F), "W1": (L, K, F), "b1": (L, F), "W2": (L, F, F), "b2": (L, F),
          "Wo1": (L, F, F), "bo1": (L, F), "Wo2": (L, F, F), "bo2": (L, F), "R1": (F, H), "c1": (H,),
          "R2": (H,)}.items()}
    w["c2"] = 0.0
    return oracle.Model(n_types=T, F=F, K=K, L=L, rbf_min=rmin, rbf_max=rmax, rbf_sigma=sigma, cutoff=rc,
                        weights=w)


def _readout_chain(m, layer=0):
    """Weights that carry channel 1 of m through the atom-wise path to the
    energy: x = [1, 0] -> h = [0, 1]; q_0 = m_1; v_1 = ssp(q_0); eps = ssp(x_1).
    Every matrix is asymmetric, so a transposed [in,out] convention breaks it."""
    w = m.weights
    w["emb"][0] = [1.0, 0.0]
    w["W_in"][layer] = [[0.0, 1.0], [0.0, 0.0]]     # h_1 = x_0
    w["Wo1"][layer] = [[0.0, 0.0], [1.0, 0.0]]      # q_0 = m_1
    w["Wo2"][layer] = [[0.0, 1.0], [0.0, 0.0]]      # v_1 = a_0
    w["R1"][:] = [[0.0], [1.0]]                     # pr = x_1
    w["R2"][:] = [1.0]


def _pair(d):
    return np.array([[0.0, 0.0, 0.0], [d * 0.6, d * 0.8, 0.0]])


def test_hand_case_filter_bias_path():
    # W1 = b1 = 0 -> a = ssp(0) = 0, so W = f_c(d) b2; b2_1 = 2 ln 3, f_c = 1/2:
    # q_0 = ln 3, x_1 = ssp(ln 3) = ln 2, eps = ssp(ln 2) = ln 1.5 per atom.
    m = _zeros_model(rc=10.0)
    _readout_chain(m)
    m.weights["W2"][0] = [[5.0, -3.0], [2.0, 7.0]]   # multiplied by a = 0
    m.weights["b2"][0] = [0.7, 2 * math.log(3.0)]
    pos = _pair(5.0)
    E, eps, F = oracle.energy_forces(m, pos, [0, 0])
    assert abs(E[0] - 2 * math.log(1.5)) < 1e-14
    # dE/dd = 2 ssp'(ln 2) ssp'(ln 3) b2_1 f_c'(r_c/2) = -pi ln3 / r_c
    dEdd = -math.pi * math.log(3.0) / 10.0
    unit = (pos[1] - pos[0]) / 5.0
    assert np.allclose(F[1], -dEdd * unit, rtol=0, atol=1e-14)
    assert np.allclose(F[0], dEdd * unit, rtol=0, atol=1e-14)


def test_hand_case_first_filter_layer_and_centres():
    # K = 2 centres at 1.0 and 2.6; only W1 row k=1 is nonzero: p_0 = g e_1(d).
    # At d = 2.6 + sigma = 2.9, e_1 = e^{-1/2}; g = ln 3 e^{1/2} -> p_0 = ln 3,
    # a_0 = ln 2; W2 moves a_0 to channel 1: W_1 = f_c ln 2 = (ln 2)/2 (r_c = 5.8).
    # x_1 = ssp(ln sqrt2) = ln((1+sqrt2)/2); eps = ln((3+sqrt2)/4).
    m = _zeros_model(K=2, rmin=1.0, rmax=2.6, sigma=0.3, rc=5.8)
    _readout_chain(m)
    g = math.log(3.0) * math.exp(0.5)
    m.weights["W1"][0] = [[0.0, 0.0], [g, 0.0]]
    m.weights["W2"][0] = [[0.0, 1.0], [0.0, 0.0]]
    E, _, _ = oracle.energy_forces(m, _pair(2.9), [0, 0])
    assert abs(E[0] - 2 * math.log((3 + math.sqrt(2.0)) / 4)) < 1e-14


def test_hand_case_filter_hidden_bias():
    # b1_0 = ln 3 with W1 = 0: a = [ln 2, 0]; same energy as the case above.
    m = _zeros_model(rc=10.0)
    _readout_chain(m)
    m.weights["b1"][0] = [math.log(3.0), 0.0]
    m.weights["W2"][0] = [[0.0, 1.0], [0.0, 0.0]]
    E, _, _ = oracle.energy_forces(m, _pair(5.0), [0, 0])
    assert abs(E[0] - 2 * math.log((3 + math.sqrt(2.0)) / 4)) < 1e-14


def test_hand_case_atomwise_biases():
    # zero filter (m = 0): q = bo1 = [ln 3, 0] -> a_o = [ln 2, 0]; v = a_o Wo2 + bo2
    # with bo2 = [0, ln 2] -> x = [1, ln 4]; c1 = ln(3/2) -> pr = ln 6;
    # eps = ssp(ln 6) + c2 = ln 3.5 + 1; no position dependence, zero forces.
    m = _zeros_model(rc=10.0)
    _readout_chain(m)
    m.weights["bo1"][0] = [math.log(3.0), 0.0]
    m.weights["bo2"][0] = [0.0, LN2]
    m.weights["c1"][:] = [math.log(1.5)]
    m.weights["c2"] = 1.0
    E, _, F = oracle.energy_forces(m, _pair(5.0), [0, 0])
    assert abs(E[0] - 2 * (math.log(3.5) + 1.0)) < 1e-14
    assert np.all(F == 0.0)


@pytest.mark.parametrize("active", [0, 1])
def test_hand_case_layer_indexing(active):
    # L = 2; one layer carries the case-A weights, the other is all-zero (an
    # all-zero interaction leaves x unchanged).  Both orders give 2 ln 1.5.
    m = _zeros_model(L=2, rc=10.0)
    _readout_chain(m, layer=active)
    m.weights["b2"][active] = [0.0, 2 * math.log(3.0)]
    E, _, _ = oracle.energy_forces(m, _pair(5.0), [0, 0])
    assert abs(E[0] - 2 * math.log(1.5)) < 1e-14


# ---------------------------------------------------------------------------
# invariances and finite differences on a random small system
# ---------------------------------------------------------------------------

def _random_model(seed=0, F=8, K=6, L=2, T=3, rc=8.0, bias=0.3, periodic=False, box=(0, 0, 0)):
    rng = np.random.default_rng(seed)
    w = inputs.schnet_weights(rng, T, F, K, L, bias_scale=bias)
    # larger-than-Xavier weights so every path carries signal
    for k in ["W1", "W2", "Wo1", "Wo2", "W_in"]:
        w[k] = w[k] * 3.0
    return oracle.Model(n_types=T, F=F, K=K, L=L, rbf_min=0.0, rbf_max=rc, rbf_sigma=0.6, cutoff=rc,
                        weights=w, periodic=periodic, box=box)


def _small_system(seed=1, n=24):
    rng = np.random.default_rng(seed)
    pos = inputs.chain(n, rng)
    pos = pos - pos.mean(0)
    types = inputs.bead_types(n, 3, rng)
    return pos, types


def test_invariances_rotation_translation_permutation():
    from scipy.spatial.transform import Rotation

    m = _random_model()
    pos, types = _small_system()
    E0, eps0, F0 = oracle.energy_forces(m, pos, types)
    assert abs(E0[0]) > 1e-3
    Rm = Rotation.random(random_state=3).as_matrix()
    E1, _, F1 = oracle.energy_forces(m, pos @ Rm.T + np.array([3.1, -7.2, 0.4]), types)
    assert abs(E1[0] - E0[0]) <= 1e-12 * abs(E0[0])
    assert np.max(np.abs(F1 - F0 @ Rm.T)) <= 1e-12 * np.max(np.abs(F0))
    perm = np.random.default_rng(5).permutation(len(types))
    E2, eps2, F2 = oracle.energy_forces(m, pos[perm], types[perm])
    assert abs(E2[0] - E0[0]) <= 1e-12 * abs(E0[0])
    assert np.max(np.abs(F2 - F0[perm])) <= 1e-12 * np.max(np.abs(F0))
    assert np.max(np.abs(eps2 - eps0[perm])) <= 1e-12 * np.max(np.abs(eps0))


def test_forces_match_central_differences():
    m = _random_model()
    pos, types = _small_system()
    _, _, F = oracle.energy_forces(m, pos, types)
    h = 1e-5
    fd = np.zeros_like(pos)
    for i in range(pos.shape[0]):
        for c in range(3):
            p = pos.copy(); p[i, c] += h
            Ep, _, _ = oracle.energy_forces(m, p, types, forces=False)
            p[i, c] -= 2 * h
            Em, _, _ = oracle.energy_forces(m, p, types, forces=False)
            fd[i, c] = -(Ep[0] - Em[0]) / (2 * h)
    rel = np.linalg.norm(F - fd) / np.linalg.norm(F)
    assert rel <= 1e-6, rel


def test_zero_net_force_and_torque():
    m = _random_model(seed=7)
    pos, types = _small_system(seed=8, n=30)
    _, _, F = oracle.energy_forces(m, pos, types)
    scale = np.abs(F).max()
    assert np.abs(F.sum(0)).max() <= 1e-12 * scale * len(F)
    assert np.abs(np.cross(pos, F).sum(0)).max() <= 1e-11 * scale * len(F) * np.abs(pos).max()


def test_replicas_are_independent():
    m = _random_model(seed=2)
    pa, ta = _small_system(seed=11, n=20)
    pb, tb = _small_system(seed=12, n=17)
    Ea, _, Fa = oracle.energy_forces(m, pa, ta)
    Eb, _, Fb = oracle.energy_forces(m, pb, tb)
    # overlapping in space, but separate replicas: no cross edges
    E, _, F = oracle.energy_forces(m, np.concatenate([pa, pb]), np.concatenate([ta, tb]),
                                   replica_offsets=[0, 20, 37])
    assert abs(E[0] - Ea[0]) < 1e-13 * abs(Ea[0]) and abs(E[1] - Eb[0]) < 1e-13 * abs(Eb[0])
    assert np.allclose(F, np.concatenate([Fa, Fb]), rtol=0, atol=1e-13)


def test_isolated_atoms_are_additive():
    m = _random_model(seed=4)
    types = np.array([0, 1, 2, 1], dtype=np.int32)
    far = np.array([[0, 0, 0], [100, 0, 0], [0, 100, 0], [0, 0, 100.0]])
    E, eps, F = oracle.energy_forces(m, far, types)
    singles = [oracle.energy_forces(m, far[i:i + 1], types[i:i + 1])[0][0] for i in range(4)]
    assert abs(E[0] - sum(singles)) < 1e-13
    assert np.all(F == 0.0)
    assert abs(eps[1] - eps[3]) == 0.0       # same type, same environment


def test_zero_filter_gives_position_independent_energy():
    m = _random_model(seed=9)
    m.weights["W2"] = m.weights["W2"] * 0.0
    m.weights["b2"] = m.weights["b2"] * 0.0
    pos, types = _small_system(seed=10)
    E, _, F = oracle.energy_forces(m, pos, types)
    far = pos * 50.0
    E2, _, _ = oracle.energy_forces(m, far, types)
    assert abs(E[0] - E2[0]) < 1e-13 * abs(E[0])
    assert np.all(F == 0.0)


def test_periodic_image_shift_and_net_force():
    box = (14.0, 15.0, 16.0)
    m = _random_model(seed=3, rc=6.0, periodic=True, box=box)
    rng = np.random.default_rng(21)
    pos = np.concatenate([inputs.periodic_box(40, 14.0, rng, min_dist=2.0)[:, :1],
                          rng.uniform(0, 15.0, (40, 1)), rng.uniform(0, 16.0, (40, 1))], axis=1)
    types = inputs.bead_types(40, 3, rng)
    E, eps, F = oracle.energy_forces(m, pos, types)
    shifted = pos.copy()
    shifted[3] += [14.0, -15.0, 32.0]
    E2, eps2, F2 = oracle.energy_forces(m, shifted, types)
    assert abs(E2[0] - E[0]) < 1e-12 * abs(E[0])
    assert np.max(np.abs(F2 - F)) < 1e-11 * np.abs(F).max()
    assert np.abs(F.sum(0)).max() < 1e-11 * np.abs(F).max() * 40


def test_filter_derivative_matches_finite_difference():
    m = _random_model(seed=6)
    for d in [0.8, 3.3, 7.9]:
        W, dW = oracle.filter_(m, 1, d)
        h = 1e-6
        Wp, _ = oracle.filter_(m, 1, d + h)
        Wm, _ = oracle.filter_(m, 1, d - h)
        assert np.max(np.abs((Wp - Wm) / (2 * h) - dW)) < 1e-7 * max(1.0, np.abs(dW).max())


# ---------------------------------------------------------------------------
# aggregation: CSR segment sum == naive scatter sum
# ---------------------------------------------------------------------------

def test_csr_segment_sum_equals_scatter_sum():
    m = _random_model(seed=12, F=8)
    pos, _ = _small_system(seed=13, n=40)
    h = np.random.default_rng(14).normal(size=(40, 8))
    seg = oracle.cfconv(m, 1, pos, h)
    row, col, d = oracle.cut_edges(m, pos)
    assert len(row) > 40
    msg = np.stack([oracle.filter_(m, 1, dd)[0] for dd in d]) * h[col]
    scat = np.zeros_like(h)
    np.add.at(scat, row, msg)      # scatter-add in edge order
    assert np.max(np.abs(seg - scat)) <= 1e-14 * np.abs(scat).max() * 8


# ---------------------------------------------------------------------------
# neighbour list semantics
# ---------------------------------------------------------------------------

def test_neighbor_inclusion_is_strict_and_exact():
    x = np.array([0.0, 16.999, 17.001, 40.0, 57.0], dtype=np.float32)
    pos = np.stack([x, np.zeros(5, np.float32), np.zeros(5, np.float32)], 1)
    rp, col = oracle.neighbors(pos, 15.0, 2.0)
    rows = [sorted(col[rp[i]:rp[i + 1]].tolist()) for i in range(5)]
    # (0,1): 16.999 < 17 in; (0,2): 17.001 out; (1,2): 0.002 in; (3,4): exactly 17.0 out
    assert rows == [[1], [0, 2], [1], [], []]


def test_neighbor_periodic_and_replicas():
    pos = np.array([[0.5, 1, 1], [29.5, 1, 1], [0.5, 1, 1], [29.5, 1, 1]], dtype=np.float32)
    rp, col = oracle.neighbors(pos, 15.0, 2.0, replica_offsets=[0, 2, 4], periodic=True, box=(30, 30, 30))
    assert rp.tolist() == [0, 1, 2, 3, 4] and col.tolist() == [1, 0, 3, 2]
    rp, col = oracle.neighbors(pos[:2], 0.5, 0.4, periodic=True, box=(30, 30, 30))
    assert rp.tolist() == [0, 0, 0]           # image distance 1.0 >= 0.9


def test_neighbor_list_matches_kdtree():
    from scipy.spatial import cKDTree

    rng = np.random.default_rng(30)
    pos = inputs.periodic_box(600, 40.0, rng, min_dist=1.0).astype(np.float32)
    for periodic in [False, True]:
        rp, col = oracle.neighbors(pos, 5.0, 1.0, periodic=periodic, box=(40, 40, 40))
        t = cKDTree(pos.astype(np.float64), boxsize=40.0 if periodic else None)
        pairs = t.query_pairs(6.0, output_type="ndarray")
        ref = set(map(tuple, pairs.tolist())) | set((b, a) for a, b in pairs.tolist())
        got = set((i, int(j)) for i in range(600) for j in col[rp[i]:rp[i + 1]])
        assert got == ref
        for i in range(600):
            r = col[rp[i]:rp[i + 1]]
            assert np.all(np.diff(r) > 0)


# ---------------------------------------------------------------------------
# random numbers
# ---------------------------------------------------------------------------

def _kat():
    import os
    rows = []
    with open(os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([int(t, 16) for t in line.split()])
    return rows


def test_philox_known_answers():
    for r in _kat():
        assert oracle.philox4x32_10(r[0:4], r[4:6]).tolist() == r[6:10]


def test_normals_moments_and_stream_separation():
    xi = oracle.noise(12345, 7, 40000).ravel()
    n = xi.size
    assert abs(xi.mean()) < 4.0 / math.sqrt(n)
    assert abs(xi.var() - 1.0) < 4.0 * math.sqrt(2.0 / n)
    assert abs((xi ** 4).mean() - 3.0) < 0.1
    xi2 = oracle.noise(12345, 8, 40000).ravel()
    assert abs(np.corrcoef(xi, xi2)[0, 1]) < 4.0 / math.sqrt(n)


# ---------------------------------------------------------------------------
# integrator
# ---------------------------------------------------------------------------

def test_unit_conversion_matches_codata():
    from scipy import constants as sc

    acc = 4184.0 / sc.N_A / 1e-10 / sc.atomic_mass * 1e10 * 1e-30   # (kcal/mol/A)/amu in A/fs^2
    v = oracle.b_kick(np.zeros((1, 3)), np.ones((1, 3)), np.ones(1), 2.0)
    assert abs(v[0, 0] / acc - 1.0) < 1e-6


def test_ornstein_uhlenbeck_step_is_exact_in_distribution():
    from scipy import constants as sc

    kB = sc.R / 4184.0          # kcal/mol/K
    acc = 4184.0 / sc.N_A / sc.atomic_mass * 1e-10     # (kcal/mol)/amu in A^2/fs^2
    n, dt, gamma, T, mass = 5, 4.0, 0.1, 300.0, 12.0
    xi = np.random.default_rng(0).normal(size=(n, 3))
    pos, vel = oracle.baoa(np.zeros((n, 3)), np.zeros((n, 3)), np.zeros((n, 3)), np.full(n, mass), dt, gamma,
                           T, xi)
    c1 = math.exp(-gamma * 1e-3 * dt)
    expect = math.sqrt((1 - c1 * c1) * kB * T * acc / mass) * xi
    assert np.max(np.abs(vel / expect - 1.0)) < 1e-6
    assert np.allclose(pos, 0.5 * dt * vel, rtol=1e-15, atol=0)


def test_free_flight_is_exact():
    rng = np.random.default_rng(1)
    p0, v0 = rng.normal(size=(4, 3)), rng.normal(size=(4, 3)) * 0.01
    p, v = p0, v0
    for _ in range(100):
        p, v = oracle.baoa(p, v, np.zeros((4, 3)), np.full(4, 12.0), 2.0, 0.0, 300.0)
        v = oracle.b_kick(v, np.zeros((4, 3)), np.full(4, 12.0), 2.0)
    assert np.allclose(p, p0 + 200.0 * v0, rtol=0, atol=1e-12)
    assert np.array_equal(v, v0)


def test_velocity_verlet_harmonic_shadow_energy():
    # For x'' = -w^2 x, velocity Verlet exactly conserves
    # H~ = v^2 + w^2 x^2 (1 - (w dt)^2 / 4)  (a textbook property of the map).
    acc, mass, k, dt = 4.184e-4, 12.0, 3.0, 1.0
    w2 = k * acc / mass
    x = np.array([[1.3, -0.4, 0.2]]); v = np.array([[0.0, 0.01, -0.02]])
    H0 = (v ** 2).sum() + w2 * (x ** 2).sum() * (1 - w2 * dt * dt / 4)
    for _ in range(2000):
        x, v = oracle.baoa(x, v, -k * x, np.array([mass]), dt, 0.0, 0.0)
        v = oracle.b_kick(v, -k * x, np.array([mass]), dt)
    H = (v ** 2).sum() + w2 * (x ** 2).sum() * (1 - w2 * dt * dt / 4)
    assert abs(H / H0 - 1.0) < 1e-12


def test_md_step_energy_error_is_second_order():
    # Without friction the step is velocity Verlet: the total-energy error over
    # a fixed time is O(dt^2) and small against the potential's own swing
    # (a wrong force sign or unit would break both).
    rng = np.random.default_rng(31)
    w = inputs.schnet_weights(rng, 3, 8, 6, 2, bias_scale=0.1)
    m = oracle.Model(n_types=3, F=8, K=6, L=2, rbf_min=0.0, rbf_max=8.0, rbf_sigma=0.6, cutoff=8.0, weights=w)
    pos0, types = _small_system(seed=32, n=16)
    mass = np.full(16, 12.0)
    vel0 = np.random.default_rng(33).normal(size=(16, 3)) * 0.01
    _, _, F0 = oracle.energy_forces(m, pos0, types)
    errs = []
    for dt in [1.0, 0.5]:
        pos, vel, F = pos0.copy(), vel0.copy(), F0.copy()
        tot, pot = [], []
        for s in range(int(40 / dt)):
            pos, vel, F, ep, ek = oracle.md_step(m, pos, vel, types, mass, F, dt, 0.0, 0.0, 1, s)
            tot.append(ep[0] + ek[0]); pot.append(ep[0])
        errs.append(np.ptp(tot))
        assert errs[-1] < 1e-3 * np.ptp(pot)
    assert 3.5 < errs[0] / errs[1] < 4.5
