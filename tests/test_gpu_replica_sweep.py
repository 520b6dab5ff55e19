"""Replica-sweep workloads against the float64 oracle: single compact globules of
2,048 and 8,192 beads (the only inputs whose per-replica cell grids have several
cells per axis under open boundaries) and batches of 256 and 1,024 replicas of
269 beads (more rows per CTA in the row partition of the tensor-core kernels).
FlashSchNet summary, Achievement 1 / Fig. 1 (throughput and memory across
system sizes) is the motivation; the checks are the suite's tolerances:
neighbour rows bit-exact, energies relative 1e-5 per replica, forces relative
Frobenius 1e-4.  The globules are checked whole (energy, every force, the whole
list); the large batches on whole sampled replicas (replicas are independent)."""
import numpy as np
import pytest
import torch

import oracle
from _helpers import FORCE_RTOL, check_energies, oracle_model, rel_frobenius
from schnet_gnn_molecular_b200 import api, workloads

pytestmark = pytest.mark.gpu


def _run(w, bias_scale=0.05):
    pos = workloads.positions(w)
    types = workloads.types(w)
    weights = workloads.weights(w, bias_scale=bias_scale)
    model = api.from_workload(w, weights)
    p, t = torch.as_tensor(pos, device="cuda"), torch.as_tensor(types, device="cuda")
    model.build_neighbors(p)
    E, F = model.energy_forces(p, t)
    torch.cuda.synchronize()
    assert model.status() == 0
    out = dict(pos=pos, types=types, weights=weights, E=E.cpu().numpy(), F=F.cpu().numpy(),
               list=model.neighbors())
    model.close()
    return out


@pytest.mark.parametrize("beads", [2048, 8192])
def test_globule_whole_against_oracle(beads):
    w = workloads.globule(beads)
    r = _run(w)
    rp, col, rev = r["list"]
    rp_o, col_o = oracle.neighbors(r["pos"], w.cutoff, w.skin)
    assert np.array_equal(rp, rp_o)
    assert np.array_equal(col, col_o)
    Eo, eps_o, Fo = oracle.energy_forces(oracle_model(w, r["weights"]), r["pos"].astype(np.float64), r["types"])
    check_energies(r["E"], Eo, eps_o, label=f"globule {beads}")
    err = rel_frobenius(r["F"], Fo)
    print(f"[errors globule {beads}] forces {err:.3e}, {len(col) / beads:.1f} listed neighbours per bead")
    assert err <= FORCE_RTOL


@pytest.mark.parametrize("n_replicas,sample", [(256, (0, 100, 255)), (1024, (0, 511, 777, 1023))],
                         ids=["256x269", "1024x269"])
def test_replica_batch_sampled_against_oracle(n_replicas, sample):
    w = workloads.sweep(n_replicas)
    r = _run(w)
    rp, col, _ = r["list"]
    m = oracle_model(w, r["weights"])
    for k in sample:
        sl = slice(k * w.beads, (k + 1) * w.beads)
        x = r["pos"][sl]
        rp_o, col_o = oracle.neighbors(x, w.cutoff, w.skin)
        # the replica's rows of the whole list, in local indices
        a, b = rp[k * w.beads], rp[(k + 1) * w.beads]
        assert np.array_equal(rp[sl.start:sl.stop + 1] - a, rp_o)
        assert np.array_equal(col[a:b] - k * w.beads, col_o)
        Eo, eps_o, Fo = oracle.energy_forces(m, x.astype(np.float64), r["types"][sl])
        check_energies(r["E"][k:k + 1], Eo, eps_o, label=f"{n_replicas} x 269 replica {k}")
        err = rel_frobenius(r["F"][sl], Fo)
        print(f"[errors {n_replicas} x 269 replica {k}] forces {err:.3e}")
        assert err <= FORCE_RTOL
