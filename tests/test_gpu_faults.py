"""Failure detection without GPU faults: every fault is made on the host (bad
input, undersized buffer, moved atom) or is a bounded device-side wait that
nothing completes, and must come back as a status, with the context still
usable afterwards."""
import ctypes as C

import numpy as np
import pytest
import torch

from schnet_gnn_molecular_b200 import _native as nat
from schnet_gnn_molecular_b200 import api, workloads

pytestmark = pytest.mark.gpu

W = workloads.PROTEIN64.with_(name="cg_protein_4x269", n_replicas=4)


def _model(**kw):
    return api.from_workload(W, workloads.weights(W), **kw)


def _dev(a, dtype=None):
    return torch.as_tensor(np.ascontiguousarray(a), dtype=dtype).cuda()


def test_capacity_overflow_is_reported_and_recoverable():
    pos = workloads.positions(W)
    small = _model(edge_capacity=1000)          # far below the ~150 neighbours x 1076 beads
    small.build_neighbors(_dev(pos))
    assert small.status() & nat.FLAG_CAPACITY
    with pytest.raises(api.SchNetError) as e:
        small.neighbors()
    assert e.value.status == 3
    ok = _model()
    ok.build_neighbors(_dev(pos))
    assert ok.status() == 0


def test_skin_violation_flag():
    pos = workloads.positions(W)
    types = _dev(workloads.types(W), torch.int32)
    m = _model()
    p = _dev(pos)
    m.build_neighbors(p)
    moved = pos.copy()
    moved[5] += np.array([1.2, 0.0, 0.0], np.float32)   # more than skin / 2 = 1 A
    m.energy_forces(_dev(moved), types)
    assert m.status() & nat.FLAG_SKIN
    m.energy_forces(p, types)
    assert m.status() == 0                                # flags are cleared by reading them


def test_nonfinite_position_flag():
    pos = workloads.positions(W).copy()
    pos[17, 1] = np.nan
    m = _model()
    m.build_neighbors(_dev(pos))
    m.energy_forces(_dev(pos), _dev(workloads.types(W), torch.int32))
    assert m.status() & nat.FLAG_NONFINITE


def test_bad_type_flag():
    types = workloads.types(W).copy()
    types[3] = W.n_types + 4
    m = _model()
    p = _dev(workloads.positions(W))
    m.build_neighbors(p)
    m.energy_forces(p, _dev(types, torch.int32))
    assert m.status() & nat.FLAG_BADTYPE


def test_step_reports_flags_as_status():
    pos = workloads.positions(W)
    m = _model()
    p, v = _dev(pos), torch.zeros((W.n_atoms, 3), device="cuda")
    types = workloads.types(W).copy()
    types[0] = -1
    _, _, st = m.step(p, v, _dev(types, torch.int32), _dev(workloads.masses(W)), 2, raise_on_flag=False)
    assert st == 6   # SCHNET_ERR_BADTYPE


def test_bounded_wait_gives_up_and_context_survives():
    lib = nat.load()
    pos = workloads.positions(W)
    types = workloads.types(W)
    m = _model()
    p, t = _dev(pos), _dev(types, torch.int32)
    m.build_neighbors(p)
    E0, F0 = m.energy_forces(p, t)
    assert m.status() == 0
    # a barrier that completes: the wait succeeds, no flag
    assert lib.schnet_test_timeout(m.ctx, 1000, 1) == 0
    assert m.status() == 0
    # a barrier nothing completes: the wait gives up after its polls and raises TIMEOUT
    assert lib.schnet_test_timeout(m.ctx, 1000, 0) == 0
    assert m.status() == nat.FLAG_TIMEOUT
    assert m.status() == 0                      # the read cleared it
    # the context (and its tensor memory) is still usable: the same results again
    E1, F1 = m.energy_forces(p, t)
    torch.cuda.synchronize()
    assert m.status() == 0
    assert torch.equal(E0, E1) and torch.equal(F0, F1)
    # a step reports a flag raised before it as its status
    assert lib.schnet_test_timeout(m.ctx, 1000, 0) == 0
    v = torch.zeros((W.n_atoms, 3), device="cuda")
    _, _, st = m.step(p, v, t, _dev(workloads.masses(W)), 1, raise_on_flag=False)
    assert st == 8   # SCHNET_ERR_TIMEOUT
    assert lib.schnet_test_timeout(None, 1000, 0) == 1 and lib.schnet_test_timeout(m.ctx, 0, 0) == 1


def test_argument_errors_and_state():
    m = _model()
    lib = nat.load()
    assert lib.schnet_build_neighbors(m.ctx, None) == 1
    p = _dev(workloads.positions(W))
    with pytest.raises(api.SchNetError) as e:
        m.energy_forces(p, _dev(workloads.types(W), torch.int32))   # no list built yet
    assert e.value.status == 7
    # workspace smaller than required
    cfg = m.cfg
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    ctx = C.c_void_p()
    w = nat.Weights()
    assert lib.schnet_create(C.byref(cfg), C.byref(w), None, C.c_void_p(ws.data_ptr()), 1024, C.byref(ctx)) == 1
    # the context is still usable after the errors
    m.build_neighbors(p)
    E, F = m.energy_forces(p, _dev(workloads.types(W), torch.int32))
    torch.cuda.synchronize()
    assert torch.isfinite(E).all() and m.status() == 0
