"""The allocation-free neighbour build (schnet_build_neighbors_noalloc) against the
context-based build (schnet_build_neighbors + schnet_get_neighbors).

This entry point serves callers that cannot allocate device memory where they
call the library; its scratch is a fixed device array inside the library.  The
test calls it through the C ABI twice in a row (different positions, so the
second call must not see the first call's leftovers) and requires exact
equality with the existing entry point, the tolerance used for neighbour
lists everywhere in this suite.  Small periodic boxes (one to three cells
per axis) are checked against the brute-force oracle directly, and so are the
status bits it returns for a list over capacity and for non-finite positions.
It lives in its own file, collected last."""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
from _helpers import random_box_positions
from schnet_gnn_molecular_b200 import _native as nat
from schnet_gnn_molecular_b200 import api, workloads

pytestmark = pytest.mark.gpu

FLAG_CAPACITY, FLAG_NONFINITE = 0x1, 0x4


def _noalloc_raw(lib, pos, ro_host, cutoff, skin, periodic, box3, cap):
    """One call; returns (status, row_ptr, col buffer, rev buffer, n_edges, flags) after a sync."""
    dev = torch.device("cuda")
    n = len(pos)
    p = torch.as_tensor(np.ascontiguousarray(pos, dtype=np.float32), device=dev)
    ro = torch.as_tensor(np.asarray(ro_host, dtype=np.int32), device=dev)
    rp = torch.full((n + 1,), -7, dtype=torch.int32, device=dev)
    col = torch.full((cap,), -7, dtype=torch.int32, device=dev)
    rev = torch.full((cap,), -7, dtype=torch.int32, device=dev)
    ne = torch.zeros(1, dtype=torch.int64, device=dev)
    flags = torch.full((1,), 0xFF, dtype=torch.int32, device=dev)
    box = (C.c_float * 3)(*(box3 if periodic else (0.0, 0.0, 0.0)))
    stream = torch.cuda.current_stream()
    st = lib.schnet_build_neighbors_noalloc(C.c_void_p(p.data_ptr()), n, len(ro_host) - 1,
                                            C.c_void_p(ro.data_ptr()), cutoff, skin, int(periodic), box,
                                            C.c_void_p(rp.data_ptr()), C.c_void_p(col.data_ptr()),
                                            C.c_void_p(rev.data_ptr()), cap, C.c_void_p(ne.data_ptr()),
                                            C.c_void_p(flags.data_ptr()), C.c_void_p(stream.cuda_stream))
    torch.cuda.synchronize()
    return st, rp.cpu().numpy(), col.cpu().numpy(), rev.cpu().numpy(), int(ne.item()), int(flags.item())


def _noalloc(lib, pos, w, cap):
    st, rp, col, rev, E, flags = _noalloc_raw(lib, pos, w.replica_offsets(), w.cutoff, w.skin, w.periodic,
                                              (w.box,) * 3, cap)
    assert st == 0 and flags == 0
    assert E <= cap
    return rp, col[:E], rev[:E]


def _with_context(pos, w):
    model = api.from_workload(w, workloads.weights(w))
    model.build_neighbors(torch.as_tensor(pos, device="cuda"))
    out = model.neighbors()
    model.close()
    return out


@pytest.mark.parametrize("w", [workloads.PROTEIN64.with_(n_replicas=16, name="cg_protein_16x269"),
                               workloads.BOX1M.with_(name="periodic_box_20000", beads=20000,
                                                     box=(20000 / 0.01) ** (1 / 3))],
                         ids=lambda w: w.name)
def test_noalloc_matches_context_build_twice(w):
    lib = nat.load()
    pos_a = workloads.positions(w)
    pos_b = (pos_a + np.random.default_rng(1).normal(scale=0.7, size=pos_a.shape)).astype(np.float32)
    cap = 4_000_000
    for pos in (pos_a, pos_b):
        rp, col, rev = _noalloc(lib, pos, w, cap)
        rp_c, col_c, rev_c = _with_context(pos, w)
        assert np.array_equal(rp, rp_c)
        assert np.array_equal(col, col_c)
        assert np.array_equal(rev, rev_c)


def test_noalloc_rejects_oversize():
    lib = nat.load()
    box = (C.c_float * 3)(0.0, 0.0, 0.0)
    d = torch.zeros(8, dtype=torch.int32, device="cuda")
    st = lib.schnet_build_neighbors_noalloc(C.c_void_p(d.data_ptr()), 70000, 1, C.c_void_p(d.data_ptr()), 10.0,
                                            2.0, 0, box, C.c_void_p(d.data_ptr()), C.c_void_p(d.data_ptr()),
                                            C.c_void_p(d.data_ptr()), 8, C.c_void_p(d.data_ptr()), None, None)
    assert st == 9   # SCHNET_ERR_UNSUPPORTED: more atoms than the fixed scratch holds


RL = 14.0   # r_c 12 + skin 2


@pytest.mark.parametrize("box3", [(2 * RL,) * 3, (2.5 * RL,) * 3, (2 * RL, 2.5 * RL, 3.25 * RL)],
                         ids=["one_cell", "two_cells", "one_two_three"])
def test_noalloc_small_periodic_boxes_match_oracle(box3):
    # one, two or three cells per axis: every cell is visited once by absolute index
    lib = nat.load()
    rng = np.random.default_rng(23)
    pos = random_box_positions(int(0.012 * np.prod(box3)), box3, rng, min_dist=2.5)
    for shift in (0.0, 0.37):   # two calls in a row, the second with moved atoms
        x = (pos + shift * rng.normal(size=pos.shape)).astype(np.float32)
        st, rp, col, rev, E, flags = _noalloc_raw(lib, x, [0, len(x)], 12.0, 2.0, True, box3, 400_000)
        assert st == 0 and flags == 0
        rp_o, col_o = oracle.neighbors(x, 12.0, 2.0, None, True, box3)
        assert np.array_equal(rp, rp_o)
        assert np.array_equal(col[:E], col_o)
        rows = np.repeat(np.arange(len(x)), np.diff(rp))
        assert np.array_equal(col[:E][rev[:E]], rows)


def test_noalloc_over_capacity_writes_nothing_past_it():
    lib = nat.load()
    w = workloads.PROTEIN64.with_(n_replicas=4, name="cg_protein_4x269")
    pos = workloads.positions(w)
    rp_o, col_o = oracle.neighbors(pos, w.cutoff, w.skin, w.replica_offsets())
    cap = len(col_o) - 1
    st, rp, col, rev, E, flags = _noalloc_raw(lib, pos, w.replica_offsets(), w.cutoff, w.skin, False,
                                              (0.0, 0.0, 0.0), cap)
    assert st == 0
    assert E == len(col_o)                      # the true count is reported
    assert flags & FLAG_CAPACITY
    assert np.array_equal(rp, rp_o)             # row pointers are complete
    assert np.all(col == -7) and np.all(rev == -7)   # the too-small buffers are left untouched


def test_noalloc_reports_non_finite_positions():
    lib = nat.load()
    w = workloads.TINY
    pos = workloads.positions(w).copy()
    pos[5, 1] = np.nan
    pos[9, 0] = np.inf
    st, rp, col, rev, E, flags = _noalloc_raw(lib, pos, w.replica_offsets(), w.cutoff, w.skin, False,
                                              (0.0, 0.0, 0.0), 100_000)
    assert st == 0 and flags & FLAG_NONFINITE
    # and a clean call right after reports nothing
    st, rp, col, rev, E, flags = _noalloc_raw(lib, workloads.positions(w), w.replica_offsets(), w.cutoff,
                                              w.skin, False, (0.0, 0.0, 0.0), 100_000)
    assert st == 0 and flags == 0
