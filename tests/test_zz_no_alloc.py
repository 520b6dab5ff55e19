"""The allocation-free neighbour build (schnet_build_neighbors_noalloc) against the
context-based build (schnet_build_neighbors + schnet_get_neighbors).

This entry point serves callers that cannot allocate device memory where they
call the library; its scratch is a fixed device array inside the library.  The
test calls it through the C ABI twice in a row (different positions, so the
second call must not see the first call's leftovers) and requires exact
equality with the existing entry point, the tolerance used for neighbour
lists everywhere in this suite.  It lives in its own file, collected last."""
import ctypes as C

import numpy as np
import pytest
import torch

from schnet_gnn_molecular_b200 import _native as nat
from schnet_gnn_molecular_b200 import api, workloads

pytestmark = pytest.mark.gpu


def _noalloc(lib, pos, w, cap):
    dev = torch.device("cuda")
    p = torch.as_tensor(pos, device=dev)
    ro = torch.as_tensor(w.replica_offsets(), device=dev)
    rp = torch.full((w.n_atoms + 1,), -7, dtype=torch.int32, device=dev)
    col = torch.full((cap,), -7, dtype=torch.int32, device=dev)
    rev = torch.full((cap,), -7, dtype=torch.int32, device=dev)
    ne = torch.zeros(1, dtype=torch.int64, device=dev)
    box = (C.c_float * 3)(*([w.box] * 3 if w.periodic else [0.0, 0.0, 0.0]))
    stream = torch.cuda.current_stream()
    st = lib.schnet_build_neighbors_noalloc(C.c_void_p(p.data_ptr()), w.n_atoms, w.n_replicas,
                                            C.c_void_p(ro.data_ptr()), w.cutoff, w.skin, int(w.periodic), box,
                                            C.c_void_p(rp.data_ptr()), C.c_void_p(col.data_ptr()),
                                            C.c_void_p(rev.data_ptr()), cap, C.c_void_p(ne.data_ptr()),
                                            C.c_void_p(stream.cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    E = int(ne.item())
    assert E <= cap
    return rp.cpu().numpy(), col[:E].cpu().numpy(), rev[:E].cpu().numpy()


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
                                            C.c_void_p(d.data_ptr()), 8, C.c_void_p(d.data_ptr()), None)
    assert st == 9   # SCHNET_ERR_UNSUPPORTED: more atoms than the fixed scratch holds
