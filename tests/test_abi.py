"""CPU checks of the C ABI library: it builds/loads, exports every symbol the
header declares, and validates configurations without touching a GPU."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from schnet_gnn_molecular_b200 import _native as nat
from schnet_gnn_molecular_b200 import build, workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return nat.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "schnet.h")).read()
    return sorted(set(re.findall(r"SCHNET_API\s+[\w\s\*]+?\b(schnet_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(nat.EXPORTED) == names


def _cfg(w, **kw):
    ro = w.replica_offsets()
    c = nat.Config()
    c.n_types, c.n_features, c.n_rbf, c.n_interactions = w.n_types, w.F, w.K, w.L
    c.rbf_min, c.rbf_max, c.rbf_sigma, c.cutoff, c.skin = w.rbf_min, w.rbf_max, w.rbf_sigma, w.cutoff, w.skin
    c.periodic = int(w.periodic)
    c.box = (C.c_float * 3)(*([w.box] * 3 if w.periodic else [0, 0, 0]))
    c.n_atoms, c.n_replicas = w.n_atoms, w.n_replicas
    c.replica_offsets = ro.ctypes.data_as(C.POINTER(C.c_int32))
    c.edge_capacity = 0
    c.weight_dtype = 0
    for k, v in kw.items():
        setattr(c, k, v)
    return c, ro


def test_workspace_sizes_and_validation(lib):
    sizes = {}
    for w in [workloads.TINY, workloads.PROTEIN64, workloads.BOX1M]:
        c, ro = _cfg(w)
        n = C.c_size_t(0)
        assert lib.schnet_workspace_bytes(C.byref(c), C.byref(n)) == 0
        sizes[w.name] = n.value
        # activations alone: 2 L N 128 floats
        assert n.value > 2 * w.L * w.n_atoms * 128 * 4
    assert sizes["periodic_box_1M"] < 40e9
    w = workloads.TINY
    for bad, st in [(dict(n_features=256), 9), (dict(n_features=3), 9), (dict(n_rbf=65), 9),
                    (dict(n_interactions=0), 9), (dict(cutoff=0.0), 1), (dict(n_types=0), 1),
                    (dict(weight_dtype=7), 1)]:
        c, ro = _cfg(w, **bad)
        n = C.c_size_t(0)
        assert lib.schnet_workspace_bytes(C.byref(c), C.byref(n)) == st, bad
    c, ro = _cfg(workloads.BOX1M)
    c.box = (C.c_float * 3)(20.0, 20.0, 20.0)       # smaller than 2 (r_c + skin)
    assert lib.schnet_workspace_bytes(C.byref(c), C.byref(C.c_size_t(0))) == 9
    c, ro = _cfg(w)
    ro[-1] = 63                                       # offsets must end at n_atoms
    assert lib.schnet_workspace_bytes(C.byref(c), C.byref(C.c_size_t(0))) == 1


def test_create_rejects_bad_arguments_without_gpu(lib):
    c, ro = _cfg(workloads.TINY)
    ctx = C.c_void_p()
    # null weights / unaligned or missing workspace are argument errors caught before any CUDA call
    assert lib.schnet_create(C.byref(c), None, None, None, 0, C.byref(ctx)) == 1
    assert ctx.value is None
    assert lib.schnet_build_neighbors(None, None) == 1
    assert lib.schnet_destroy(None) == 0
    assert lib.schnet_kernel_launches(None) == 0
