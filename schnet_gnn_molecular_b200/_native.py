"""ctypes declarations of the C ABI in ``include/schnet.h`` (argument marshalling only).

Loading fails loudly if the in-tree ``libschnet_b200.so`` is missing: there is
no fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libschnet_b200.so")

OK = 0
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "CUDA", 3: "CAPACITY", 4: "SKIN", 5: "NONFINITE", 6: "BADTYPE",
                7: "STATE", 8: "TIMEOUT", 9: "UNSUPPORTED"}
FLAG_CAPACITY, FLAG_SKIN, FLAG_NONFINITE, FLAG_BADTYPE, FLAG_TIMEOUT = 0x1, 0x2, 0x4, 0x8, 0x10
WEIGHT_DTYPES = {"fp32": 0, "fp16": 1, "bf16": 2, "fp16fast": 3}

EXPORTED = ["schnet_workspace_bytes", "schnet_create", "schnet_build_neighbors", "schnet_energy_forces",
            "schnet_step", "schnet_step_host", "schnet_get_status", "schnet_last_error", "schnet_destroy",
            "schnet_get_neighbors", "schnet_get_atom_energies", "schnet_kernel_launches", "schnet_profile_steps",
            "schnet_build_neighbors_noalloc", "schnet_test_exp2", "schnet_test_timeout"]
KERNEL_CLASSES = ["cfconv_fwd", "cfconv_bwd", "atomwise", "neighbors", "forces", "integrate", "reduce", "mask",
                  "cfconv_dh"]


class Config(C.Structure):
    _fields_ = [("n_types", C.c_int32), ("n_features", C.c_int32), ("n_rbf", C.c_int32),
                ("n_interactions", C.c_int32), ("rbf_min", C.c_float), ("rbf_max", C.c_float),
                ("rbf_sigma", C.c_float), ("cutoff", C.c_float), ("skin", C.c_float), ("periodic", C.c_int32),
                ("box", C.c_float * 3), ("n_atoms", C.c_int32), ("n_replicas", C.c_int32),
                ("replica_offsets", C.POINTER(C.c_int32)), ("edge_capacity", C.c_int64),
                ("weight_dtype", C.c_int32)]


_FP = C.POINTER(C.c_float)
WEIGHT_NAMES = ["emb", "W_in", "W1", "b1", "W2", "b2", "Wo1", "bo1", "Wo2", "bo2", "R1", "c1", "R2"]


class Weights(C.Structure):
    _fields_ = [(k, _FP) for k in WEIGHT_NAMES] + [("c2", C.c_float)]


class StepParams(C.Structure):
    _fields_ = [("dt_fs", C.c_float), ("gamma_per_ps", C.c_float), ("temperature_K", C.c_float),
                ("n_rebuild", C.c_int32), ("seed", C.c_uint64), ("step0", C.c_uint64),
                ("d_noise", C.c_void_p), ("resume", C.c_int32), ("use_graph", C.c_int32)]


_lib = None


def load() -> C.CDLL:
    """Load the in-tree shared library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m schnet_gnn_molecular_b200.build` "
                           "(there is no CPU fallback)")
    L = C.CDLL(LIB_PATH)
    vp, i32p, i64p, u32p, dp = C.c_void_p, C.POINTER(C.c_int32), C.POINTER(C.c_int64), C.POINTER(C.c_uint32), \
        C.POINTER(C.c_double)
    L.schnet_workspace_bytes.argtypes = [C.POINTER(Config), C.POINTER(C.c_size_t)]
    L.schnet_create.argtypes = [C.POINTER(Config), C.POINTER(Weights), vp, vp, C.c_size_t, C.POINTER(vp)]
    L.schnet_build_neighbors.argtypes = [vp, vp]
    L.schnet_energy_forces.argtypes = [vp, vp, vp, vp, vp]
    L.schnet_step.argtypes = [vp, vp, vp, vp, vp, C.c_int64, C.POINTER(StepParams), vp, vp]
    L.schnet_step_host.argtypes = [vp, vp, vp, vp, vp, C.c_int64, C.POINTER(StepParams), vp, vp]
    L.schnet_get_status.argtypes = [vp, u32p]
    L.schnet_last_error.argtypes = [vp]
    L.schnet_last_error.restype = C.c_char_p
    L.schnet_destroy.argtypes = [vp]
    L.schnet_get_neighbors.argtypes = [vp, vp, vp, vp, i64p, C.c_int64]
    L.schnet_get_atom_energies.argtypes = [vp, vp]
    L.schnet_test_exp2.argtypes = [vp, vp, C.c_int64, vp]
    L.schnet_test_timeout.argtypes = [vp, C.c_uint32, C.c_int32]
    L.schnet_profile_steps.argtypes = [vp, vp, vp, vp, vp, C.c_int64, C.POINTER(StepParams), dp, i64p]
    L.schnet_build_neighbors_noalloc.argtypes = [vp, C.c_int32, C.c_int32, vp, C.c_float, C.c_float, C.c_int32,
                                                 C.POINTER(C.c_float), vp, vp, vp, C.c_int64, vp, vp, vp]
    L.schnet_kernel_launches.argtypes = [vp]
    L.schnet_kernel_launches.restype = C.c_int64
    for name in EXPORTED:
        if name not in ("schnet_last_error", "schnet_kernel_launches"):
            getattr(L, name).restype = C.c_int
    _lib = L
    return L
