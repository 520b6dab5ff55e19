"""Float64 CPU oracle for the SchNet CFConv energy/force path -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never imports, links or executes anything here, and this package
imports nothing from the product.

The arithmetic lives in ``schnet_oracle.c`` (plain C, float64, explicit loops,
brute-force O(N^2) pairs, OpenMP over atoms); this module compiles it with gcc
on first use and wraps it with ctypes.  Pinning tests live in
``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "schnet_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fused multiply-add, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp",
               "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


class _Model(C.Structure):
    _fields_ = [("T", C.c_int), ("F", C.c_int), ("K", C.c_int), ("L", C.c_int),
                ("rbf_min", C.c_double), ("rbf_max", C.c_double),
                ("rbf_sigma", C.c_double), ("cutoff", C.c_double),
                ("periodic", C.c_int), ("box", C.c_double * 3)]


_WNAMES = ["emb", "W_in", "W1", "b1", "W2", "b2", "Wo1", "bo1", "Wo2", "bo2", "R1", "c1", "R2"]


class _Weights(C.Structure):
    _fields_ = [(k, C.POINTER(C.c_double)) for k in _WNAMES] + [("c2", C.c_double)]


_dp = C.POINTER(C.c_double)
_ip = C.POINTER(C.c_int)
_i32p = C.POINTER(C.c_int32)
_u32p = C.POINTER(C.c_uint32)
_fp = C.POINTER(C.c_float)


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            L.or_ssp.restype = C.c_double; L.or_ssp.argtypes = [C.c_double]
            L.or_dssp.restype = C.c_double; L.or_dssp.argtypes = [C.c_double]
            L.or_fc.restype = C.c_double; L.or_fc.argtypes = [C.c_double, C.c_double]
            L.or_dfc.restype = C.c_double; L.or_dfc.argtypes = [C.c_double, C.c_double]
            L.or_rbf_center.restype = C.c_double
            L.or_rbf_center.argtypes = [C.c_int, C.c_int, C.c_double, C.c_double]
            L.or_rbf.restype = None
            L.or_rbf.argtypes = [C.c_double, C.c_int, C.c_double, C.c_double, C.c_double, _dp, _dp]
            L.or_filter.restype = None
            L.or_filter.argtypes = [C.POINTER(_Model), C.POINTER(_Weights), C.c_int, C.c_double, _dp, _dp, _dp]
            L.or_neighbors.restype = C.c_int64
            L.or_neighbors.argtypes = [C.c_int, _fp, C.c_int, _ip, C.c_float, C.c_float, C.c_int, _fp,
                                       C.c_int64, _i32p, _i32p]
            L.or_cfconv.restype = C.c_int
            L.or_cfconv.argtypes = [C.POINTER(_Model), C.POINTER(_Weights), C.c_int, C.c_int, _dp, C.c_int,
                                    _ip, _dp, _dp]
            L.or_cut_edges.restype = C.c_int64
            L.or_cut_edges.argtypes = [C.POINTER(_Model), C.c_int, _dp, C.c_int, _ip, C.c_int64, _i32p,
                                       _i32p, _dp]
            L.or_energy_forces.restype = C.c_int
            L.or_energy_forces.argtypes = [C.POINTER(_Model), C.POINTER(_Weights), C.c_int, _dp, _ip, C.c_int,
                                           _ip, _dp, _dp, _dp]
            L.or_philox4x32_10.restype = None
            L.or_philox4x32_10.argtypes = [_u32p, _u32p, _u32p]
            L.or_noise.restype = None
            L.or_noise.argtypes = [C.c_uint64, C.c_uint64, C.c_int, _dp]
            L.or_baoa.restype = None
            L.or_baoa.argtypes = [C.c_int, _dp, _dp, _dp, _dp, C.c_double, C.c_double, C.c_double, _dp]
            L.or_b.restype = None
            L.or_b.argtypes = [C.c_int, _dp, _dp, _dp, C.c_double]
            L.or_kinetic.restype = None
            L.or_kinetic.argtypes = [C.c_int, _dp, _dp, C.c_int, _ip, _dp]
            L.or_md_step.restype = C.c_int
            L.or_md_step.argtypes = [C.POINTER(_Model), C.POINTER(_Weights), C.c_int, _dp, _dp, _ip, _dp,
                                     C.c_int, _ip, C.c_double, C.c_double, C.c_double, C.c_uint64,
                                     C.c_uint64, _dp, _dp, _dp, _dp]
            _lib = L
    return _lib


def _p(a, t=_dp):
    return a.ctypes.data_as(t) if a is not None else None


def set_threads(n: int) -> None:
    """Set the OpenMP thread count used by the oracle (before first call)."""
    os.environ["OMP_NUM_THREADS"] = str(int(n))


# --------------------------------------------------------------------------
# Model handle
# --------------------------------------------------------------------------

@dataclass
class Model:
    """Hyper-parameters plus float64 weights, in the oracle's own layout.

    ``weights`` maps the names emb, W_in, W1, b1, W2, b2, Wo1, bo1, Wo2, bo2,
    R1, c1, R2 (arrays) and c2 (float) to values; dense weights are [in, out].
    """
    n_types: int
    F: int
    K: int
    L: int
    rbf_min: float
    rbf_max: float
    rbf_sigma: float
    cutoff: float
    weights: dict
    periodic: bool = False
    box: tuple = (0.0, 0.0, 0.0)

    def _structs(self):
        m = _Model(self.n_types, self.F, self.K, self.L, float(self.rbf_min), float(self.rbf_max),
                   float(self.rbf_sigma), float(self.cutoff), int(bool(self.periodic)),
                   (C.c_double * 3)(*[float(b) for b in self.box]))
        keep = {}
        w = _Weights()
        F, K, L, H = self.F, self.K, self.L, self.F // 2
        shapes = {"emb": (self.n_types, F), "W_in": (L, F, F), "W1": (L, K, F), "b1": (L, F),
                  "W2": (L, F, F), "b2": (L, F), "Wo1": (L, F, F), "bo1": (L, F), "Wo2": (L, F, F),
                  "bo2": (L, F), "R1": (F, H), "c1": (H,), "R2": (H,)}
        for k in _WNAMES:
            a = np.ascontiguousarray(np.asarray(self.weights[k], dtype=np.float64).reshape(shapes[k]))
            keep[k] = a
            setattr(w, k, _p(a))
        w.c2 = float(self.weights["c2"])
        return m, w, keep


def _offsets(n, replica_offsets):
    if replica_offsets is None:
        replica_offsets = [0, n]
    ro = np.ascontiguousarray(np.asarray(replica_offsets, dtype=np.int32))
    return ro, len(ro) - 1


# --------------------------------------------------------------------------
# Wrapped entry points
# --------------------------------------------------------------------------

def ssp(x):
    return lib().or_ssp(float(x))


def dssp(x):
    return lib().or_dssp(float(x))


def fc(d, rc):
    return lib().or_fc(float(d), float(rc))


def dfc(d, rc):
    return lib().or_dfc(float(d), float(rc))


def rbf_center(k, K, rmin, rmax):
    return lib().or_rbf_center(int(k), int(K), float(rmin), float(rmax))


def rbf(d, K, rmin, rmax, sigma):
    e = np.zeros(K); de = np.zeros(K)
    lib().or_rbf(float(d), int(K), float(rmin), float(rmax), float(sigma), _p(e), _p(de))
    return e, de


def filter_(model: Model, layer: int, d: float):
    """Filter W(d) and dW/dd of one interaction at one distance."""
    m, w, keep = model._structs()
    W = np.zeros(model.F); dW = np.zeros(model.F)
    work = np.zeros(2 * model.K + 4 * model.F)
    lib().or_filter(C.byref(m), C.byref(w), int(layer), float(d), _p(W), _p(dW), _p(work))
    return W, dW


def neighbors(pos32, cutoff, skin, replica_offsets=None, periodic=False, box=(0, 0, 0), cap=None):
    """Brute-force list with skin; returns (row_ptr int32 [n+1], col int32 [E])."""
    pos32 = np.ascontiguousarray(np.asarray(pos32, dtype=np.float32).reshape(-1, 3))
    n = pos32.shape[0]
    ro, R = _offsets(n, replica_offsets)
    if cap is None:
        sizes = np.diff(ro).astype(np.int64)
        cap = int((sizes * np.maximum(sizes - 1, 0)).sum())
    row_ptr = np.zeros(n + 1, dtype=np.int32)
    col = np.zeros(max(cap, 1), dtype=np.int32)
    boxa = np.ascontiguousarray(np.asarray(box, dtype=np.float32))
    E = lib().or_neighbors(n, _p(pos32, _fp), R, _p(ro, _ip), C.c_float(cutoff), C.c_float(skin),
                           int(bool(periodic)), _p(boxa, _fp), int(cap), _p(row_ptr, _i32p), _p(col, _i32p))
    if E > cap:
        raise ValueError(f"edge capacity {cap} < {E}")
    return row_ptr, col[:E].copy()


def cut_edges(model: Model, pos, replica_offsets=None):
    """Exact-cutoff edges (row, col, d) in CSR order (rows ascending, cols ascending)."""
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.float64).reshape(-1, 3))
    n = pos.shape[0]
    ro, R = _offsets(n, replica_offsets)
    m, _, _ = model._structs()
    E = lib().or_cut_edges(C.byref(m), n, _p(pos), R, _p(ro, _ip), 0, None, None, None)
    row = np.zeros(max(E, 1), np.int32); col = np.zeros(max(E, 1), np.int32); d = np.zeros(max(E, 1))
    lib().or_cut_edges(C.byref(m), n, _p(pos), R, _p(ro, _ip), E, _p(row, _i32p), _p(col, _i32p), _p(d))
    return row[:E], col[:E], d[:E]


def cfconv(model: Model, layer: int, pos, h, replica_offsets=None):
    """Segment-sum aggregation m_i = sum_j h_j (.) W(d_ij) over exact-cutoff rows."""
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.float64).reshape(-1, 3))
    n = pos.shape[0]
    h = np.ascontiguousarray(np.asarray(h, dtype=np.float64).reshape(n, model.F))
    ro, R = _offsets(n, replica_offsets)
    m, w, keep = model._structs()
    out = np.zeros((n, model.F))
    rc = lib().or_cfconv(C.byref(m), C.byref(w), int(layer), n, _p(pos), R, _p(ro, _ip), _p(h), _p(out))
    if rc:
        raise RuntimeError(f"or_cfconv failed ({rc})")
    return out


def energy_forces(model: Model, pos, types, replica_offsets=None, forces=True):
    """Returns (E [R], eps [n], F [n,3] or None), all float64."""
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.float64).reshape(-1, 3))
    n = pos.shape[0]
    types = np.ascontiguousarray(np.asarray(types, dtype=np.int32))
    ro, R = _offsets(n, replica_offsets)
    m, w, keep = model._structs()
    E = np.zeros(R); eps = np.zeros(n)
    F = np.zeros((n, 3)) if forces else None
    rc = lib().or_energy_forces(C.byref(m), C.byref(w), n, _p(pos), _p(types, _ip), R, _p(ro, _ip),
                                _p(E), _p(eps), _p(F) if forces else None)
    if rc == -2:
        raise ValueError("atom type outside [0, n_types)")
    if rc:
        raise RuntimeError(f"or_energy_forces failed ({rc})")
    return E, eps, F


def philox4x32_10(ctr, key):
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    o = np.zeros(4, dtype=np.uint32)
    lib().or_philox4x32_10(_p(c, _u32p), _p(k, _u32p), _p(o, _u32p))
    return o


def noise(seed, step, n):
    xi = np.zeros((n, 3))
    lib().or_noise(C.c_uint64(seed), C.c_uint64(step), int(n), _p(xi))
    return xi


def baoa(pos, vel, F, mass, dt, gamma, temperature, xi=None):
    """In-place B-A-O-A on float64 copies; returns (pos, vel)."""
    pos = np.array(pos, dtype=np.float64).reshape(-1, 3)
    vel = np.array(vel, dtype=np.float64).reshape(-1, 3)
    F = np.ascontiguousarray(np.asarray(F, dtype=np.float64).reshape(-1, 3))
    mass = np.ascontiguousarray(np.asarray(mass, dtype=np.float64))
    n = pos.shape[0]
    xi = None if xi is None else np.ascontiguousarray(np.asarray(xi, dtype=np.float64).reshape(n, 3))
    if gamma != 0.0 and xi is None:
        raise ValueError("noise required when gamma != 0")
    lib().or_baoa(n, _p(pos), _p(vel), _p(F), _p(mass), float(dt), float(gamma), float(temperature), _p(xi))
    return pos, vel


def b_kick(vel, F, mass, dt):
    vel = np.array(vel, dtype=np.float64).reshape(-1, 3)
    F = np.ascontiguousarray(np.asarray(F, dtype=np.float64).reshape(-1, 3))
    mass = np.ascontiguousarray(np.asarray(mass, dtype=np.float64))
    lib().or_b(vel.shape[0], _p(vel), _p(F), _p(mass), float(dt))
    return vel


def kinetic(vel, mass, replica_offsets=None):
    vel = np.ascontiguousarray(np.asarray(vel, dtype=np.float64).reshape(-1, 3))
    mass = np.ascontiguousarray(np.asarray(mass, dtype=np.float64))
    n = vel.shape[0]
    ro, R = _offsets(n, replica_offsets)
    ek = np.zeros(R)
    lib().or_kinetic(n, _p(vel), _p(mass), R, _p(ro, _ip), _p(ek))
    return ek


def md_step(model: Model, pos, vel, types, mass, F, dt, gamma, temperature, seed, step,
            replica_offsets=None, noise_override=None):
    """One BAOAB step (gamma = 0: velocity Verlet).  F are the forces at pos.
    Returns (pos, vel, F_new, epot [R], ekin [R])."""
    pos = np.array(pos, dtype=np.float64).reshape(-1, 3)
    vel = np.array(vel, dtype=np.float64).reshape(-1, 3)
    F = np.array(F, dtype=np.float64).reshape(-1, 3)
    n = pos.shape[0]
    types = np.ascontiguousarray(np.asarray(types, dtype=np.int32))
    mass = np.ascontiguousarray(np.asarray(mass, dtype=np.float64))
    ro, R = _offsets(n, replica_offsets)
    m, w, keep = model._structs()
    nz = None if noise_override is None else np.ascontiguousarray(
        np.asarray(noise_override, dtype=np.float64).reshape(n, 3))
    ep = np.zeros(R); ek = np.zeros(R)
    rc = lib().or_md_step(C.byref(m), C.byref(w), n, _p(pos), _p(vel), _p(types, _ip), _p(mass), R,
                          _p(ro, _ip), float(dt), float(gamma), float(temperature), C.c_uint64(seed),
                          C.c_uint64(step), _p(nz), _p(F), _p(ep), _p(ek))
    if rc:
        raise RuntimeError(f"or_md_step failed ({rc})")
    return pos, vel, F, ep, ek
