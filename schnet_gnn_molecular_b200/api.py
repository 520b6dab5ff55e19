"""Python binding of the B200 SchNet library: torch tensors in, C ABI calls out.

Every step of the energy/force/integration path runs in the library's CUDA
kernels; this module only marshals arguments.  PyTorch supplies device
memory (the workspace is one uint8 tensor) and the stream.
"""
from __future__ import annotations

import ctypes as C

import numpy as np
import torch

from . import _native as nat


class SchNetError(RuntimeError):
    def __init__(self, status: int, msg: str = ""):
        self.status = status
        super().__init__(f"schnet: {nat.STATUS_NAMES.get(status, status)} {msg}".strip())


def _ptr(t):
    return C.c_void_p(t.data_ptr()) if t is not None else None


class SchNet:
    """One context: model, replicas and a device workspace.

    weights: dict of float32 arrays named as in include/schnet.h ([in, out] dense weights).
    """

    def __init__(self, *, n_types, F, K, L, rbf_min, rbf_max, rbf_sigma, cutoff, skin, replica_offsets, weights,
                 periodic=False, box=(0.0, 0.0, 0.0), edge_capacity=0, weight_dtype="fp32", device=None,
                 stream=None):
        if not torch.cuda.is_available():
            raise RuntimeError("SchNet needs a CUDA device (there is no CPU fallback)")
        self.lib = nat.load()
        self.device = torch.device(device or "cuda")
        ro = np.ascontiguousarray(np.asarray(replica_offsets, dtype=np.int32))
        self._ro = ro
        self.n_atoms = int(ro[-1])
        self.n_replicas = len(ro) - 1
        cfg = nat.Config()
        cfg.n_types, cfg.n_features, cfg.n_rbf, cfg.n_interactions = int(n_types), int(F), int(K), int(L)
        cfg.rbf_min, cfg.rbf_max, cfg.rbf_sigma = float(rbf_min), float(rbf_max), float(rbf_sigma)
        cfg.cutoff, cfg.skin, cfg.periodic = float(cutoff), float(skin), int(bool(periodic))
        cfg.box = (C.c_float * 3)(*[float(b) for b in box])
        cfg.n_atoms, cfg.n_replicas = self.n_atoms, self.n_replicas
        cfg.replica_offsets = ro.ctypes.data_as(C.POINTER(C.c_int32))
        cfg.edge_capacity = int(edge_capacity)
        cfg.weight_dtype = nat.WEIGHT_DTYPES[weight_dtype]
        self.cfg = cfg
        nbytes = C.c_size_t(0)
        st = self.lib.schnet_workspace_bytes(C.byref(cfg), C.byref(nbytes))
        if st != nat.OK:
            raise SchNetError(st, "workspace_bytes")
        self.workspace_bytes = int(nbytes.value)
        with torch.cuda.device(self.device):
            self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=self.device)
        keep = {}
        w = nat.Weights()
        for k in nat.WEIGHT_NAMES:
            a = np.ascontiguousarray(np.asarray(weights[k], dtype=np.float32))
            keep[k] = a
            setattr(w, k, a.ctypes.data_as(C.POINTER(C.c_float)))
        w.c2 = float(weights["c2"])
        self.stream = stream if stream is not None else torch.cuda.current_stream(self.device)
        ctx = C.c_void_p()
        with torch.cuda.device(self.device):
            st = self.lib.schnet_create(C.byref(cfg), C.byref(w), C.c_void_p(self.stream.cuda_stream),
                                        _ptr(self.workspace), C.c_size_t(self.workspace_bytes), C.byref(ctx))
        if st != nat.OK:
            raise SchNetError(st, "create")
        self.ctx = ctx

    # ------------------------------------------------------------------
    def _check(self, st, what):
        if st != nat.OK:
            msg = self.lib.schnet_last_error(self.ctx)
            raise SchNetError(st, f"{what}: {msg.decode() if msg else ''}")

    def close(self):
        if getattr(self, "ctx", None):
            self.lib.schnet_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------------
    def build_neighbors(self, pos: torch.Tensor):
        assert pos.is_cuda and pos.dtype == torch.float32 and pos.is_contiguous()
        self._check(self.lib.schnet_build_neighbors(self.ctx, _ptr(pos)), "build_neighbors")

    def energy_forces(self, pos: torch.Tensor, types: torch.Tensor, forces: bool = True):
        energy = torch.empty(self.n_replicas, dtype=torch.float64, device=self.device)
        F = torch.empty((self.n_atoms, 3), dtype=torch.float32, device=self.device) if forces else None
        self._check(self.lib.schnet_energy_forces(self.ctx, _ptr(pos), _ptr(types), _ptr(energy), _ptr(F)),
                    "energy_forces")
        return energy, F

    def step(self, pos, vel, types, mass, n_steps, *, dt=4.0, gamma=0.1, temperature=300.0, n_rebuild=20,
             seed=0, step0=0, noise=None, resume=False, use_graph=True, raise_on_flag=True):
        p = nat.StepParams(float(dt), float(gamma), float(temperature), int(n_rebuild), int(seed), int(step0),
                           C.c_void_p(noise.data_ptr()) if noise is not None else None, int(bool(resume)),
                           int(bool(use_graph)))
        epot = torch.empty(self.n_replicas, dtype=torch.float64, device=self.device)
        ekin = torch.empty(self.n_replicas, dtype=torch.float64, device=self.device)
        st = self.lib.schnet_step(self.ctx, _ptr(pos), _ptr(vel), _ptr(types), _ptr(mass), int(n_steps),
                                  C.byref(p), _ptr(epot), _ptr(ekin))
        if raise_on_flag or st not in (3, 4, 5, 6, 8):
            self._check(st, "step")
        return epot, ekin, st

    def step_host(self, pos: np.ndarray, vel: np.ndarray, types: np.ndarray, mass: np.ndarray, n_steps, *,
                  dt=4.0, gamma=0.1, temperature=300.0, n_rebuild=20, seed=0, step0=0, resume=False,
                  use_graph=True, epot=None, ekin=None):
        """Host buffers in/out (pinned numpy views recommended); updates pos/vel in place."""
        p = nat.StepParams(float(dt), float(gamma), float(temperature), int(n_rebuild), int(seed), int(step0),
                           None, int(bool(resume)), int(bool(use_graph)))
        epot = np.empty(self.n_replicas) if epot is None else epot
        ekin = np.empty(self.n_replicas) if ekin is None else ekin
        vp = lambda a: C.c_void_p(a.ctypes.data)
        st = self.lib.schnet_step_host(self.ctx, vp(pos), vp(vel), vp(types), vp(mass), int(n_steps), C.byref(p),
                                       vp(epot), vp(ekin))
        self._check(st, "step_host")
        return epot, ekin

    def status(self) -> int:
        f = C.c_uint32(0)
        self._check(self.lib.schnet_get_status(self.ctx, C.byref(f)), "get_status")
        return int(f.value)

    def neighbors(self):
        """(row_ptr, col, rev) as numpy int32 arrays (synchronizes)."""
        n_e = C.c_int64(0)
        rp = np.zeros(self.n_atoms + 1, dtype=np.int32)
        self._check(self.lib.schnet_get_neighbors(self.ctx, C.c_void_p(rp.ctypes.data), None, None, C.byref(n_e),
                                                  0), "get_neighbors")
        E = int(n_e.value)
        col = np.zeros(max(E, 1), dtype=np.int32)
        rev = np.zeros(max(E, 1), dtype=np.int32)
        self._check(self.lib.schnet_get_neighbors(self.ctx, None, C.c_void_p(col.ctypes.data),
                                                  C.c_void_p(rev.ctypes.data), C.byref(n_e), E), "get_neighbors")
        return rp, col[:E], rev[:E]

    def atom_energies(self) -> torch.Tensor:
        out = torch.empty(self.n_atoms, dtype=torch.float32, device=self.device)
        self._check(self.lib.schnet_get_atom_energies(self.ctx, _ptr(out)), "get_atom_energies")
        return out

    def profile_steps(self, pos, vel, types, mass, n_steps, *, dt=4.0, gamma=0.1, temperature=300.0, n_rebuild=20,
                      seed=0, step0=0, resume=True):
        """Eager steps with CUDA events around every kernel on the library stream.
        Returns {class: (total_ms, launches)}."""
        p = nat.StepParams(float(dt), float(gamma), float(temperature), int(n_rebuild), int(seed), int(step0), None,
                           int(bool(resume)), 0)
        ms = (C.c_double * len(nat.KERNEL_CLASSES))()
        cnt = (C.c_int64 * len(nat.KERNEL_CLASSES))()
        st = self.lib.schnet_profile_steps(self.ctx, _ptr(pos), _ptr(vel), _ptr(types), _ptr(mass), int(n_steps),
                                           C.byref(p), ms, cnt)
        self._check(st, "profile_steps")
        return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(nat.KERNEL_CLASSES)}

    def kernel_launches(self) -> int:
        return int(self.lib.schnet_kernel_launches(self.ctx))


def from_workload(w, weights: dict, device=None, edge_capacity=0, weight_dtype=None) -> SchNet:
    """Context for a ``workloads.Workload``."""
    return SchNet(n_types=w.n_types, F=w.F, K=w.K, L=w.L, rbf_min=w.rbf_min, rbf_max=w.rbf_max,
                  rbf_sigma=w.rbf_sigma, cutoff=w.cutoff, skin=w.skin, replica_offsets=w.replica_offsets(),
                  weights=weights, periodic=w.periodic, box=(w.box,) * 3 if w.periodic else (0.0, 0.0, 0.0),
                  edge_capacity=edge_capacity, weight_dtype=weight_dtype or w.weight_dtype, device=device)
