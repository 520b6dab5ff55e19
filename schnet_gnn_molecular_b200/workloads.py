"""The synthetic workloads the library is tested and benchmarked on.

Each stands in for the pages' benchmark system (a 269-bead coarse-grained
protein, 64 parallel replicas, on one GPU -- FlashSchNet summary, section
Achievement 1), which is not available here; shapes, sizes and model
hyper-parameters follow the five workload descriptions the library targets.
Nothing here computes any part of the method.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from functools import lru_cache

import numpy as np

from . import inputs


@dataclass(frozen=True)
class Workload:
    name: str
    n_replicas: int
    beads: int                 # beads per replica
    geometry: str              # "chain" | "compact" | "box"
    n_types: int
    F: int
    K: int
    rbf_min: float
    rbf_max: float
    rbf_sigma: float
    cutoff: float
    L: int
    skin: float = 2.0
    periodic: bool = False
    box: float = 0.0
    density: float = 0.0
    integrator: str = "baoab"  # "baoab" | "vv"
    dt_fs: float = 4.0
    gamma_per_ps: float = 0.1
    temperature: float = 300.0
    n_rebuild: int = 20
    steps: int = 1
    weight_dtype: str = "fp32"  # "fp32" | "fp16" | "bf16" | "fp16fast" (fp16 weights and filter activations)
    seed: int = 0
    radius: float | None = None  # confinement radius for compact chains
    rg_target: float = 12.0
    mass: float = 72.0         # amu per bead (MARTINI-style bead, see the mass reading)
    pool: int = 0              # >0: replicas r >= pool are random rotations of replica r % pool

    @property
    def n_atoms(self) -> int:
        return self.n_replicas * self.beads

    def replica_offsets(self) -> np.ndarray:
        return (np.arange(self.n_replicas + 1, dtype=np.int32) * self.beads).astype(np.int32)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY = Workload(name="tiny_chain64", n_replicas=1, beads=64, geometry="chain", n_types=16, F=64, K=32,
                rbf_min=0.0, rbf_max=10.0, rbf_sigma=0.3, cutoff=10.0, L=2, steps=1, seed=0)

PROTEIN64 = Workload(name="cg_protein_64x269", n_replicas=64, beads=269, geometry="compact", n_types=25,
                     F=128, K=50, rbf_min=0.0, rbf_max=15.0, rbf_sigma=0.3, cutoff=15.0, L=3,
                     steps=10000, seed=1000)

PROTEIN64_FP16 = PROTEIN64.with_(name="cg_protein_64x269_fp16w", weight_dtype="fp16", seed=2000)
PROTEIN64_BF16 = PROTEIN64.with_(name="cg_protein_64x269_bf16w", weight_dtype="bf16", seed=2000)
PROTEIN64_FP16FAST = PROTEIN64.with_(name="cg_protein_64x269_fp16fast", weight_dtype="fp16fast", seed=2000)


def sweep(n_replicas: int) -> Workload:
    """Replica-count sweep: 64 independently drawn chains, the rest rotated copies
    (same per-replica work; drawing 1024 chains would take minutes)."""
    return PROTEIN64.with_(name=f"cg_protein_{n_replicas}x269", n_replicas=n_replicas, seed=3000, pool=64)


def globule(beads: int) -> Workload:
    # same bead density as the 269-bead compact chain
    r269 = math.sqrt(5.0 / 3.0) * 12.0
    radius = r269 * (beads / 269.0) ** (1.0 / 3.0)
    return PROTEIN64.with_(name=f"cg_globule_{beads}", n_replicas=1, beads=beads, seed=3000 + beads,
                           radius=radius, rg_target=math.sqrt(3.0 / 5.0) * radius)


BOX1M = Workload(name="periodic_box_1M", n_replicas=1, beads=1_000_000, geometry="box", n_types=10, F=128,
                 K=50, rbf_min=0.0, rbf_max=12.0, rbf_sigma=0.3, cutoff=12.0, L=3, periodic=True,
                 density=0.01, box=(1_000_000 / 0.01) ** (1.0 / 3.0), integrator="vv", gamma_per_ps=0.0,
                 steps=1000, seed=4000)

ALL = {w.name: w for w in [TINY, PROTEIN64, PROTEIN64_FP16, PROTEIN64_BF16, PROTEIN64_FP16FAST, BOX1M]}


@lru_cache(maxsize=16)
def _positions(w: Workload) -> np.ndarray:
    out = np.zeros((w.n_atoms, 3))
    for r in range(w.n_replicas):
        if w.pool and r >= w.pool:
            base = out[(r % w.pool) * w.beads:(r % w.pool + 1) * w.beads]
            rot = inputs.random_rotation(np.random.default_rng(w.seed + r))
            out[r * w.beads:(r + 1) * w.beads] = base @ rot.T
            continue
        rng = np.random.default_rng(w.seed + r)
        if w.geometry == "chain":
            p = inputs.chain(w.beads, rng)
            p = p - p.mean(0)
        elif w.geometry == "compact":
            tol = 0.5 if w.radius is None else 0.04 * w.rg_target
            p = inputs.compact_chain(w.beads, rng, rg_target=w.rg_target, rg_tol=tol, radius=w.radius)
        elif w.geometry == "box":
            p = inputs.periodic_box(w.beads, w.box, rng)
        else:
            raise ValueError(w.geometry)
        out[r * w.beads:(r + 1) * w.beads] = p
    return out


def positions(w: Workload) -> np.ndarray:
    """float32-representable positions [n_atoms, 3] (float32 array)."""
    return _positions(w).astype(np.float32)


def types(w: Workload) -> np.ndarray:
    return inputs.bead_types(w.n_atoms, w.n_types, np.random.default_rng(w.seed + 777))


def weights(w: Workload, bias_scale: float = 0.0, seed_offset: int = 0) -> dict:
    return inputs.schnet_weights(np.random.default_rng(w.seed + 999 + seed_offset), w.n_types, w.F, w.K, w.L,
                                 bias_scale=bias_scale)


def masses(w: Workload) -> np.ndarray:
    return np.full(w.n_atoms, w.mass, dtype=np.float32)


def velocity_normals(w: Workload) -> np.ndarray:
    return inputs.standard_normals(w.n_atoms, np.random.default_rng(w.seed + 555))
