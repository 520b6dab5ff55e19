#!/usr/bin/env python
"""Throughput of the SchNet energy + force + integrate path on B200.

One step = one BAOAB Langevin step of every replica (B-A-O-A, forward over all
interactions, backward for forces, closing B), with the neighbour list rebuilt
every n_rebuild steps (its cost amortised inside the timed steps).  Workload
(default): 64 replicas x 269-bead compact chains, F=128, 50 Gaussians on
0-15 A, cutoff 15 A, 3 interactions, skin 2 A, rebuild every 20 steps, dt 4 fs.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

With N > 1 (torchrun) every rank simulates its own replica batch (weak
scaling, no data-path collective); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "atom-steps/s & ns/day (SchNet E+F+integrate, 1 B200); HBM GB/s % of peak"
KB = 0.0019872041            # kcal/mol/K
ACC = 4.184e-4               # (kcal/mol/A)/amu -> A/fs^2
FWD_FLOP_PER_EDGE = None     # set from the workload: 2 (K F + F^2)


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle sampling (every 200 ms).  Started before the warm-up so
    that the tool is already polling when the timed region begins; ``stop(t0, t1)``
    keeps the samples whose timestamps fall inside [t0, t1] (host wall clock)."""

    def __init__(self, index=0):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(index), f"--query-gpu={q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        """End sampling and keep the samples (summarise windows with ``window``)."""
        self.rows = []
        if self.p is None:
            return self
        self.p.terminate()
        self.p.wait(timeout=10)
        self.f.flush()
        self.f.seek(0)
        for line in self.f.read().splitlines():
            t = [x.strip() for x in line.split(",")]
            if len(t) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(t[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                self.rows.append((ts, float(t[1]), float(t[2]), t[5:9]))
            except ValueError:
                continue
        os.unlink(self.f.name)
        return self

    def window(self, t0=None, t1=None):
        """Median SM clock, max clock and active throttle reasons of the samples in [t0, t1]."""
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = self.rows
        inside = [r for r in rows if t0 is None or (t0 <= r[0] <= t1)]
        window = "timed region"
        if not inside:                       # region shorter than the sampling period
            inside = [min(rows, key=lambda r: abs(r[0] - t1))] if rows and t1 is not None else rows
            window = "nearest sample to the end of the timed region"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = {n for r in inside for n, v in zip(names, r[3]) if v.lower().startswith("active")}
        sm = [r[1] for r in inside]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(r[2] for r in inside) if inside else None,
                "reasons": sorted(reasons), "samples": len(inside), "window": window}


def tensor_peak(peaks, clk):
    """Dense fp16/bf16 tensor peak for kernels timed under the clocks `clk`: the burst
    figure when the SM clock held its maximum with no power cap, else the sustained one."""
    burst = peaks.get("bf16_tflops")
    sustained = peaks.get("bf16_tflops_sustained", burst)
    full = (clk and clk.get("sm_mhz") and clk.get("sm_max_mhz") and clk["sm_mhz"] >= 0.97 * clk["sm_max_mhz"]
            and "sw_power_cap" not in clk.get("reasons", []))
    return (burst, "burst") if full else (sustained, "sustained")


# MUFU (special-function unit) operations counted from the kernel source: forward kernel, per
# directed edge -- one ex2 per evaluated Gaussian (K), and per feature one ex2 and one lg2 for the
# base-2 softplus, except that one feature pair in four takes its ex2 on the FMA pipe; pair
# kernel, per unordered pair -- K Gaussian ex2, per feature ex2 and lg2 for the softplus (one
# feature pair in four with its ex2 on the FMA pipe) and one more ex2 for the logistic.  148 SMs
# x 16 MUFU results per clock.
def mufu_per_edge(K, F):
    return {"fwd": K + 2 * F - F // 4, "bwd": K + 3 * F - F // 4}


def fused_work_per_step(K, F, L, E_cut):
    """Algorithmic FLOP and MUFU operations per MD step of the two fused kernels.  The filter
    network K -> F -> F costs 2 (K F + F^2) FLOP per evaluation.  k_cfconv_fwd evaluates it once
    per directed edge inside the cutoff in each interaction's forward (E_cut) and once per edge of
    the complementary list (E_cut / 2) in the dE/dh launches of interactions 1..L-1; k_cfconv_bwd
    forms W and its derivative W' (twice the contraction) per unordered pair (E_cut / 2) in every
    interaction."""
    f1 = 2.0 * (K * F + F * F)
    mu = mufu_per_edge(K, F)
    fwd_edges = (L + (L - 1) * 0.5) * E_cut
    return {"k_cfconv_fwd": {"classes": ("cfconv_fwd", "cfconv_dh"), "flop_step": f1 * fwd_edges,
                             "mufu_step": mu["fwd"] * fwd_edges},
            "k_cfconv_bwd": {"classes": ("cfconv_bwd",), "flop_step": 2.0 * f1 * L * E_cut / 2,
                             "mufu_step": mu["bwd"] * L * E_cut / 2}}


def hbm_kernel_bytes(w, E_list, E_cut):
    """Algorithmic HBM bytes of the memory-bound kernels (per launch; the neighbour build per
    build).  forces: per listed edge col, rev and s_e (4 B each), per atom the position (16 B),
    row pointer and slot map (8 B) and the force (16 B).  integrate: per atom and step, B-A-O-A
    reads slot map, mass, force, velocity, position, build reference (4+4+16+12+12+16 B) and
    writes velocity, position, slot-order position (12+12+16 B); the closing B reads mass, force,
    velocity (4+16+12 B) and writes velocity and kinetic energy (12+4 B).  mask: per listed edge
    its row and column (8 B), per edge inside the cutoff row, column, index (12 B).  neighbours:
    positions in (12 B per atom), col and rev out (8 B per listed edge), row pointers (4 B per atom)."""
    N = w.n_atoms
    return {"forces": 12 * E_list + 40 * N,
            "integrate": (104 + 48) * N,
            "mask": 8 * E_list + 12 * E_cut,
            "neighbors": 12 * N + 8 * E_list + 4 * N}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def aggregate_ranks(ms_local: float, atoms_local: int, steps: int, dist=None, device=None):
    """Whole-job timing over ranks: the slowest rank's device time and the atoms
    advanced by all ranks.  Returns (max_ms, total_atoms, atom_steps_per_s)."""
    import torch
    ms, atoms = float(ms_local), int(atoms_local)
    if dist is not None and dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=device)
        a = torch.tensor([atoms], dtype=torch.int64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(a, op=dist.ReduceOp.SUM)
        ms, atoms = float(t.item()), int(a.item())
    return ms, atoms, atoms * steps / (ms * 1e-3)


def _workload(name):
    from schnet_gnn_molecular_b200 import workloads
    if name in workloads.ALL:
        return workloads.ALL[name]
    if name.startswith("cg_protein_") and name.endswith("x269"):
        return workloads.sweep(int(name[len("cg_protein_"):-len("x269")]))
    if name.startswith("cg_globule_"):
        return workloads.globule(int(name[len("cg_globule_"):]))
    if name.startswith("periodic_box_") and name[len("periodic_box_"):].isdigit():
        # the 10^6-bead box's model and density, n beads
        n = int(name[len("periodic_box_"):])
        return workloads.BOX1M.with_(name=name, beads=n, box=(n / workloads.BOX1M.density) ** (1.0 / 3.0))
    raise SystemExit(f"unknown workload {name}")


def _inputs(w, rank):
    from schnet_gnn_molecular_b200 import workloads
    wr = w.with_(seed=w.seed + 100000 * rank) if rank else w
    pos = workloads.positions(wr)
    types = workloads.types(wr)
    weights = workloads.weights(w)            # same model on every rank
    mass = workloads.masses(wr)
    vel = (workloads.velocity_normals(wr) * np.sqrt(KB * w.temperature * ACC / w.mass)).astype(np.float32)
    return pos, types, weights, mass, vel


def cpu_baseline(w, seconds: float):
    """The float64 oracle timed on this host on whole replicas (one MD step each)."""
    import oracle
    from schnet_gnn_molecular_b200 import workloads
    pos, types, weights, mass, vel = _inputs(w, 0)
    om = oracle.Model(n_types=w.n_types, F=w.F, K=w.K, L=w.L, rbf_min=w.rbf_min, rbf_max=w.rbf_max,
                      rbf_sigma=w.rbf_sigma, cutoff=w.cutoff, weights=weights, periodic=w.periodic,
                      box=(w.box,) * 3 if w.periodic else (0.0, 0.0, 0.0))
    oracle.lib()
    cores = len(os.sched_getaffinity(0))
    atoms, t0, reps = 0, time.perf_counter(), 0
    if w.periodic:
        # a ball of radius L r_c around one bead, unwrapped by the minimum image: one force
        # evaluation of a ~2k-bead open cluster with the workload's density and model
        om_open = oracle.Model(n_types=w.n_types, F=w.F, K=w.K, L=w.L, rbf_min=w.rbf_min, rbf_max=w.rbf_max,
                               rbf_sigma=w.rbf_sigma, cutoff=w.cutoff, weights=weights)
        rad = w.L * w.cutoff
        dt = 0.0
        while True:
            c = (reps * 7919) % w.n_atoms
            d = pos.astype(np.float64) - pos[c].astype(np.float64)
            d -= w.box * np.rint(d / w.box)
            sel = np.flatnonzero((d * d).sum(1) < rad * rad)
            x = pos[c].astype(np.float64) + d[sel]
            t1 = time.perf_counter()
            oracle.energy_forces(om_open, x, types[sel])
            dt += time.perf_counter() - t1
            atoms += len(sel)
            reps += 1
            if dt >= seconds:
                break
        return {"value": atoms / dt, "unit": "atom-steps/s", "cores": cores, "kind": "oracle",
                "sample": f"{reps} energy+force evaluations of open balls of radius {rad:.0f} A "
                          f"({atoms // reps} beads on average) cut from this box, {dt:.1f} s timed"}
    dt = 0.0
    while True:
        r = reps % w.n_replicas
        sl = slice(r * w.beads, (r + 1) * w.beads)
        x = pos[sl].astype(np.float64)
        _, _, F = oracle.energy_forces(om, x, types[sl])          # forces at the start (not timed)
        t1 = time.perf_counter()
        oracle.md_step(om, x, vel[sl].astype(np.float64), types[sl], mass[sl].astype(np.float64), F, w.dt_fs,
                       w.gamma_per_ps, w.temperature, 1, reps)
        dt += time.perf_counter() - t1
        atoms += w.beads
        reps += 1
        if dt >= seconds:
            break
    return {"value": atoms / dt, "unit": "atom-steps/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} BAOAB steps, each of one whole {w.beads}-bead replica of this workload, "
                      f"{dt:.1f} s timed"}


def _edge_stats(model, pos, w):
    """Listed and within-cutoff directed edges of the current list (host-side count)."""
    rp, col, _ = model.neighbors()
    rows = np.repeat(np.arange(w.n_atoms), np.diff(rp))
    p = pos.astype(np.float64)
    v = p[col] - p[rows]
    if w.periodic:
        v -= w.box * np.rint(v / w.box)
    d = np.sqrt((v * v).sum(1))
    return int(len(col)), int((d < w.cutoff).sum())


def _traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu capture, or None when
    the kernel sources have changed since that capture (hash recorded beside the figure)."""
    import hashlib
    try:
        d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
        h = hashlib.sha256()
        for src in d["sources"]:
            h.update(open(os.path.join(ROOT, src), "rb").read())
        if h.hexdigest()[:16] != d["sources_sha256_16"]:
            return None
        return d.get(kernel)
    except Exception:
        return None


def nat_status(st):
    from schnet_gnn_molecular_b200 import _native
    return _native.STATUS_NAMES.get(int(st), str(st))


def run_native(args):
    import torch
    import torch.distributed as dist
    from schnet_gnn_molecular_b200 import api

    ws, rank, local = _dist()
    if ws > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    torch.cuda.set_device(local)
    w = _workload(args.workload)
    pos, types, weights, mass, vel = _inputs(w, rank)
    n_rb = w.n_rebuild
    steps = int(args.steps)
    model = api.from_workload(w, weights, device=f"cuda:{local}", edge_capacity=args.edge_capacity)
    dev = torch.device(f"cuda:{local}")
    p = torch.tensor(pos, device=dev)
    v = torch.tensor(vel, device=dev)
    t = torch.tensor(types, device=dev)
    m = torch.tensor(mass, device=dev)
    kw = dict(dt=w.dt_fs, gamma=w.gamma_per_ps, temperature=w.temperature, n_rebuild=n_rb, seed=1234)
    # warm-up: initial build + forces, graph capture, W steps
    clocks = ClockSampler(local) if rank == 0 else None
    flagged = []
    _, _, st = model.step(p, v, t, m, args.warmup, step0=0, raise_on_flag=False, **kw)
    flagged.append(st)
    torch.cuda.synchronize()

    edges_start = _edge_stats(model, p.cpu().numpy(), w) if rank == 0 else None
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    l0 = model.kernel_launches()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wall0 = time.time()
    ev0.record()
    _, _, st = model.step(p, v, t, m, steps, step0=args.warmup, resume=True, raise_on_flag=False, **kw)
    ev1.record()
    flagged.append(st)
    torch.cuda.synchronize()
    wall1 = time.time()
    if ws > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    launches = model.kernel_launches() - l0
    free_b, total_b = torch.cuda.mem_get_info(dev)
    memory = {"workspace_MB": round(model.workspace_bytes / 1e6, 1),
              "torch_peak_allocated_MB": round(torch.cuda.max_memory_allocated(dev) / 1e6, 1),
              "device_used_MB": round((total_b - free_b) / 1e6, 1),
              "note": "device_used includes the CUDA context, the library image and the captured graphs"}
    t_max, atoms_total, value = aggregate_ranks(ms, w.n_atoms, steps, dist, dev)
    step_s = t_max * 1e-3 / steps
    ns_day_rep = (1.0 / step_s) * w.dt_fs * 86400 * 1e-6

    out = None
    if rank == 0:
        # per-kernel device times on the library stream (eager profiling pass, same trajectory)
        prof_t0 = time.time()
        prof = model.profile_steps(p, v, t, m, n_rb, step0=args.warmup + steps, **kw)
        prof_t1 = time.time()
        clocks.stop()
        clk = clocks.window(wall0, wall1)
        clk_prof = clocks.window(prof_t0, prof_t1)
        E_list, E_cut = _edge_stats(model, p.cpu().numpy(), w)
        peaks, src = _peaks()
        # algorithmic work per step (45,568 FLOP per filter evaluation for the 64 x 269 model)
        kern = fused_work_per_step(w.K, w.F, w.L, E_cut)
        for k, v in kern.items():
            v["ms"] = sum(prof[c][0] for c in v["classes"])        # over the n_rb profiled steps
            v["launches"] = sum(prof[c][1] for c in v["classes"])
            v["ms_per_launch"] = v["ms"] / max(v["launches"], 1)
            v["flop_launch"] = v["flop_step"] * n_rb / max(v["launches"], 1)
            v["mufu"] = v["mufu_step"] * n_rb / max(v["launches"], 1)
        per_launch = {k: x[0] / max(x[1], 1) for k, x in prof.items()}
        per_step = {k: x[0] / n_rb for k, x in prof.items()}
        tot_ms = sum(x[0] for x in prof.values())
        dominant = max(kern, key=lambda k: kern[k]["ms"])
        kms = kern[dominant]["ms_per_launch"]
        flops = kern[dominant]["flop_launch"]
        peak, peak_kind = tensor_peak(peaks, clk_prof)
        achieved = flops / (kms * 1e-3) / 1e12
        traffic = _traffic(dominant)
        # end-to-end roofline: per kernel class the slowest of its tensor, MUFU and HBM bounds
        hbm = peaks["hbm_gbs"] * 1e9
        f_clk = (clk_prof.get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)) * 1e6
        mufu_peak = 148 * 16 * f_clk
        hb = hbm_kernel_bytes(w, E_list, E_cut)
        n_aw = 6 * w.L                                    # atom-wise layer applications per step
        fw, bw = kern["k_cfconv_fwd"], kern["k_cfconv_bwd"]
        share_dh = (w.L - 1) * 0.5 / (w.L + (w.L - 1) * 0.5)     # the dE/dh launches' part of fw
        fw_bound = max(fw["flop_step"] / (peak * 1e12), fw["mufu_step"] / mufu_peak)
        bounds = {
            "cfconv_fwd": fw_bound * (1.0 - share_dh),
            "cfconv_dh": fw_bound * share_dh,
            "cfconv_bwd": max(bw["flop_step"] / (peak * 1e12), bw["mufu_step"] / mufu_peak),
            "atomwise": max(n_aw * 2.0 * w.F * w.F * w.n_atoms / (peak * 1e12),
                            n_aw * 2 * w.n_atoms * w.F * 4 / hbm),
            "forces": hb["forces"] / hbm, "integrate": hb["integrate"] / hbm, "mask": hb["mask"] / hbm,
            "neighbors": hb["neighbors"] / hbm / n_rb, "reduce": 8 * w.n_atoms / hbm}
        bound_ms = {k: v * 1e3 for k, v in bounds.items()}
        e2e_frac = sum(bound_ms.values()) / (step_s * 1e3)
        hbm_kernels = {}
        for k in ("forces", "integrate", "mask", "neighbors"):
            ms_k = per_launch[k] if k == "neighbors" else per_step[k]
            gbs = hb[k] / (ms_k * 1e-3) / 1e9 if ms_k > 0 else None
            hbm_kernels[k] = {"bytes": int(hb[k]), "per": "build" if k == "neighbors" else "step",
                              "ms": round(ms_k, 5), "achieved_GBs": round(gbs, 1) if gbs else None,
                              "frac": round(gbs / peaks["hbm_gbs"], 4) if gbs else None}
        k_interval = max(1, int(round(launches / steps * n_rb)))
        floor = {"ms_per_step": round(_launch_floor(dev, k_interval) / n_rb, 4),
                 "kernels_per_step": round(launches / steps, 2),
                 "how": f"one CUDA Graph of {k_interval} trivial kernels (one rebuild interval's count), "
                        f"replayed; per step = replay time / {n_rb}"}
        fused = {k: {"launches_per_step": round(v["launches"] / n_rb, 2), "ms_per_launch": round(v["ms_per_launch"], 4),
                     "flop_per_launch": v["flop_launch"],
                     "tflops": round(v["flop_launch"] / (v["ms_per_launch"] * 1e-3) / 1e12, 2),
                     "frac_tensor": round(v["flop_launch"] / (v["ms_per_launch"] * 1e-3) / 1e12 / peak, 4),
                     "mufu_per_launch": v["mufu"],
                     "frac_mufu": round(v["mufu"] / (v["ms_per_launch"] * 1e-3) / mufu_peak, 4)}
                 for k, v in kern.items()}
        roofline = {"bound": "tensor", "kernel": dominant, "achieved": round(achieved, 2),
                    "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                    "peak_source": f"{src} dense bf16/fp16 {peak_kind} (per-kernel times taken at "
                                   f"{clk_prof.get('sm_mhz')} MHz, reasons {clk_prof.get('reasons')})",
                    "flop_per_launch": flops, "ms_per_launch": round(kms, 4),
                    "per_kernel_ms_per_step": {k: round(x, 4) for k, x in per_step.items()},
                    "kernel_share": {k: round(x[0] / tot_ms, 4) for k, x in prof.items()},
                    "e2e_frac": round(e2e_frac, 4),
                    "e2e_bound_ms_per_step": {k: round(x, 4) for k, x in bound_ms.items()},
                    "e2e_how": "sum over kernel classes of max(tensor FLOP / tensor peak, MUFU ops / MUFU peak, "
                               "algorithmic HBM bytes / HBM peak), divided by the measured ms_per_step",
                    "fused_kernels": fused,
                    "mufu_per_edge_interaction": mufu_per_edge(w.K, w.F), "mufu_peak_per_s": mufu_peak,
                    "hbm_peak_GBs": peaks["hbm_gbs"], "hbm_kernels": hbm_kernels}
        cfg = dict(_workload_config(w, n_rb, ws))
        cfg.update({"edges_listed": E_list, "edges_within_cutoff": E_cut,
               "edges_within_cutoff_at_start": edges_start[1],
               "edges_note": "no bonded terms: chains slowly expand, so the graph shrinks during the run; "
                             "edges_within_cutoff is counted after the timed steps",
               "l2": "no flush: state carried step to step; per-step working set "
                     f"{(E_list * 20 + w.n_atoms * 128 * 4 * (2 * w.L + 4)) / 1e6:.0f} MB > 126 MB L2"})
        out = {"metric": METRIC, "value": round(value, 1), "unit": "atom-steps/s", "n_gpus": ws, "steps": steps,
               "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 4), "higher_is_better": True,
               "scaling": "weak", "vs_baseline": None, "dtype": "f32",
               "mma": "fp16 hi/lo split operands, fp32 accumulate (tcgen05 kind::f16)", "data": "synthetic",
               "ns_per_day_per_replica": round(ns_day_rep, 2),
               "ns_per_day_aggregate": round(ns_day_rep * w.n_replicas * ws, 1),
               "config": cfg, "gpu_launches": int(launches), "launch_floor": floor, "clocks": clk,
               "clocks_profile_pass": clk_prof,
               "roofline": roofline,
               "memory": memory,
               "status": {"warmup": nat_status(flagged[0]), "timed": nat_status(flagged[1])}}
    if not args.no_e2e:
        # every rank drives its own GPU through the host-buffer entry point; the job's
        # rate is all ranks' atom-steps over the slowest rank's wall time
        if ws > 1:
            dist.barrier()
        sec, n_e, h2d, d2h = e2e(model, w, pos, vel, types, mass, kw, args)
        t_e, _, v_e = aggregate_ranks(sec * 1e3, w.n_atoms, n_e, dist, dev)
        if rank == 0:
            out["e2e"] = {"value": round(v_e, 1), "unit": "atom-steps/s", "h2d_bytes_per_step": int(h2d),
                          "d2h_bytes_per_step": int(d2h), "steps": n_e, "ms_per_step": round(t_e / n_e, 4),
                          "how": "schnet_step_host, one step per call, pinned host buffers, wall clock, "
                                 "slowest rank"}
    if rank == 0 and not args.no_cpu_baseline and ws == 1:
        out["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    model.close()
    if out is not None:
        print(json.dumps(out), flush=True)


def e2e(model, w, pos, vel, types, mass, kw, args):
    """Same metric through the host-buffer entry point: every step copies the step's inputs
    from pinned host memory and reads the step's results back (schnet_step_host, one step per call).
    Returns (seconds, steps, host-to-device bytes per step, device-to-host bytes per step)."""
    import torch
    hp = torch.from_numpy(pos.copy()).pin_memory().numpy()
    hv = torch.from_numpy(vel.copy()).pin_memory().numpy()
    ht = torch.from_numpy(types.copy()).pin_memory().numpy()
    hm = torch.from_numpy(mass.copy()).pin_memory().numpy()
    ep = torch.empty(w.n_replicas, dtype=torch.float64).pin_memory().numpy()
    ek = torch.empty(w.n_replicas, dtype=torch.float64).pin_memory().numpy()
    model.step_host(hp, hv, ht, hm, 0, step0=0, resume=False, epot=ep, ekin=ek, **kw)  # initial forces
    n = max(w.n_rebuild, int(args.e2e_steps))
    for s in range(3):
        model.step_host(hp, hv, ht, hm, 1, step0=s, resume=True, epot=ep, ekin=ek, **kw)
    t0 = time.perf_counter()
    for s in range(n):
        model.step_host(hp, hv, ht, hm, 1, step0=3 + s, resume=True, epot=ep, ekin=ek, **kw)
    dt = time.perf_counter() - t0
    h2d = hp.nbytes + hv.nbytes + ht.nbytes + hm.nbytes
    d2h = hp.nbytes + hv.nbytes + ep.nbytes + ek.nbytes
    return dt, n, h2d, d2h


def run_drift(args):
    """NVE drift: velocity Verlet (gamma = 0) on the workload for --drift-steps steps;
    total energy (potential + kinetic, summed over replicas) read after every rebuild
    interval; reported as the least-squares slope per atom, over the whole run and per
    window of --drift-window steps, with the within-cutoff edge count at every window
    boundary (the chains have no bonded terms and slowly fly apart, so the graph
    shrinks; the slope over the leading windows whose graph keeps >= 90 % of its
    starting edges is the one measured on an intact graph)."""
    import torch
    from schnet_gnn_molecular_b200 import api
    w = _workload(args.workload).with_(gamma_per_ps=0.0)
    pos, types, weights, mass, vel = _inputs(w, 0)
    dev = torch.device("cuda:0")
    model = api.from_workload(w, weights, device="cuda:0", edge_capacity=args.edge_capacity)
    p, v = torch.tensor(pos, device=dev), torch.tensor(vel, device=dev)
    t, m = torch.tensor(types, device=dev), torch.tensor(mass, device=dev)
    kw = dict(dt=w.dt_fs, gamma=0.0, temperature=w.temperature, n_rebuild=w.n_rebuild, seed=1234)
    chunk = w.n_rebuild
    n_chunks = max(1, args.drift_steps // chunk)
    win_chunks = max(1, args.drift_window // chunk)
    ep, _, st = model.step(p, v, t, m, 0, step0=0, raise_on_flag=False, **kw)   # initial forces
    edges = [(0, _edge_stats(model, pos, w)[1])]
    ek0 = 0.5 * float((mass.astype(np.float64)[:, None] * vel.astype(np.float64) ** 2).sum()) / ACC
    times, etot, flags = [0.0], [float(ep.sum()) + ek0], int(st)
    ms = 0.0
    for c in range(n_chunks):
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        ep, ek, st = model.step(p, v, t, m, chunk, step0=c * chunk, resume=c > 0, raise_on_flag=False, **kw)
        ev1.record()
        torch.cuda.synchronize()
        ms += ev0.elapsed_time(ev1)
        flags |= int(st)
        times.append((c + 1) * chunk * w.dt_fs * 1e-6)          # ns
        etot.append(float((ep + ek).sum()))
        if (c + 1) % win_chunks == 0 or c == n_chunks - 1:
            # the list of the last rebuild covers every pair within the cutoff at these positions
            edges.append(((c + 1) * chunk, _edge_stats(model, p.cpu().numpy(), w)[1]))
    tt, ee = np.array(times), np.array(etot) / w.n_atoms
    kcal_to_uev = 4.3364e4                   # 1 kcal/mol = 43.364 meV

    def fit(a, b):
        sl, ic = np.polyfit(tt[a:b + 1], ee[a:b + 1], 1)
        res = ee[a:b + 1] - (sl * tt[a:b + 1] + ic)
        return float(sl), float(np.sqrt((res ** 2).mean()))

    slope, rms = fit(0, len(tt) - 1)
    windows, intact_end = [], 0
    for (s0, e0), (s1, e1) in zip(edges[:-1], edges[1:]):
        sl, _ = fit(s0 // chunk, s1 // chunk)
        windows.append({"steps": [s0, s1], "slope_kcal_mol_atom_ns": sl, "slope_ueV_atom_ps": sl * kcal_to_uev / 1e3,
                        "edges_within_cutoff": [e0, e1]})
        if intact_end == s0 and min(e0, e1) >= 0.9 * edges[0][1]:
            intact_end = s1
    intact = None
    if intact_end > 0:
        sl, r = fit(0, intact_end // chunk)
        intact = {"steps": [0, intact_end], "slope_kcal_mol_atom_ns": sl, "slope_ueV_atom_ps": sl * kcal_to_uev / 1e3,
                  "rms_about_fit_kcal_mol_atom": r,
                  "edges_within_cutoff_min": int(min(e for s_, e in edges if s_ <= intact_end))}
    ekin0 = float(ek.sum()) / w.n_atoms
    out = {"metric": "NVE energy drift (velocity Verlet)", "value": slope, "unit": "kcal/mol/atom/ns",
           "ueV_per_atom_per_ps": slope * kcal_to_uev / 1e3, "steps": n_chunks * chunk,
           "dt_fs": w.dt_fs, "simulated_ns": float(tt[-1]), "higher_is_better": False,
           "etot_per_atom_first_last": [float(ee[0]), float(ee[-1])],
           "etot_per_atom_rms_about_fit": rms, "ekin_per_atom_last": ekin0, "status": nat_status(flags),
           "ms_per_step": round(ms / (n_chunks * chunk), 4),
           "intact_graph": intact, "windows": windows,
           "edges_within_cutoff_first_last": [edges[0][1], edges[-1][1]],
           "note": "no bonded terms: the chains expand during the run, so the graph shrinks; 'intact_graph' is "
                   "the fit over the leading windows that keep >= 90 % of the starting edges",
           "config": {"workload": w.name, "replicas": w.n_replicas, "atoms": w.n_atoms, "n_rebuild": w.n_rebuild,
                      "skin_A": w.skin, "read_every_steps": chunk, "window_steps": win_chunks * chunk},
           "data": "synthetic"}
    model.close()
    print(json.dumps(out), flush=True)


def _launch_floor(dev, kernels, reps=20):
    """Device time of one CUDA Graph of `kernels` trivial one-element kernels (the
    replay floor a graph of that many nodes cannot beat on this GPU), in ms."""
    import torch
    x = torch.zeros(1, device=dev)
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        x.add_(1.0)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(kernels):
            x.add_(1.0)
    g.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / reps
    del g
    return ms


def _workload_config(w, n_rebuild, ranks):
    """The static description of a workload, shared by both arms' `config`."""
    return {"workload": w.name, "replicas": w.n_replicas, "beads_per_replica": w.beads, "atoms": w.n_atoms,
            "F": w.F, "K": w.K, "L": w.L, "cutoff_A": w.cutoff, "skin_A": w.skin, "n_rebuild": n_rebuild,
            "dt_fs": w.dt_fs, "integrator": "BAOAB" if w.gamma_per_ps > 0 else "velocity Verlet",
            "weight_dtype": w.weight_dtype, "parallelism": f"replicas x{ranks} ranks (independent)"}


def run_reference(args):
    """The float64 oracle as the reference arm (rank 0 only).  One step = one BAOAB
    step of a replica-shaped sample: a whole replica when the run fits the time
    budget, else the first n beads of replica 0 (a contiguous chain segment)."""
    ws, rank, _ = _dist()
    if rank != 0:
        return
    w = _workload(args.workload)
    import oracle
    pos, types, weights, mass, vel = _inputs(w, 0)
    om = oracle.Model(n_types=w.n_types, F=w.F, K=w.K, L=w.L, rbf_min=w.rbf_min, rbf_max=w.rbf_max,
                      rbf_sigma=w.rbf_sigma, cutoff=w.cutoff, weights=weights)
    oracle.lib()
    cores = len(os.sched_getaffinity(0))

    def sample(nb):
        sl = slice(0, nb)
        x = pos[sl].astype(np.float64); vv = vel[sl].astype(np.float64); ms = mass[sl].astype(np.float64)
        _, _, F = oracle.energy_forces(om, x, types[sl])
        return sl, x, vv, ms, F

    # calibrate one whole-replica step (not counted), then size the per-step sample
    sl, x, vv, ms, F = sample(w.beads)
    t0 = time.perf_counter()
    oracle.md_step(om, x, vv, types[sl], ms, F, w.dt_fs, w.gamma_per_ps, w.temperature, 1, 0)
    t_unit = time.perf_counter() - t0
    nb = w.beads
    total = (args.steps + args.warmup) * t_unit
    if total > args.ref_budget:
        nb = max(16, int(w.beads * (args.ref_budget / total) ** 0.5))
    sl, x, vv, ms, F = sample(nb)
    for s in range(args.warmup):
        x, vv, F, _, _ = oracle.md_step(om, x, vv, types[sl], ms, F, w.dt_fs, w.gamma_per_ps, w.temperature, 1, s)
    t0 = time.perf_counter()
    for s in range(args.steps):
        x, vv, F, _, _ = oracle.md_step(om, x, vv, types[sl], ms, F, w.dt_fs, w.gamma_per_ps, w.temperature, 1,
                                        args.warmup + s)
    dt = time.perf_counter() - t0
    value = nb * args.steps / dt
    what = (f"replica 0 of {w.n_replicas} ({w.beads} beads)" if nb == w.beads else
            f"first {nb} of the {w.beads} beads of replica 0 (chain segment; time budget)")
    out = {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "atom-steps/s", "n_gpus": ws,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": dict(_workload_config(w, w.n_rebuild, ws),
                          sample=what),
           "cpu_baseline": {"value": round(value, 2), "unit": "atom-steps/s", "cores": cores, "kind": "oracle",
                            "sample": f"{args.steps} BAOAB steps of {what}"},
           "e2e": {"value": round(value, 2), "unit": "atom-steps/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=40)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="cg_protein_64x269")
    ap.add_argument("--edge-capacity", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=40)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=150.0, help="seconds for the reference arm's timed steps")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--nve-drift", action="store_true", help="measure NVE energy drift instead of throughput")
    ap.add_argument("--drift-steps", type=int, default=10000)
    ap.add_argument("--drift-window", type=int, default=100)
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.nve_drift:
        run_drift(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
