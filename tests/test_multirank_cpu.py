"""The N>1 path of bench.py on CPU: two gloo ranks, each with its own replica
batch (weak scaling, no data-path collective); whole-job time is the max over
ranks and the atom count the sum."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from schnet_gnn_molecular_b200 import workloads
    w = workloads.TINY
    pos, types, weights, mass, vel = bench._inputs(w, rank)
    ms_local = 10.0 + 5.0 * rank
    t_max, atoms, value = bench.aggregate_ranks(ms_local, w.n_atoms, 4, dist, "cpu")
    out[rank] = (t_max, atoms, value, float(pos[0, 0]), float(weights["W1"].ravel()[3]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_and_shard():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    r0, r1 = out[0], out[1]
    assert r0[0] == r1[0] == 15.0                 # slowest rank's time
    assert r0[1] == r1[1] == 2 * 64               # atoms of both ranks
    assert np.isclose(r0[2], 128 * 4 / 15e-3)
    assert r0[3] != r1[3]                          # each rank its own replica geometry
    assert r0[4] == r1[4]                          # the same model on every rank
