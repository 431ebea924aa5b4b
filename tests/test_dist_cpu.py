"""The multi-process path on CPU (gloo, world size 2): each process runs its
own TSP rank of a tiny layer (with the oracle standing in for the GPU step),
the timing reduction takes the maximum over ranks, and the ranks' outputs,
gathered and put back at their zigzag positions, equal the unsharded layer."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from folded_tensor_sequence_rank_b200 import dist as tdist
from folded_tensor_sequence_rank_b200 import inputs
from oracle import tsp_oracle as O

T, h, H, F, D = 64, 64, 4, 256, 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w_, g_, l_ = tdist.world_info()
        assert (w_, g_, l_) == (world, rank, rank)
        r = tdist.tsp_rank_for(g_, D)
        raw = inputs.layer_inputs(T, h, F, 3)
        x = raw["x"].double().numpy()
        w = {n: raw[n].double().numpy() for n in inputs.WEIGHT_NAMES}
        K, V = O.kv_all_gather_sharded(x, D, w)
        idx = O.zigzag_index(T, D, r)
        y = O.rank_forward_sharded(r, D, x[idx], K, V, w, H)
        ys = [torch.zeros(T // D, h, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(ys, torch.from_numpy(np.ascontiguousarray(y)))
        mx = tdist.max_over_ranks([10.0 * (rank + 1), -rank])
        if rank == 0:
            full = np.zeros((T, h))
            for gr in range(world):
                full[O.zigzag_index(T, D, tdist.tsp_rank_for(gr, D))] = ys[gr].numpy()
            ref = O.layer_forward(x, w, H)["y"]
            out_q.put((float(np.abs(full - ref).max()), mx))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_process_ranks_reassemble_the_layer():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    err, mx = q.get(timeout=5)
    assert err < 1e-10
    assert mx == [20.0, 0.0]


def test_rank_plan_cycles_through_ranks():
    assert [tdist.tsp_rank_for(g, 8) for g in range(10)] == [0, 1, 2, 3, 4, 5, 6, 7, 0, 1]
    with pytest.raises(ValueError):
        tdist.tsp_rank_for(0, 0)
    assert tdist.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
