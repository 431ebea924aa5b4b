"""The exchange schedule (exchange.rank_forward_exchanged) driving the CUDA
per-shard steps over a real NCCL process group.  Every call on this machine
gets one GPU, and ranks that wait on one another must not share a GPU, so the
group has one rank: D = 1, where the broadcast is from the rank to itself,
the all-gather has one part and the ring has no step.  What runs is the
composition the multi-GPU path uses - NCCL collectives on the layer's own
buffers between the library's per-shard launches - checked against the
oracle with the layer's gates."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from folded_tensor_sequence_rank_b200 import build as tsp_build
from folded_tensor_sequence_rank_b200 import exchange, inputs, tsp
from oracle import tsp_oracle as O

pytestmark = pytest.mark.gpu


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("T,h,H,F,seed", [(512, 256, 4, 1024, 80), (1024, 512, 4, 2048, 81)])
def test_exchange_over_nccl_world_one(T, h, H, F, seed):
    tsp_build.build()
    tsp.lib()
    torch.cuda.set_device(0)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_port()))
    from datetime import timedelta
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        D = 1
        raw = inputs.layer_inputs(T, h, F, seed)
        dev = {k: v.cuda() for k, v in raw.items()}
        dims = tsp.make_dims(T, h, H, F)
        sw = tsp.pack_shards(dims, D, dev)
        comp = exchange.GpuShardCompute(dims, D, 0)
        own = {n: sw.shard(n, 0, comp.shapes[n]).clone() for n in ("wq", "wk", "wv", "wo", "w1", "w2")}
        x = dev["x"].index_select(0, tsp.zigzag_index(T, D, 0).long()).contiguous()
        y = exchange.rank_forward_exchanged(exchange.Exchange(0, D), comp, x, own, T // 2)
        torch.cuda.synchronize()
        assert tsp.get_device_status(comp.ws) == tsp.TSP_OK
        got = y.double().cpu().numpy()
        xr = raw["x"].double().numpy()
        w = {n: raw[n].double().numpy() for n in inputs.WEIGHT_NAMES}
        for storage in (None, "fp16"):
            ref = O.layer_forward(xr, w, H, storage=storage)["y"]
            err = float(np.abs(got - ref).max())
            rl = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
            print(f"exchange over NCCL, T={T}, oracle storage={storage}: max-abs {err:.3e} rel-L2 {rl:.3e}")
            assert err <= 2e-2 and rl <= 5e-3
    finally:
        dist.destroy_process_group()
