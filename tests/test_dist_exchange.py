"""The TSP exchange schedule (folded_tensor_sequence_rank_b200.exchange) on CPU
ranks over gloo, world sizes 2 and 3: each process holds only its own shards
(head group r, FFN block r) and its own zigzag tokens; the attention shards
arrive by broadcast, each head group's K/V by the zigzag all-gather, the FFN
blocks around the point-to-point ring.  An fp64 stand-in built from the
oracle's functions does each shard step, so the gathered outputs must equal
the oracle's unsharded layer to rounding."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from folded_tensor_sequence_rank_b200 import exchange, inputs
from oracle import tsp_oracle as O


class OracleShardCompute:
    """The shard steps in fp64 with the oracle's functions.  Shards are the
    math-orientation blocks: wq, wk, wv [h, h/D] (columns of head group k),
    wo [h/D, h] (its rows), w1 [h, F/D], w2 [F/D, h]."""

    def __init__(self, T, D, rank, h, H, F):
        self.T, self.D, self.rank, self.H = T, D, rank, H
        self.h, self.hs, self.Fs = h, h // D, F // D
        self.pos = O.zigzag_index(T, D, rank)
        self.scale = 1.0 / np.sqrt(h // H)
        self.shapes = {"wq": (h, self.hs), "wk": (h, self.hs), "wv": (h, self.hs), "wo": (self.hs, h),
                       "w1": (h, self.Fs), "w2": (self.Fs, h)}
        self.steps = []

    def empty_like_shard(self, n):
        return torch.zeros(self.shapes[n], dtype=torch.float64)

    def layernorm(self, x):
        return torch.from_numpy(O.layer_norm(x.numpy()))

    def residual(self, x):
        return x.clone()

    def clone(self, y):
        return y.clone()

    def qkv(self, k, wq, wk, wv, xn1):
        self.steps.append(("attn", k))
        kk = torch.zeros(self.T, self.hs, dtype=torch.float64)
        vv = torch.zeros_like(kk)
        kk[self.pos] = xn1 @ wk
        vv[self.pos] = xn1 @ wv
        return xn1 @ wq, kk, vv

    def attention(self, k, q, kk, vv):
        return torch.from_numpy(O.causal_attention(q.numpy(), kk.numpy(), vv.numpy(), self.pos, self.H // self.D,
                                                   self.scale))

    def ffn_up(self, w1, xn2):
        self.steps.append(("ffn", w1))
        return torch.from_numpy(O.gelu_tanh((xn2 @ w1).numpy()))

    def accumulate(self, y, act, w, which):
        y += act @ w


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, cfg, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        T, h, H, F = cfg
        D = world
        raw = inputs.layer_inputs(T, h, F, 17)
        x = raw["x"].double()
        w = {n: raw[n].double() for n in inputs.WEIGHT_NAMES}
        hs, Fs = h // D, F // D
        cols, fcols = slice(rank * hs, (rank + 1) * hs), slice(rank * Fs, (rank + 1) * Fs)
        own = {"wq": w["wq"][:, cols].contiguous(), "wk": w["wk"][:, cols].contiguous(),
               "wv": w["wv"][:, cols].contiguous(), "wo": w["wo"][cols, :].contiguous(),
               "w1": w["w1"][:, fcols].contiguous(), "w2": w["w2"][fcols, :].contiguous()}
        comp = OracleShardCompute(T, D, rank, h, H, F)
        idx = torch.from_numpy(O.zigzag_index(T, D, rank))
        ex = exchange.Exchange(rank, D)
        y = exchange.rank_forward_exchanged(ex, comp, x[idx].contiguous(), own, T // (2 * D))
        # the FFN blocks this rank applied, in order: (r + s) mod D
        seen = [int(np.argmax([np.array_equal(st[1].numpy(), w["w1"][:, k * Fs:(k + 1) * Fs].numpy())
                               for k in range(D)])) for st in comp.steps if st[0] == "ffn"]
        ys = [torch.zeros(T // D, h, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(ys, y)
        if rank == 0:
            full = np.zeros((T, h))
            for r in range(world):
                full[O.zigzag_index(T, D, r)] = ys[r].numpy()
            ref = O.layer_forward(x.numpy(), {n: a.numpy() for n, a in w.items()}, H, storage=None)["y"]
            out_q.put((float(np.abs(full - ref).max()), seen, [s[1] for s in comp.steps if s[0] == "attn"]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,cfg", [(2, (64, 64, 4, 256)), (3, (96, 48, 3, 192))])
def test_exchange_schedule_reproduces_the_layer(world, cfg):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cfg, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    err, seen, attn_order = q.get(timeout=5)
    assert err < 1e-10, err
    assert seen == [(0 + s) % world for s in range(world)]     # rank 0's ring order
    assert attn_order == list(range(world))                     # broadcast order
