"""The TSP exchange across D GPUs: what moves between ranks, and when.

The TSP news item (zubnet.ai, paragraph 2) gives the communication of one
layer on the folded TP+SP axis of D ranks, each holding 1/D of the weights
(head group k, FFN block k: shard k lives on rank k) and 1/D of the tokens
(zigzag chunks r and 2D-1-r):

* attention: the weight shards are broadcast one after another; every rank
  applies each shard to its own tokens; K and V are all-gathered under the
  zigzag partition (here per head group, right after the group's
  projection);
* MLP: the shards travel around a ring point to point - at step s rank r
  holds FFN block (r + s) mod D, passes it to rank r - 1 and receives the
  next from rank r + 1 - and each rank adds up its blocks' contributions
  locally, so no all-reduce is needed.

``rank_forward_exchanged`` runs that schedule for one rank over a
``torch.distributed`` process group (NCCL on GPUs), calling a compute object
per shard step.  The next attention shard's broadcast and the next FFN
block's ring transfer are posted before the current shard's compute, so
they overlap it; the head group's K/V all-gather sits between its projection
and its attention.  ``GpuShardCompute`` runs the steps in the CUDA library's
per-shard calls (tsp_shard_*); every tensor a kernel reads through TMA is in
this GPU's own memory (collectives copy into local buffers first).
"""
from __future__ import annotations

import ctypes

import torch
import torch.distributed as dist

from . import tsp

ATTN_NAMES = ("wq", "wk", "wv", "wo")
FFN_NAMES = ("w1", "w2")


class Exchange:
    """The collectives of one TSP rank in a group of D ranks."""

    def __init__(self, rank: int, D: int, group=None):
        self.rank, self.D, self.group = rank, D, group

    def broadcast(self, tensors, src: int, async_op: bool = False):
        """Shard `src`'s tensors from their owner to every rank."""
        return [dist.broadcast(t, src, group=self.group, async_op=async_op) for t in tensors]

    def all_gather_zigzag(self, full: torch.Tensor, c: int):
        """`full` [2Dc, cols] holds this rank's rows - chunks r and 2D-1-r - at
        their global positions; fill in every other rank's.  Chunks 0..D-1
        belong to ranks 0..D-1 and chunks D..2D-1 to ranks D-1..0, so each half
        is one all-gather into row views of `full`."""
        D, r = self.D, self.rank
        lo = [full[j * c:(j + 1) * c] for j in range(D)]
        hi = [full[(2 * D - 1 - j) * c:(2 * D - j) * c] for j in range(D)]
        dist.all_gather(lo, lo[r].clone(), group=self.group)
        dist.all_gather(hi, hi[r].clone(), group=self.group)

    def ring(self, send, recv):
        """Post the ring step: `send` to rank r-1, `recv` from rank r+1."""
        D, r = self.D, self.rank
        prev_r, next_r = (r - 1) % D, (r + 1) % D
        ops = [dist.P2POp(dist.isend, t, prev_r, group=self.group) for t in send]
        ops += [dist.P2POp(dist.irecv, t, next_r, group=self.group) for t in recv]
        return dist.batch_isend_irecv(ops)


def rank_forward_exchanged(ex: Exchange, comp, x_local, own: dict, c: int):
    """Rank ex.rank's layer output for its tokens x_local (rank-local order),
    given only its own shards `own` (name -> tensor) and the group's
    collectives.  Returns the output in the compute object's format."""
    D, r = ex.D, ex.rank
    xn1 = comp.layernorm(x_local)
    y1 = comp.residual(x_local)
    # attention: shard k is broadcast by its owner, the next one in flight
    # while this one is applied
    bufs = [[own[n] if k == r else comp.empty_like_shard(n) for n in ATTN_NAMES] for k in range(D)]
    pending = ex.broadcast(bufs[0], 0, async_op=True)
    for k in range(D):
        for h in pending:
            h.wait()
        if k + 1 < D:
            pending = ex.broadcast(bufs[k + 1], k + 1, async_op=True)
        wq, wk, wv, wo = bufs[k]
        q_k, k_k, v_k = comp.qkv(k, wq, wk, wv, xn1)
        ex.all_gather_zigzag(k_k, c)
        ex.all_gather_zigzag(v_k, c)
        a_k = comp.attention(k, q_k, k_k, v_k)
        comp.accumulate(y1, a_k, wo, "attn")
        bufs[k] = None if k != r else bufs[k]
    # MLP: FFN block (r + s) mod D at step s, the next one arriving from rank
    # r + 1 while this one is applied
    xn2 = comp.layernorm(y1)
    y = comp.clone(y1)
    cur = [own[n] for n in FFN_NAMES]
    for s in range(D):
        reqs = []
        if s + 1 < D:
            nxt = [comp.empty_like_shard(n) for n in FFN_NAMES]
            reqs = ex.ring(cur, nxt)
        w1, w2 = cur
        h_k = comp.ffn_up(w1, xn2)
        comp.accumulate(y, h_k, w2, "ffn")
        for q in reqs:
            q.wait()
        if s + 1 < D:
            cur = nxt
    return y


class GpuShardCompute:
    """The shard steps on this GPU, in the library's per-shard calls.  Shard
    tensors are the packed fp16 shards (K-major, as tsp_pack_shards lays
    them out); activations stay in the layer's formats (fp16 operands, fp32
    residual stream)."""

    def __init__(self, dims: tsp.Dims, D: int, rank: int, device="cuda"):
        self.dims, self.D, self.rank, self.dev = dims, D, rank, device
        self.L, self.h, self.T = dims.T // D, dims.h, dims.T
        self.hs, self.Fs = dims.h // D, dims.ffn // D
        self.ws = torch.zeros(tsp.lib().tsp_shard_workspace_bytes(), dtype=torch.uint8, device=device)
        self.shapes = {"wq": (self.hs, self.h), "wk": (self.hs, self.h), "wv": (self.hs, self.h),
                       "wo": (self.h, self.hs), "w1": (self.Fs, self.h), "w2": (self.h, self.Fs)}

    def _s(self):
        return torch.cuda.current_stream().cuda_stream

    def empty_like_shard(self, name):
        return torch.empty(self.shapes[name], dtype=torch.float16, device=self.dev)

    def layernorm(self, x):
        y = torch.empty(x.shape, dtype=torch.float16, device=self.dev)
        tsp._check(tsp.lib().tsp_layernorm(x.shape[0], x.shape[1], self.dims.ln_eps, x.data_ptr(),
                                           int(x.dtype == torch.float32), y.data_ptr(), self._s()), "tsp_layernorm")
        return y

    def residual(self, x):
        return x.float()

    def clone(self, y):
        return y.clone()

    def qkv(self, k, wq, wk, wv, xn1):
        q = torch.empty(self.L, self.hs, dtype=torch.float16, device=self.dev)
        kk = torch.empty(self.T, self.hs, dtype=torch.float16, device=self.dev)
        vv = torch.empty_like(kk)
        tsp._check(tsp.lib().tsp_shard_qkv(ctypes.byref(self.dims), self.D, self.rank, wq.data_ptr(), wk.data_ptr(),
                                           wv.data_ptr(), xn1.data_ptr(), q.data_ptr(), kk.data_ptr(), vv.data_ptr(),
                                           self.ws.data_ptr(), self._s()), "tsp_shard_qkv")
        return q, kk, vv

    def attention(self, k, q, kk, vv):
        a = torch.empty(self.L, self.hs, dtype=torch.float16, device=self.dev)
        tsp._check(tsp.lib().tsp_shard_attention(ctypes.byref(self.dims), self.D, self.rank, q.data_ptr(),
                                                 kk.data_ptr(), vv.data_ptr(), a.data_ptr(), self.ws.data_ptr(),
                                                 self._s()), "tsp_shard_attention")
        return a

    def ffn_up(self, w1, xn2):
        hk = torch.empty(self.L, self.Fs, dtype=torch.float16, device=self.dev)
        tsp._check(tsp.lib().tsp_shard_ffn_up(ctypes.byref(self.dims), self.D, w1.data_ptr(), xn2.data_ptr(),
                                              hk.data_ptr(), self.ws.data_ptr(), self._s()), "tsp_shard_ffn_up")
        return hk

    def accumulate(self, y, act, w, which):
        k_dim = self.hs if which == "attn" else self.Fs
        tsp._check(tsp.lib().tsp_shard_accumulate(ctypes.byref(self.dims), self.D, act.data_ptr(), k_dim,
                                                  w.data_ptr(), y.data_ptr(), self.ws.data_ptr(), self._s()),
                   "tsp_shard_accumulate")
