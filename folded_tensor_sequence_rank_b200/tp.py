"""The tensor-parallel (TP) layer TSP is compared with, on one GPU.

The TSP news item (zubnet.ai, paragraphs 1-2) measures TSP against tensor
parallelism, where each of D ranks holds 1/D of the weights but every
token: its attention head group and FFN block produce partial products that
an all-reduce sums - twice per layer.  Here the D ranks run one after
another on one GPU and the all-reduce is a sum over their partials in
device memory (tsp_tp_all_reduce).  This module only orders calls into the
library: every step runs in its kernels.
"""
from __future__ import annotations

import torch

from . import tsp


def tp_layer_forward(dims: tsp.Dims, w: tsp.ShardedWeights, x: torch.Tensor, ws: torch.Tensor,
                     y_dtype=torch.bfloat16, parts: list | None = None, stream=None) -> torch.Tensor:
    """The layer over the whole sequence x [T, h] (bf16, natural order) as D
    tensor-parallel ranks compute it: every rank's attention partial, the
    all-reduce into Y1 (fp32), every rank's MLP partial, the all-reduce into
    Y.  `parts`: D fp32 [T, h] buffers (allocated when None)."""
    T, h, D = dims.T, dims.h, w.D
    if parts is None:
        parts = [torch.empty(T, h, dtype=torch.float32, device=x.device) for _ in range(D)]
    for k in range(D):
        tsp.tp_attention_partial(dims, w, k, x, parts[k], ws, stream=stream)
    y1 = torch.empty(T, h, dtype=torch.float32, device=x.device)
    tsp.tp_all_reduce(dims, parts, x, y1, stream=stream)
    for k in range(D):
        tsp.tp_mlp_partial(dims, w, k, y1, parts[k], ws, stream=stream)
    y = torch.empty(T, h, dtype=y_dtype, device=x.device)
    tsp.tp_all_reduce(dims, parts, y1, y, stream=stream)
    return y


def memory_account(dims: tsp.Dims, D: int) -> dict:
    """Bytes one GPU holds for one layer's forward when D TP ranks run on D
    GPUs: its weight shards (fp16), the whole sequence's input and output
    (bf16) and fp32 residual stream, one partial product [T, h] fp32 (what
    the all-reduce sums), and the workspace (LN output over all T tokens, its
    head group's Q, K, V, A, its FFN block's activations)."""
    T, h, F = dims.T, dims.h, dims.ffn
    acc = {
        "weights_own_shards": (4 * h * h + 2 * h * F) * 2 // D,
        "tokens_in_out": 2 * T * h * 2,
        "residual_fp32": T * h * 4,
        "partial_product": T * h * 4,
        "workspace": tsp.lib().tsp_tp_workspace_bytes(tsp.ctypes.byref(dims), D),
    }
    acc["total"] = sum(acc.values())
    return acc
