"""Forward of a stack of TSP layers, and its memory account.

On one GPU every rank runs in turn, as the single-GPU form of the method does
(TSP news item, zubnet.ai, paragraph 2).  For each layer:
- each rank's `tsp_kv_project` writes its own tokens' K/V rows to their global
  positions, which together form what the all-gather gives every rank;
- then each rank's `tsp_layer_forward` produces its tokens' output.
A rank keeps its tokens in rank-local zigzag order from layer to layer, so its
output is directly its next layer's input.  This module only orders calls into
the library: every step runs in its kernels.
"""
from __future__ import annotations

import torch

from . import tsp


def stack_forward(dims: tsp.Dims, layers: list, x_locals: list, k_full: torch.Tensor, v_full: torch.Tensor,
                  ws: torch.Tensor, y_dtype=torch.bfloat16, stream=None) -> list:
    """Runs every layer of `layers` (ShardedWeights, one per layer, all with the
    same D) over all D ranks.  `x_locals[r]` is rank r's input [T/D, h] bf16 in
    rank-local order; K/V [T, h] fp16 and the workspace are reused by every
    layer.  Returns the last layer's outputs per rank (y_dtype; bf16 between
    layers, as the layer's input is bf16)."""
    if not layers:
        return list(x_locals)
    D = layers[0].D
    if len(x_locals) != D or any(w.D != D for w in layers):
        raise ValueError("one input per rank and the same D for every layer")
    L, h = dims.T // D, dims.h
    dev = x_locals[0].device
    bufs = [[torch.empty(L, h, dtype=torch.bfloat16, device=dev) for _ in range(D)] for _ in range(2)]
    xs = list(x_locals)
    for li, w in enumerate(layers):
        last = li == len(layers) - 1
        for r in range(D):
            tsp.kv_project(dims, w, r, xs[r], k_full, v_full, ws, stream=stream)
        ys = ([torch.empty(L, h, dtype=y_dtype, device=dev) for _ in range(D)] if last and y_dtype != torch.bfloat16
              else bufs[li % 2])
        for r in range(D):
            tsp.layer_forward(dims, w, r, xs[r], k_full, v_full, ys[r], ws, stream=stream)
        xs = ys
    return xs


def memory_account(dims: tsp.Dims, D: int, n_layers: int) -> dict:
    """Bytes one GPU holds for a forward pass of `n_layers` layers when the D
    ranks run on D GPUs (one rank each):
    - its 1/D of every layer's weights (fp16 shards);
    - a receive buffer for one layer's other D-1 weight shards, which the
      broadcast and ring stream through;
    - its own tokens' input and output [T/D, h] bf16;
    - the current layer's all-gathered K/V [T, h] fp16;
    - the layer workspace (LN outputs, Q, attention output, fp32 residual,
      FFN activations) from tsp_workspace_bytes.
    Nothing is kept for a backward pass."""
    T, h, F = dims.T, dims.h, dims.ffn
    L = T // D
    layer_w = (4 * h * h + 2 * h * F) * 2
    acc = {
        "weights_own_shards": n_layers * layer_w // D,
        "weights_receive_buffer": layer_w * (D - 1) // D,
        "tokens_in_out": 2 * L * h * 2,
        "kv_all_gathered": 2 * T * h * 2,
        "workspace": tsp.workspace_bytes(dims, D),
    }
    acc["total"] = sum(acc.values())
    return acc
