"""A stack of TSP layers on one GPU (every rank in turn) against the oracle
applied layer by layer: the fp16-storage oracle chained on its own hand-offs,
and each layer against the plain fp64 layer given the stack's hand-off.
Each layer's output is handed on in bf16, the layer's input format, on both
sides: the kernels' bf16 output is the fp32 output rounded to nearest even,
and the oracle's fp64 output is rounded the same way."""
import numpy as np
import pytest
import torch

from folded_tensor_sequence_rank_b200 import build as tsp_build
from folded_tensor_sequence_rank_b200 import inputs, stack, tsp
from oracle import tsp_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    tsp_build.build()
    tsp.lib()
    torch.cuda.init()


@pytest.mark.parametrize("T,h,H,F,D,n_layers", [
    (512, 256, 4, 1024, 2, 3),
    (1024, 512, 4, 2048, 4, 2),   # head_dim 128
])
def test_stack_matches_oracle_layer_by_layer(T, h, H, F, D, n_layers):
    raws = [inputs.layer_inputs(T, h, F, 40 + i) for i in range(n_layers)]
    x = raws[0]["x"]
    dims = tsp.make_dims(T, h, H, F)
    layers = [tsp.pack_shards(dims, D, {n: r[n].cuda() for n in inputs.WEIGHT_NAMES}) for r in raws]
    idx = [tsp.zigzag_index(T, D, r).long() for r in range(D)]
    xd = x.cuda()
    x_locals = [xd.index_select(0, i).contiguous() for i in idx]
    K = torch.zeros(T, h, dtype=torch.float16, device="cuda")
    V = torch.zeros_like(K)
    ws = tsp.alloc_workspace(dims, D)
    ys = stack.stack_forward(dims, layers, x_locals, K, V, ws, y_dtype=torch.float32)
    assert tsp.get_device_status(ws) == tsp.TSP_OK
    Y = torch.zeros(T, h, dtype=torch.float64)
    for r in range(D):
        Y[idx[r].cpu()] = ys[r].double().cpu()
    # the fp16-storage oracle chained layer by layer on its own bf16 hand-offs
    xr = x.double().numpy()
    for i, raw in enumerate(raws):
        w = {n: raw[n].double().numpy() for n in inputs.WEIGHT_NAMES}
        y = O.layer_forward(xr, w, H)["y"]
        xr = O.round_bf16(y) if i < n_layers - 1 else y
    got = Y.numpy()
    err = float(np.max(np.abs(got - xr)))
    rl = float(np.linalg.norm(got - xr) / np.linalg.norm(xr))
    print(f"stack of {n_layers}, T={T} D={D}: max-abs {err:.3e} rel-L2 {rl:.3e}")
    assert err <= 2e-2 and rl <= 5e-3
    # every layer of the stack against the plain fp64 layer (storage=None), fed
    # the stack's own bf16 hand-off: a chained plain oracle would let single
    # bf16 rounding flips (0.031 at |y| >= 4) compound from layer to layer
    prev = x.double().numpy()
    for i, raw in enumerate(raws):
        ys_i = stack.stack_forward(dims, layers[: i + 1], x_locals, K, V, ws, y_dtype=torch.float32)
        Yi = torch.zeros(T, h, dtype=torch.float32)
        for r in range(D):
            Yi[idx[r].cpu()] = ys_i[r].cpu()
        w = {n: raw[n].double().numpy() for n in inputs.WEIGHT_NAMES}
        plain = O.layer_forward(prev, w, H, storage=None)["y"]
        got_i = Yi.double().numpy()
        err = float(np.max(np.abs(got_i - plain)))
        rl = float(np.linalg.norm(got_i - plain) / np.linalg.norm(plain))
        print(f"  layer {i} vs plain layer: max-abs {err:.3e} rel-L2 {rl:.3e}")
        assert err <= 2e-2 and rl <= 5e-3, i
        prev = Yi.to(torch.bfloat16).double().numpy()  # the bf16 hand-off the stack passes on
