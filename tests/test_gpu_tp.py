"""The tensor-parallel baseline layer (D ranks in turn, the all-reduce as a
sum of their partials on one GPU) against the oracle: it computes the same
layer as TSP, so the same gates apply - max-abs <= 2e-2 and rel-L2 <= 5e-3
on the fp32 output, against the plain fp64 layer and the fp16-storage
oracle (both round where the kernels store fp16 in the same places)."""
import numpy as np
import pytest
import torch

from folded_tensor_sequence_rank_b200 import build as tsp_build
from folded_tensor_sequence_rank_b200 import inputs, tp, tsp
from oracle import tsp_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    tsp_build.build()
    tsp.lib()
    torch.cuda.init()


@pytest.mark.parametrize("T,h,H,F,D,seed", [
    (512, 256, 4, 1024, 2, 50),     # the tiny layer
    (1024, 256, 4, 1024, 4, 51),    # D = 4: one head of 64 per rank
    (800, 256, 4, 1024, 2, 52),     # T/2 = 400: ragged query tiles
    (2048, 512, 4, 2048, 2, 53),    # head_dim 128
    (8192, 4096, 32, 16384, 8, 54),  # the 7B layer at T = 8192, D = 8
])
def test_tp_layer_matches_oracle(T, h, H, F, D, seed):
    raw = inputs.layer_inputs(T, h, F, seed)
    dev = {k: v.cuda() for k, v in raw.items()}
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, dev)
    ws = tsp.alloc_tp_workspace(dims, D)
    y = tp.tp_layer_forward(dims, sw, dev["x"], ws, y_dtype=torch.float32)
    assert tsp.get_device_status(ws) == tsp.TSP_OK
    got = y.double().cpu().numpy()
    x = raw["x"].double().numpy()
    w = {n: raw[n].double().numpy() for n in inputs.WEIGHT_NAMES}
    rows = np.arange(T) if T <= 2048 else np.array(inputs.sample_rows(T, 48, seed, must=(0, T // 2, T - 1)))
    for storage in (None, "fp16"):
        ws_ = O.stored_weights(w, storage)
        if T <= 2048:
            ref = O.layer_forward(x, ws_, H, storage=storage)["y"]
        else:   # sampled rows, given the oracle's K/V of the whole sequence
            K, V = O.kv_project(x, ws_, storage=storage)
            ref = O.rank_rows_forward(x[rows], rows, K, V, ws_, H, storage=storage)["y"]
        g = got[rows]
        err = float(np.abs(g - ref).max())
        rl = float(np.linalg.norm(g - ref) / np.linalg.norm(ref))
        print(f"TP T={T} D={D} vs oracle storage={storage}: max-abs {err:.3e} rel-L2 {rl:.3e}")
        assert err <= 2e-2 and rl <= 5e-3, storage


def test_tp_bf16_output_is_rounded_fp32_output():
    T, h, H, F, D = 512, 256, 4, 1024, 2
    dev = {k: v.cuda() for k, v in inputs.layer_inputs(T, h, F, 55).items()}
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, dev)
    ws = tsp.alloc_tp_workspace(dims, D)
    y32 = tp.tp_layer_forward(dims, sw, dev["x"], ws, y_dtype=torch.float32)
    y16 = tp.tp_layer_forward(dims, sw, dev["x"], ws, y_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))
