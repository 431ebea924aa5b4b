"""The per-shard CUDA steps that the cross-GPU exchange drives
(tsp_shard_qkv, tsp_shard_attention, tsp_shard_ffn_up, tsp_shard_accumulate,
tsp_layernorm), composed on one GPU for every rank in the exchange's order:
head group by head group (each group's K/V rows from every rank fill one
buffer - what the zigzag all-gather delivers), then the FFN blocks in ring
order (r + s) mod D.  Gates as for the layer: max-abs <= 2e-2 and rel-L2 <=
5e-3 against the plain fp64 layer and the fp16-storage oracle; and against
tsp_layer_forward, which sums the shards inside one product instead of in
the fp32 output, rel-L2 <= 1e-4."""
import numpy as np
import pytest
import torch

from folded_tensor_sequence_rank_b200 import build as tsp_build
from folded_tensor_sequence_rank_b200 import exchange, inputs, tsp
from oracle import tsp_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    tsp_build.build()
    tsp.lib()
    torch.cuda.init()


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


@pytest.mark.parametrize("T,h,H,F,D,seed", [
    (512, 256, 4, 1024, 2, 60),
    (960, 320, 5, 1280, 5, 61),     # D = 5, ragged chunks c = 96
    (2048, 512, 4, 2048, 4, 62),    # head_dim 128, one head per shard
    (8192, 4096, 32, 16384, 8, 63),
])
def test_shard_steps_compose_the_layer(T, h, H, F, D, seed):
    raw = inputs.layer_inputs(T, h, F, seed)
    dev = {k: v.cuda() for k, v in raw.items()}
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, dev)
    L, hs, Fs = T // D, h // D, F // D
    shard = lambda n, k: sw.shard(n, k, exchange.GpuShardCompute(dims, D, 0).shapes[n])
    idx = [tsp.zigzag_index(T, D, r).long() for r in range(D)]
    xs = [dev["x"].index_select(0, i).contiguous() for i in idx]
    comps = [exchange.GpuShardCompute(dims, D, r) for r in range(D)]
    xn1 = [comps[r].layernorm(xs[r]) for r in range(D)]
    y1 = [comps[r].residual(xs[r]) for r in range(D)]
    for k in range(D):
        qs, kk, vv = [], torch.empty(T, hs, dtype=torch.float16, device="cuda"), None
        vv = torch.empty_like(kk)
        for r in range(D):   # every rank's projection; its K/V rows land in the shared buffers
            q, kr, vr = comps[r].qkv(k, shard("wq", k), shard("wk", k), shard("wv", k), xn1[r])
            rows = idx[r]
            kk[rows] = kr[rows]
            vv[rows] = vr[rows]
            qs.append(q)
        for r in range(D):
            a = comps[r].attention(k, qs[r], kk, vv)
            comps[r].accumulate(y1[r], a, shard("wo", k), "attn")
    ys = []
    for r in range(D):
        xn2 = comps[r].layernorm(y1[r])
        y = y1[r].clone()
        for s in range(D):
            kb = (r + s) % D
            comps[r].accumulate(y, comps[r].ffn_up(shard("w1", kb), xn2), shard("w2", kb), "ffn")
        ys.append(y)
    for c in comps:
        assert tsp.get_device_status(c.ws) == tsp.TSP_OK
    torch.cuda.synchronize()
    x = raw["x"].double().numpy()
    w = {n: raw[n].double().numpy() for n in inputs.WEIGHT_NAMES}
    checked = [0, D - 1] if T > 2048 else list(range(D))
    for storage in (None, "fp16"):
        ws_ = O.stored_weights(w, storage)
        K, V = O.kv_project(x, ws_, storage=storage)
        for r in checked:
            pos = O.zigzag_index(T, D, r)
            rows = np.arange(L) if T <= 2048 else np.array(inputs.sample_rows(L, 32, seed + r, must=(0, L - 1)))
            ref = O.rank_rows_forward(x[pos[rows]], pos[rows], K, V, ws_, H, storage=storage)["y"]
            got = f64(ys[r])[rows]
            err = float(np.abs(got - ref).max())
            rl = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
            print(f"T={T} D={D} rank {r} vs oracle storage={storage}: max-abs {err:.3e} rel-L2 {rl:.3e}")
            assert err <= 2e-2 and rl <= 5e-3
    # the same rank through the whole-layer call
    ws = tsp.alloc_workspace(dims, D)
    Kf = torch.zeros(T, h, dtype=torch.float16, device="cuda")
    Vf = torch.zeros_like(Kf)
    for r in range(D):
        tsp.kv_project(dims, sw, r, xs[r], Kf, Vf, ws)
    yl = torch.empty(L, h, dtype=torch.float32, device="cuda")
    tsp.layer_forward(dims, sw, 0, xs[0], Kf, Vf, yl, ws)
    torch.cuda.synchronize()
    a, b = f64(ys[0]), f64(yl)
    assert np.linalg.norm(a - b) / np.linalg.norm(b) <= 1e-4
