"""Parity of the whole layer's backward - tsp_layer_backward on every rank,
the dK/dV sum over ranks (the reduce-scatter, here the kernels' additions
into one buffer), then tsp_kv_backward on every key owner - with the oracle,
through the C ABI.

The oracle is rank_layer_backward + kv_backward_rows in two forms: with the
kernels' precision model (fp16 forward storage and dA, bf16 gradient
operands) and plain fp64 (no rounding).  Gates per output (dX per rank, the
six weight gradients per rank, dK/dV summed over ranks):
* stored model: rel-L2 <= 2e-3, max-abs <= 2e-2 * max |ref|.  The model
  rounds where the kernels do, so what remains is fp32 accumulation order
  and one-unit flips of stored 16-bit values where fp32 and fp64 round
  differently - now at some twenty rounding points chained through dY1, dA,
  dQ and the K/V gradients, each flip 2^-9 relative in bf16;
* plain fp64: rel-L2 <= 1e-2, max-abs <= 5e-2 * max |ref|: bf16 gradient
  operands (relative 2^-9, rms 1.1e-3 each, two per weight-gradient
  product) and fp16 storage of the forward values (the oracle's two forms
  sit 1.5e-3 to 4e-3 apart on these shapes).
The sums over ranks of every gradient are also compared with the plain
oracle's sums, which its CPU pins tie to torch autograd of the unsharded
layer.
"""
import numpy as np
import pytest
import torch

from folded_tensor_sequence_rank_b200 import build as tsp_build
from folded_tensor_sequence_rank_b200 import inputs, tsp
from oracle import tsp_oracle as O

pytestmark = pytest.mark.gpu

NAMES = ("wq", "wk", "wv", "wo", "w1", "w2")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    tsp_build.build()
    tsp.lib()
    torch.cuda.init()


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def close(name, got, ref, rel, mx):
    assert np.isfinite(got).all(), name
    err = float(np.abs(got - ref).max())
    scale = float(np.abs(ref).max())
    rl = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    print(f"{name}: max-abs {err:.3e} (scale {scale:.3e}) rel-L2 {rl:.3e}")
    assert rl <= rel and err <= mx * scale, f"{name}: max-abs {err:.3e} (scale {scale:.3e}) rel-L2 {rl:.3e}"


def run_layer_backward(T, h, H, F, D, seed):
    raw = inputs.layer_inputs(T, h, F, seed)
    dev = {k: v.cuda() for k, v in raw.items()}
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, dev)
    L = T // D
    idx = [tsp.zigzag_index(T, D, r).long() for r in range(D)]
    xs = [dev["x"].index_select(0, i).contiguous() for i in idx]
    wss = [tsp.alloc_workspace(dims, D) for _ in range(D)]
    K = torch.zeros(T, h, dtype=torch.float16, device="cuda")
    V = torch.zeros_like(K)
    for r in range(D):
        tsp.kv_project(dims, sw, r, xs[r], K, V, wss[r])
    y = torch.empty(L, h, dtype=torch.float32, device="cuda")
    for r in range(D):   # each rank's forward leaves Q, A, Y1 and the stash in its workspace
        tsp.layer_forward(dims, sw, r, xs[r], K, V, y, wss[r])
    gen = torch.Generator().manual_seed(seed + 1000)
    dy_all = (torch.randn(T, h, generator=gen)).to(torch.bfloat16)
    dys = [dy_all.cuda().index_select(0, i).contiguous() for i in idx]
    bws = tsp.alloc_layer_backward_workspace(dims, D)
    kws = tsp.alloc_kv_backward_workspace(dims, D)
    dK = torch.zeros(T, h, dtype=torch.float32, device="cuda")
    dV = torch.zeros_like(dK)
    out = []
    for r in range(D):
        g = {n: torch.full(raw[n].shape, float("nan"), device="cuda") for n in NAMES}
        dx = torch.full((L, h), float("nan"), device="cuda")
        tsp.layer_backward(dims, sw, dev, r, xs[r], wss[r], K, V, dys[r], dx, g, dK, dV, bws)
        assert tsp.get_device_status(bws) == tsp.TSP_OK
        out.append(dict(dx=dx, g=g))
    dK_sum, dV_sum = f64(dK), f64(dV)
    for r in range(D):   # every key owner, after the sum over ranks
        tsp.kv_backward(dims, D, dev, r, xs[r], dK, dV, out[r]["dx"], out[r]["g"]["wk"], out[r]["g"]["wv"], kws)
        assert tsp.get_device_status(kws) == tsp.TSP_OK
    torch.cuda.synchronize()
    for r in range(D):
        out[r] = {"dx": f64(out[r]["dx"]), **{n: f64(t) for n, t in out[r]["g"].items()}}
    return raw, f64(dy_all), dK_sum, dV_sum, out


@pytest.mark.parametrize("T,h,H,F,D,seed", [
    (512, 256, 4, 1024, 2, 40),     # the tiny layer
    (768, 256, 4, 1024, 2, 41),     # c = 192: one and a half query tiles per chunk
    (1024, 256, 4, 1024, 4, 42),    # D = 4
    (1024, 512, 4, 2048, 2, 43),    # head_dim 128
])
def test_layer_backward_all_ranks(T, h, H, F, D, seed):
    raw, dy, dK, dV, got = run_layer_backward(T, h, H, F, D, seed)
    x = raw["x"].double().numpy()
    w = {n: raw[n].double().numpy() for n in NAMES}
    forms = {"stored": dict(storage="fp16", grad_storage="bf16"), "plain": {}}
    gates = {"stored": (2e-3, 2e-2), "plain": (1e-2, 5e-2)}
    for form, prec in forms.items():
        rel, mx = gates[form]
        per, dk, dv = [], np.zeros_like(dK), np.zeros_like(dV)
        for r in range(D):
            idx = O.zigzag_index(T, D, r)
            g = O.rank_layer_backward(r, D, x, w, dy[idx], H, **prec)
            per.append(g)
            dk += g["dk_full"]
            dv += g["dv_full"]
        close(f"{form}: dK summed over ranks", dK, dk, rel, mx)
        close(f"{form}: dV summed over ranks", dV, dv, rel, mx)
        sums = {n: np.zeros_like(w[n]) for n in NAMES}
        gsum = {n: np.zeros_like(w[n]) for n in NAMES}
        for r in range(D):
            idx = O.zigzag_index(T, D, r)
            kv = O.kv_backward_rows(x[idx], dk[idx], dv[idx], w, **prec)
            ref = {"dx": per[r]["dx_partial"] + kv["dx"], "wq": per[r]["dwq"], "wo": per[r]["dwo"],
                   "w1": per[r]["dw1"], "w2": per[r]["dw2"], "wk": kv["dwk"], "wv": kv["dwv"]}
            for n, v in ref.items():
                close(f"{form}: rank {r} d{n}", got[r][n], v, rel, mx)
            for n in NAMES:
                sums[n] += ref[n]
                gsum[n] += got[r][n]
        for n in NAMES:   # the layer's weight gradients: every rank's share summed
            close(f"{form}: d{n} summed over ranks", gsum[n], sums[n], rel, mx)
