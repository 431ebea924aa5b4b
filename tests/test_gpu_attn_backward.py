"""Parity of tsp_attn_backward (the backward of one rank's causal attention
against the all-gathered K/V) with the oracle, through the C ABI.

Inputs come from the CUDA forward itself: tsp_layer_forward leaves the
rank's Q, its attention output A and the log-sum-exp stash in the
workspace, K and V come from tsp_kv_project, and the gradient dA is a seeded
draw in fp16.  The oracle takes those same fp16 values.

Gates, per output (dQ, and dK, dV summed over every rank that ran):
* against the oracle's stored-value form (attention_backward_stored: dO, P
  and dS rounded to fp16 where the kernel stores them), rel-L2 <= 1e-3 and
  max-abs <= 1e-2 * max |ref|: what remains is fp32 accumulation order, the
  ex2 / polynomial exponentials (relative 2.7e-6) and rare one-unit flips of
  a stored fp16 value;
* against the plain fp64 backward (causal_attention_backward, no rounding),
  rel-L2 <= 1e-2 and max-abs <= 3e-2 * max |ref|: fp16 storage of P, dS and
  dO (relative 2^-11 at most each) bounds the distance at a few 1e-3;
* the log-sum-exp stash against the oracle's, |diff| <= 1e-4 (natural-log
  units).
"""
import math

import numpy as np
import pytest
import torch

from folded_tensor_sequence_rank_b200 import build as tsp_build
from folded_tensor_sequence_rank_b200 import inputs, tsp
from oracle import tsp_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    tsp_build.build()
    tsp.lib()
    torch.cuda.init()


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def close(name, got, ref, rel, mx):
    assert np.isfinite(got).all(), name
    err = float(np.abs(got - ref).max())
    scale = float(np.abs(ref).max())
    rl = rel_l2(got, ref)
    print(f"{name}: max-abs {err:.3e} (scale {scale:.3e}) rel-L2 {rl:.3e}")
    assert rl <= rel and err <= mx * scale, f"{name}: max-abs {err:.3e} (scale {scale:.3e}) rel-L2 {rl:.3e}"


def forward_then_backward(T, h, H, F, D, seed, ranks):
    """Every rank projects its K/V; then, for each rank in `ranks`, its layer
    forward and its attention backward (dK, dV added up over those ranks)."""
    raw = {k: v.cuda() for k, v in inputs.layer_inputs(T, h, F, seed).items()}
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, raw)
    ws = tsp.alloc_workspace(dims, D)
    aws = tsp.alloc_attn_backward_workspace(dims, D)
    K = torch.zeros(T, h, dtype=torch.float16, device="cuda")
    V = torch.zeros_like(K)
    L = T // D
    xs = [raw["x"].index_select(0, tsp.zigzag_index(T, D, r).long()).contiguous() for r in range(D)]
    for r in range(D):
        tsp.kv_project(dims, sw, r, xs[r], K, V, ws)
    dK = torch.zeros(T, h, dtype=torch.float32, device="cuda")
    dV = torch.zeros_like(dK)
    per_rank = {}
    for r in ranks:
        y = torch.empty(L, h, dtype=torch.float32, device="cuda")
        tsp.layer_forward(dims, sw, r, xs[r], K, V, y, ws)
        q = tsp.workspace_view(ws, dims, D, "q").clone()
        a = tsp.workspace_view(ws, dims, D, "a").clone()
        lse = tsp.workspace_view(ws, dims, D, "lse").clone()
        d_o = inputs.attention_grad_inputs(L, h, seed * 100 + r).cuda()
        dq = torch.full((L, h), float("nan"), device="cuda")
        tsp.attn_backward(dims, D, r, q, K, V, a, lse, d_o, dq, dK, dV, aws)
        assert tsp.get_device_status(aws) == tsp.TSP_OK
        assert tsp.get_device_status(ws) == tsp.TSP_OK
        per_rank[r] = dict(q=f64(q), a=f64(a), lse=f64(tsp.lse_rows(lse, dims, D)), d_o=f64(d_o), dq=f64(dq))
    torch.cuda.synchronize()
    return dims, f64(K), f64(V), f64(dK), f64(dV), per_rank


SHAPES = [
    (512, 256, 4, 1024, 2, 0),      # the tiny layer, head_dim 64
    (2048, 512, 4, 2048, 2, 1),     # head_dim 128, several tiles per chunk
    (800, 256, 4, 1024, 2, 2),      # ragged chunks: c = 200
    (288, 256, 2, 512, 2, 3),       # head_dim 128, c = 72 (< one tile)
    (768, 384, 6, 1536, 3, 4),      # D = 3
    (960, 320, 5, 1280, 5, 5),      # D = 5, ragged c = 96
    (8, 256, 4, 1024, 4, 6),        # degenerate chunks: c = 1
    (1536, 384, 3, 1536, 3, 7),     # head_dim 128, one head per shard
]


@pytest.mark.parametrize("T,h,H,F,D,seed", SHAPES)
def test_attention_backward_all_ranks(T, h, H, F, D, seed):
    dims, K, V, dK, dV, per = forward_then_backward(T, h, H, F, D, seed, list(range(D)))
    s = dims.softmax_scale
    dk_ref, dv_ref = np.zeros_like(K), np.zeros_like(V)
    dk_pl, dv_pl = np.zeros_like(K), np.zeros_like(V)
    for r, g in per.items():
        pos = O.zigzag_index(T, D, r)
        lse_ref = O.attention_logsumexp(g["q"], K, pos, H, s)
        err = float(np.abs(g["lse"] * math.log(2.0) - lse_ref).max())
        assert err <= 1e-4, f"rank {r} lse: {err:.3e}"
        dq, dk, dv = O.attention_backward_stored(g["q"], K, V, g["a"], pos, g["d_o"], H, s)
        close(f"rank {r} dq", g["dq"], dq, 1e-3, 1e-2)
        dk_ref += dk
        dv_ref += dv
        dq0, dk0, dv0 = O.causal_attention_backward(g["q"], K, V, pos, g["d_o"], H, s)
        close(f"rank {r} dq vs plain", g["dq"], dq0, 1e-2, 3e-2)
        dk_pl += dk0
        dv_pl += dv0
    close("dk (sum over ranks)", dK, dk_ref, 1e-3, 1e-2)
    close("dv (sum over ranks)", dV, dv_ref, 1e-3, 1e-2)
    close("dk vs plain", dK, dk_pl, 1e-2, 3e-2)
    close("dv vs plain", dV, dv_pl, 1e-2, 3e-2)
    # dK, dV summed over ranks are the whole sequence's: the oracle's
    # unsharded backward over every position
    x_all = np.arange(T)
    q_all = np.zeros((T, dims.h))
    do_all = np.zeros((T, dims.h))
    for r, g in per.items():
        pos = O.zigzag_index(T, D, r)
        q_all[pos] = g["q"]
        do_all[pos] = g["d_o"]
    _, dk_full, dv_full = O.causal_attention_backward(q_all, K, V, x_all, do_all, H, s)
    close("dk vs the unsharded sequence", dK, dk_full, 1e-2, 3e-2)
    close("dv vs the unsharded sequence", dV, dv_full, 1e-2, 3e-2)


def test_attention_backward_7b_T8192_rank0_in_full():
    T, h, H, F, D = 8192, 4096, 32, 16384, 8
    dims, K, V, dK, dV, per = forward_then_backward(T, h, H, F, D, 11, [0])
    g = per[0]
    s = dims.softmax_scale
    pos = O.zigzag_index(T, D, 0)
    lse_ref = O.attention_logsumexp(g["q"], K, pos, H, s)
    assert float(np.abs(g["lse"] * math.log(2.0) - lse_ref).max()) <= 1e-4
    dq, dk, dv = O.attention_backward_stored(g["q"], K, V, g["a"], pos, g["d_o"], H, s)
    close("dq", g["dq"], dq, 1e-3, 1e-2)
    close("dk", dK, dk, 1e-3, 1e-2)
    close("dv", dV, dv, 1e-3, 1e-2)
    dq0, dk0, dv0 = O.causal_attention_backward(g["q"], K, V, pos, g["d_o"], H, s)
    close("dq vs plain", g["dq"], dq0, 1e-2, 3e-2)
    close("dk vs plain", dK, dk0, 1e-2, 3e-2)
    close("dv vs plain", dV, dv0, 1e-2, 3e-2)


def test_attention_backward_128k_sampled():
    """The full 128K rank (D = 8, rank 0; stand-in K/V as in the forward's
    sampled tests): dQ on sampled rows of both chunks, each computed alone by
    the oracle; dK and dV through properties of the whole sums - rows of P sum
    to 1, so the key-summed dV equals the query-summed dO, and softmax ignores
    a common shift of a row's scores, so the key-summed dK of a head is ~0
    (here exactly zero up to rounding: Delta comes from the stored output)."""
    T, h, H, F, D, seed = 131072, 4096, 32, 16384, 8, 12
    L = T // D
    c = L // 2
    raw = inputs.rank_inputs(L, T, h, F, seed)
    dev = {k: v.cuda() for k, v in raw.items()}
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, dev)
    ws = tsp.alloc_workspace(dims, D)
    aws = tsp.alloc_attn_backward_workspace(dims, D)
    y = torch.empty(L, h, dtype=torch.float32, device="cuda")
    tsp.layer_forward(dims, sw, 0, dev["x_local"], dev["k_full"], dev["v_full"], y, ws)
    q = tsp.workspace_view(ws, dims, D, "q")
    a = tsp.workspace_view(ws, dims, D, "a")
    lse = tsp.workspace_view(ws, dims, D, "lse")
    d_o = inputs.attention_grad_inputs(L, h, seed).cuda()
    dq = torch.empty(L, h, dtype=torch.float32, device="cuda")
    dK = torch.zeros(T, h, dtype=torch.float32, device="cuda")
    dV = torch.zeros_like(dK)
    tsp.attn_backward(dims, D, 0, q, dev["k_full"], dev["v_full"], a, lse, d_o, dq, dK, dV, aws)
    assert tsp.get_device_status(aws) == tsp.TSP_OK
    s = dims.softmax_scale
    rows = inputs.sample_rows(L, 14, seed, must=(0, c - 1, c, L - 1))
    pos = O.zigzag_index(T, D, 0)[rows]
    Kf, Vf = raw["k_full"].double().numpy(), raw["v_full"].double().numpy()
    qs, as_, dos = f64(q[rows]), f64(a[rows]), f64(d_o[rows])
    lse_ref = O.attention_logsumexp(qs, Kf, pos, H, s)
    assert float(np.abs(f64(tsp.lse_rows(lse, dims, D)[rows]) * math.log(2.0) - lse_ref).max()) <= 1e-4
    dq_ref, _, _ = O.attention_backward_stored(qs, Kf, Vf, as_, pos, dos, H, s)
    close("dq rows", f64(dq[rows]), dq_ref, 1e-3, 1e-2)
    dq0, _, _ = O.causal_attention_backward(qs, Kf, Vf, pos, dos, H, s)
    close("dq rows vs plain", f64(dq[rows]), dq0, 1e-2, 3e-2)
    # key sums: sum_k dV[k] = sum_q dO[q] (fp16 P: each row sums to 1 within
    # 2^-11 per entry); sum_k dK[k] per head = sum_q (stuff that cancels)
    dv_sum = dV.double().sum(0).cpu().numpy()
    do_sum = d_o.double().sum(0).cpu().numpy()
    close("sum of dV over keys vs sum of dO over queries", dv_sum, do_sum, 2e-3, 1e-2)
    dk_sum = dK.double().sum(0).cpu().numpy()
    dk_rms = float(dK.double().pow(2).mean().sqrt())
    assert np.abs(dk_sum).max() <= 1e-2 * dk_rms * math.sqrt(T), (np.abs(dk_sum).max(), dk_rms)
    # keys past the rank's last position get nothing
    assert not dK[(2 * D) * c:].any() and not dV[(2 * D) * c:].any()


def test_attention_backward_32k_d16_sampled():
    """Rank 5 of 16 at T = 32768 (c = 1024; head groups of two heads): dQ on
    sampled rows of both chunks, computed alone by the oracle."""
    T, h, H, F, D, r, seed = 32768, 4096, 32, 16384, 16, 5, 13
    L = T // D
    c = L // 2
    raw = inputs.rank_inputs(L, T, h, F, seed)
    dev = {k: v.cuda() for k, v in raw.items()}
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, dev)
    ws = tsp.alloc_workspace(dims, D)
    aws = tsp.alloc_attn_backward_workspace(dims, D)
    y = torch.empty(L, h, dtype=torch.float32, device="cuda")
    tsp.layer_forward(dims, sw, r, dev["x_local"], dev["k_full"], dev["v_full"], y, ws)
    q = tsp.workspace_view(ws, dims, D, "q")
    a = tsp.workspace_view(ws, dims, D, "a")
    d_o = inputs.attention_grad_inputs(L, h, seed).cuda()
    dq = torch.empty(L, h, dtype=torch.float32, device="cuda")
    dK = torch.zeros(T, h, dtype=torch.float32, device="cuda")
    dV = torch.zeros_like(dK)
    tsp.attn_backward(dims, D, r, q, dev["k_full"], dev["v_full"], a, tsp.workspace_view(ws, dims, D, "lse"), d_o, dq,
                      dK, dV, aws)
    assert tsp.get_device_status(aws) == tsp.TSP_OK
    s = dims.softmax_scale
    rows = inputs.sample_rows(L, 12, seed, must=(0, c - 1, c, L - 1))
    pos = O.zigzag_index(T, D, r)[rows]
    Kf, Vf = raw["k_full"].double().numpy(), raw["v_full"].double().numpy()
    qs, as_, dos = f64(q[rows]), f64(a[rows]), f64(d_o[rows])
    dq_ref, _, _ = O.attention_backward_stored(qs, Kf, Vf, as_, pos, dos, H, s)
    close("dq rows", f64(dq[rows]), dq_ref, 1e-3, 1e-2)
    dq0, _, _ = O.causal_attention_backward(qs, Kf, Vf, pos, dos, H, s)
    close("dq rows vs plain", f64(dq[rows]), dq0, 1e-2, 3e-2)
    # keys past the rank's last position get nothing
    last = (2 * D - r) * c
    assert not dK[last:].any() and not dV[last:].any()


def test_zero_gradient_gives_zeros():
    """dA = 0: dQ, dK and dV are exactly zero."""
    T, h, H, F, D = 512, 256, 4, 1024, 2
    raw = {k: v.cuda() for k, v in inputs.layer_inputs(T, h, F, 9).items()}
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, raw)
    ws = tsp.alloc_workspace(dims, D)
    aws = tsp.alloc_attn_backward_workspace(dims, D)
    K = torch.zeros(T, h, dtype=torch.float16, device="cuda")
    V = torch.zeros_like(K)
    xs = [raw["x"].index_select(0, tsp.zigzag_index(T, D, r).long()).contiguous() for r in range(D)]
    for r in range(D):
        tsp.kv_project(dims, sw, r, xs[r], K, V, ws)
    y = torch.empty(T // D, h, device="cuda")
    tsp.layer_forward(dims, sw, 1, xs[1], K, V, y, ws)
    dq = torch.full((T // D, h), 7.0, device="cuda")
    dK = torch.zeros(T, h, device="cuda")
    dV = torch.zeros(T, h, device="cuda")
    zero = torch.zeros(T // D, h, dtype=torch.float16, device="cuda")
    tsp.attn_backward(dims, D, 1, tsp.workspace_view(ws, dims, D, "q"), K, V, tsp.workspace_view(ws, dims, D, "a"),
                      tsp.workspace_view(ws, dims, D, "lse"), zero, dq, dK, dV, aws)
    torch.cuda.synchronize()
    assert not dq.any() and not dK.any() and not dV.any()
