"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Gates (the layer's stated tolerance for bf16 layer outputs): max-abs <= 2e-2
and relative-L2 <= 5e-3 on the layer output, computed in fp32 by the kernels
(y_dtype fp32); the bf16 output equals the fp32 output rounded to nearest
even bit for bit.  Every end-to-end test applies that gate twice: against
the plain fp64 layer (the oracle with storage=None: no rounding anywhere but
the bf16 inputs), and against the oracle that rounds the matmul operands to
fp16 where the kernels store them (storage="fp16"), whose distance to the
kernels is ~100x smaller and so catches smaller mistakes.  The zigzag index
map and the weight shard packing are integer / byte work and must match
exactly.  Intermediates get looser diagnostic gates that catch errors the
residual stream would hide.

Sizes: the tiny layer (h=256, 4 heads of 64, FFN 1024, T=512, D=2) and
variants (D=1, D=4, ragged chunks) are compared in full; the 7B layer at
T=8192 (D=8) in full for a rank; at T=131072 (D=8) and T=32768 (D=1..16) on
sampled rows the oracle computes one by one, in the launch configuration the
benchmark uses.
"""
import math

import numpy as np
import pytest
import torch

from folded_tensor_sequence_rank_b200 import build as tsp_build
from folded_tensor_sequence_rank_b200 import inputs
from folded_tensor_sequence_rank_b200 import tsp
from oracle import tsp_oracle as O

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 2e-2, 5e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    tsp_build.build()
    tsp.lib()
    torch.cuda.init()


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def assert_layer_close(y_gpu, y_ref, what, x=None):
    err = float(np.max(np.abs(y_gpu - y_ref)))
    rl = rel_l2(y_gpu, y_ref)
    print(f"{what}: max-abs {err:.3e} rel-L2 {rl:.3e}")
    assert np.isfinite(y_gpu).all(), what
    assert err <= MAX_ABS and rl <= REL_L2, f"{what}: max-abs {err:.3e}, rel-L2 {rl:.3e}"
    if x is not None:  # the layer's own contribution, without the residual
        rd = rel_l2(y_gpu - x, y_ref - x)
        assert rd <= 2e-2, f"{what}: rel-L2 of (Y - X) {rd:.3e}"


def assert_operand_close(g, e, what):
    """A stored fp16 operand (K, V): equal up to rounding flips.

    The kernels compute the LayerNorm output in fp32 and the oracle in fp64;
    about one entry in 2^13 lies so close to an fp16 rounding tie that the two
    round it differently, i.e. a few entries of every h = 4096 row.  One such
    flip moves every K entry of the row by ulp(xn) * |w| (2^-9 * 0.08 = 1.6e-4
    at most for |xn| < 4, |w| < 4 sigma): an ABSOLUTE error, independent of the
    K entry it lands on, so near zero it is many units of that entry.  Hence
    the floors, in units of the tensor's rms (1.28 for the 7B layer): 2^-12 *
    rms = 3.1e-4 covers one flip, 2^-10 * rms covers several in one dot
    product.  Bound: every entry within four units of itself plus 2^-10 rms;
    at most 1e-4 of the entries more than one unit plus 2^-12 rms away; and
    rel-L2 <= 1e-3."""
    scale = float(np.sqrt(np.mean(e * e)))
    diff = np.abs(g - e)
    ulp = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(e), 2.0 ** -14))) - 10), 2.0 ** -24)
    assert np.all(diff <= 4 * ulp + 2.0 ** -10 * scale), f"{what}: max {diff.max():.3e} (rms {scale:.3e})"
    frac = float(np.mean(diff > ulp * 1.0000001 + 2.0 ** -12 * scale))
    assert frac <= 1e-4, f"{what}: {frac:.2e} of entries more than one unit (plus floor) off"
    assert rel_l2(g, e) <= 1e-3, f"{what}: rel-L2 {rel_l2(g, e):.3e}"


def to_cuda(d):
    return {k: v.cuda() for k, v in d.items()}


def weights_f64(raw):
    return {n: f64(raw[n]) for n in inputs.WEIGHT_NAMES}


# --------------------------------------------------------------------------
def test_zigzag_bit_exact():
    for T, D in [(512, 2), (8192, 8), (131072, 8), (32768, 16), (100, 2), (8, 1), (768, 3)]:
        for r in sorted({0, D // 2, D - 1}):
            got = tsp.zigzag_index(T, D, r).cpu().numpy()
            assert np.array_equal(got.astype(np.int64), O.zigzag_index(T, D, r)), (T, D, r)


def test_pack_shards_exact():
    T, h, H, F, D = 512, 256, 4, 1024, 4
    raw = to_cuda(inputs.layer_inputs(T, h, F, 3))
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, raw)
    torch.cuda.synchronize()
    hs, Fs = h // D, F // D
    for k in range(D):
        cols, fcols = slice(k * hs, (k + 1) * hs), slice(k * Fs, (k + 1) * Fs)
        expect = {"wq": raw["wq"][:, cols].t(), "wk": raw["wk"][:, cols].t(), "wv": raw["wv"][:, cols].t(),
                  "wo": raw["wo"][cols, :].t(), "w1": raw["w1"][:, fcols].t(), "w2": raw["w2"][fcols, :].t()}
        for n, e in expect.items():
            got = sw.shard(n, k, tuple(e.shape))
            assert torch.equal(got.view(torch.int16), e.to(torch.float16).contiguous().view(torch.int16)), (n, k)


# --------------------------------------------------------------------------
def run_full_sequence(T, h, H, F, D, seed, y_dtype=torch.float32):
    """All D ranks on one GPU: every rank projects its K/V, then every rank runs
    its layer forward.  Returns the outputs scattered to natural order."""
    raw = inputs.layer_inputs(T, h, F, seed)
    dev = to_cuda(raw)
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, dev)
    ws = tsp.alloc_workspace(dims, D)
    K = torch.zeros(T, h, dtype=torch.float16, device="cuda")
    V = torch.zeros_like(K)
    idx = [tsp.zigzag_index(T, D, r).long() for r in range(D)]
    x_loc = [dev["x"].index_select(0, i).contiguous() for i in idx]
    for r in range(D):
        tsp.kv_project(dims, sw, r, x_loc[r], K, V, ws)
    Y = torch.zeros(T, h, dtype=y_dtype, device="cuda")
    inter = []
    for r in range(D):
        y = torch.empty(T // D, h, dtype=y_dtype, device="cuda")
        tsp.layer_forward(dims, sw, r, x_loc[r], K, V, y, ws)
        Y[idx[r]] = y
        inter.append({n: tsp.workspace_view(ws, dims, D, n).clone() for n in ("q", "a", "y1", "h", "xn")})
    assert tsp.get_device_status(ws) == tsp.TSP_OK
    torch.cuda.synchronize()
    return raw, K, V, Y, idx, inter


@pytest.mark.parametrize("T,h,H,F,D,seed", [
    (512, 256, 4, 1024, 2, 0),     # the tiny TSP layer
    (512, 256, 4, 1024, 1, 5),     # D = 1: plain layer
    (1024, 256, 4, 1024, 4, 6),    # h/D = 64, F/D = 256
    (800, 256, 4, 1024, 2, 7),     # ragged chunks: c = 200
    (288, 256, 2, 512, 2, 8),      # head_dim 128, c = 72 (< one tile)
    (2048, 512, 4, 2048, 2, 9),    # head_dim 128, several tiles per chunk
    (768, 384, 6, 1536, 3, 10),    # D = 3 (not a power of two), h/D = 128
    (960, 320, 5, 1280, 5, 11),    # D = 5, h/D = 64, ragged chunks c = 96
    (1536, 384, 3, 1536, 3, 13),   # head_dim 128 with one head per shard, D = 3
    (8, 256, 4, 1024, 4, 12),      # degenerate chunks: c = 1, two local rows per rank
    (256, 8192, 64, 16384, 2, 14),  # the widest rows supported (h = 8192, 64 heads of 128)
])
def test_full_sequence_all_ranks(T, h, H, F, D, seed):
    raw, K, V, Y, idx, inter = run_full_sequence(T, h, H, F, D, seed)
    x = f64(raw["x"])
    plain = O.layer_forward(x, weights_f64(raw), H, storage=None)
    assert_layer_close(f64(Y), plain["y"], f"T={T} D={D} vs plain layer", x)
    ref = O.layer_forward(x, weights_f64(raw), H)
    assert_layer_close(f64(Y), ref["y"], f"T={T} D={D}", x)
    for name, got in (("k", K), ("v", V)):
        assert_operand_close(f64(got), ref[name], name)
    for r in range(D):
        rows = idx[r].cpu().numpy()
        for n, gate in (("q", 1e-3), ("a", 2e-3), ("h", 2e-3)):
            rl = rel_l2(f64(inter[r][n]), ref[n][rows])
            assert rl <= gate, (r, n, rl)
        # the attention projection Y1 - X = A Wo carries A's relative error, so
        # it takes A's gate; Y1 itself is dominated by X in small layers (there
        # |A Wo| ~ 0.01 |X|) and by A Wo at h = 8192 (|A Wo| ~ 2 |X|)
        rl = rel_l2(f64(inter[r]["y1"]) - x[rows], ref["y1"][rows] - x[rows])
        assert rl <= 2e-3, (r, "y1 - x", rl)


def test_bf16_output_is_rounded_fp32_output():
    T, h, H, F, D = 1024, 256, 4, 1024, 2
    raw = to_cuda(inputs.layer_inputs(T, h, F, 11))
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, raw)
    ws = tsp.alloc_workspace(dims, D)
    K = torch.zeros(T, h, dtype=torch.float16, device="cuda")
    V = torch.zeros_like(K)
    for r in range(D):
        xl = raw["x"].index_select(0, tsp.zigzag_index(T, D, r).long()).contiguous()
        tsp.kv_project(dims, sw, r, xl, K, V, ws)
    xl = raw["x"].index_select(0, tsp.zigzag_index(T, D, 1).long()).contiguous()
    y32 = torch.empty(T // D, h, dtype=torch.float32, device="cuda")
    y16 = torch.empty(T // D, h, dtype=torch.bfloat16, device="cuda")
    tsp.layer_forward(dims, sw, 1, xl, K, V, y32, ws)
    tsp.layer_forward(dims, sw, 1, xl, K, V, y16, ws)
    torch.cuda.synchronize()
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))


def test_rank_step_equals_projection_then_layer():
    T, h, H, F, D = 2048, 512, 4, 2048, 4
    raw = to_cuda(inputs.layer_inputs(T, h, F, 12))
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, raw)
    ws = tsp.alloc_workspace(dims, D)
    K = torch.zeros(T, h, dtype=torch.float16, device="cuda")
    V = torch.zeros_like(K)
    xs = [raw["x"].index_select(0, tsp.zigzag_index(T, D, r).long()).contiguous() for r in range(D)]
    for r in range(D):
        tsp.kv_project(dims, sw, r, xs[r], K, V, ws)
    K2, V2 = K.clone(), V.clone()
    r = 2
    ya = torch.empty(T // D, h, dtype=torch.float32, device="cuda")
    tsp.layer_forward(dims, sw, r, xs[r], K, V, ya, ws)
    # wipe the rank's own rows: rank_step must write them again
    for i in tsp.zigzag_index(T, D, r).long().cpu().tolist()[:: max(1, T // D // 8)]:
        K2[i].zero_()
        V2[i].zero_()
    yb = torch.empty_like(ya)
    tsp.rank_step(dims, sw, r, xs[r], K2, V2, yb, ws)
    torch.cuda.synchronize()
    assert torch.equal(K, K2) and torch.equal(V, V2)
    assert torch.equal(ya, yb)


def test_rank_step_host_buffers():
    T, h, H, F, D = 1024, 256, 4, 1024, 2
    raw = to_cuda(inputs.layer_inputs(T, h, F, 13))
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, raw)
    ws = tsp.alloc_workspace(dims, D)
    K = torch.zeros(T, h, dtype=torch.float16, device="cuda")
    V = torch.zeros_like(K)
    xs = [raw["x"].index_select(0, tsp.zigzag_index(T, D, r).long()).contiguous() for r in range(D)]
    for r in range(D):
        tsp.kv_project(dims, sw, r, xs[r], K, V, ws)
    yd = torch.empty(T // D, h, dtype=torch.float32, device="cuda")
    tsp.rank_step(dims, sw, 0, xs[0], K, V, yd, ws)
    hx = xs[0].cpu().pin_memory()
    hy = torch.empty(T // D, h, dtype=torch.float32).pin_memory()
    xst = torch.empty_like(xs[0])
    yst = torch.empty_like(yd)
    tsp.rank_step_host(dims, sw, 0, hx, xst, K, V, yst, hy, ws)
    torch.cuda.synchronize()
    assert torch.equal(hy, yd.cpu())


def test_rank_step_host_two_lanes_chained():
    """Steps alternating between two streams, each step's kernels ordered
    after the previous step's by the call's events (as the end-to-end bench
    runs them): every rank's host result equals its device rank step."""
    T, h, H, F, D = 2048, 512, 4, 2048, 4
    raw = to_cuda(inputs.layer_inputs(T, h, F, 17))
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, raw)
    L = T // D
    K = torch.zeros(T, h, dtype=torch.float16, device="cuda")
    V = torch.zeros_like(K)
    ws0 = tsp.alloc_workspace(dims, D)
    xs = [raw["x"].index_select(0, tsp.zigzag_index(T, D, r).long()).contiguous() for r in range(D)]
    for r in range(D):
        tsp.kv_project(dims, sw, r, xs[r], K, V, ws0)
    want = []
    for r in range(D):
        y = torch.empty(L, h, dtype=torch.bfloat16, device="cuda")
        tsp.rank_step(dims, sw, r, xs[r], K, V, y, ws0)
        want.append(y.cpu())
    torch.cuda.synchronize()
    lanes = [dict(stream=torch.cuda.Stream(), ws=tsp.alloc_workspace(dims, D), K=K.clone(), V=V.clone(),
                  xs=torch.empty(L, h, dtype=torch.bfloat16, device="cuda"),
                  ys=torch.empty(L, h, dtype=torch.bfloat16, device="cuda")) for _ in range(2)]
    done = [torch.cuda.Event(), torch.cuda.Event()]
    hx = [xs[r].cpu().pin_memory() for r in range(D)]
    hy = [torch.empty(L, h, dtype=torch.bfloat16).pin_memory() for _ in range(2 * D)]
    torch.cuda.synchronize()
    for i in range(2 * D):  # every rank twice
        ln, r = lanes[i % 2], i % D
        with torch.cuda.stream(ln["stream"]):
            tsp.rank_step_host(dims, sw, r, hx[r], ln["xs"], ln["K"], ln["V"], ln["ys"], hy[i], ln["ws"],
                               stream=ln["stream"], compute_after=done[(i - 1) % 2] if i > 0 else None,
                               compute_done=done[i % 2])
    torch.cuda.synchronize()
    for ln in lanes:
        assert tsp.get_device_status(ln["ws"]) == tsp.TSP_OK
    for i in range(2 * D):
        assert torch.equal(hy[i], want[i % D]), i


# --------------------------------------------------------------------------
# the 7B layer
# --------------------------------------------------------------------------
H7, h7, F7 = 32, 4096, 16384


def test_7b_layer_T8192_rank_in_full():
    T, D = 8192, 8
    raw = inputs.layer_inputs(T, h7, F7, 1)
    dev = to_cuda(raw)
    dims = tsp.make_dims(T, h7, H7, F7)
    sw = tsp.pack_shards(dims, D, dev)
    ws = tsp.alloc_workspace(dims, D)
    K = torch.zeros(T, h7, dtype=torch.float16, device="cuda")
    V = torch.zeros_like(K)
    xs = [dev["x"].index_select(0, tsp.zigzag_index(T, D, r).long()).contiguous() for r in range(D)]
    for r in range(D):
        tsp.kv_project(dims, sw, r, xs[r], K, V, ws)
    ys = {}
    for r in (0, 5):
        y = torch.empty(T // D, h7, dtype=torch.float32, device="cuda")
        tsp.layer_forward(dims, sw, r, xs[r], K, V, y, ws)
        ys[r] = y.cpu()
    assert tsp.get_device_status(ws) == tsp.TSP_OK
    x = f64(raw["x"])
    w = O.stored_weights(weights_f64(raw))
    w0 = O.stored_weights(weights_f64(raw), None)
    Kr, Vr = O.kv_project(x, w)
    K0, V0 = O.kv_project(x, w0, storage=None)
    for r, y in ys.items():
        idx = O.zigzag_index(T, D, r)
        plain = O.rank_rows_forward(x[idx], idx, K0, V0, w0, H7, storage=None)
        assert_layer_close(f64(y), plain["y"], f"7B T=8192 rank {r} vs plain layer", x[idx])
        ref = O.rank_rows_forward(x[idx], idx, Kr, Vr, w, H7)
        assert_layer_close(f64(y), ref["y"], f"7B T=8192 rank {r}", x[idx])
    assert_operand_close(f64(K), Kr, "k")
    assert_operand_close(f64(V), Vr, "v")


def sampled_rank_check(T, D, ranks, seed, n_sample=62):
    """Full-size launches (as benchmarked) of the given ranks on one set of
    inputs - the rank's tokens, the weights and stand-in all-gathered K/V - each
    checked on sampled rows (the first and last row of both chunks plus a
    seeded sample) against the plain fp64 layer and the fp16-storage oracle.
    Each rank's own K/V projection is checked on the same rows."""
    L = T // D
    c = L // 2
    raw = inputs.rank_inputs(L, T, h7, F7, seed)
    dev = to_cuda(raw)
    dims = tsp.make_dims(T, h7, H7, F7)
    sw = tsp.pack_shards(dims, D, dev)
    ws = tsp.alloc_workspace(dims, D)
    x = f64(raw["x_local"])
    w = O.stored_weights(weights_f64(raw))
    w0 = O.stored_weights(weights_f64(raw), None)
    Kf = raw["k_full"].float().numpy()
    Vf = raw["v_full"].float().numpy()
    y = torch.empty(L, h7, dtype=torch.float32, device="cuda")
    Kp = torch.zeros(T, h7, dtype=torch.float16, device="cuda")
    Vp = torch.zeros_like(Kp)
    for rank in ranks:
        tsp.layer_forward(dims, sw, rank, dev["x_local"], dev["k_full"], dev["v_full"], y, ws)
        # the rank's own K/V projection, into scratch copies
        tsp.kv_project(dims, sw, rank, dev["x_local"], Kp, Vp, ws)
        assert tsp.get_device_status(ws) == tsp.TSP_OK
        rows = inputs.sample_rows(L, n_sample, seed + rank, must=(0, c - 1, c, L - 1))
        pos = O.zigzag_index(T, D, rank)
        y_s = f64(y[rows])
        plain = O.rank_rows_forward(x[rows], pos[rows], Kf, Vf, w0, H7, storage=None)
        assert_layer_close(y_s, plain["y"], f"7B T={T} D={D} rank {rank} vs plain layer", x[rows])
        ref = O.rank_rows_forward(x[rows], pos[rows], Kf, Vf, w, H7)
        assert_layer_close(y_s, ref["y"], f"7B T={T} D={D} rank {rank}", x[rows])
        kr, vr = O.kv_project(x[rows], w)
        gk, gv = f64(Kp[torch.as_tensor(pos[rows])]), f64(Vp[torch.as_tensor(pos[rows])])
        assert_operand_close(gk, kr, "k rows")
        assert_operand_close(gv, vr, "v rows")


def test_7b_layer_128k_rank0_sampled():
    sampled_rank_check(131072, 8, [0], 2)


def test_7b_layer_128k_last_rank_sampled():
    sampled_rank_check(131072, 8, [7], 3, n_sample=30)


def test_7b_layer_128k_middle_ranks_sampled():
    """Ranks 1-6 of the full 128K layer (every rank of the all-ranks
    configuration is then checked at full size): each holds a different
    chunk pair, so each walks a different key range and tile mix."""
    sampled_rank_check(131072, 8, [1, 2, 3, 4, 5, 6], 3, n_sample=16)


def test_7b_layer_128k_kv_from_projection_sampled():
    """The whole 128K layer as the all-ranks configuration runs it: every rank's
    tsp_kv_project fills K and V over all 131072 tokens, then ranks 0 and 5 run
    their layer forward on those K/V; sampled rows of both are checked against
    the oracle, which projects K and V of the whole sequence itself (fp64,
    ~9 TFLOP of CPU work, the slowest check here)."""
    T, D, seed = 131072, 8, 3
    L = T // D
    c = L // 2
    raw = inputs.layer_inputs(T, h7, F7, seed)
    dev = to_cuda(raw)
    dims = tsp.make_dims(T, h7, H7, F7)
    sw = tsp.pack_shards(dims, D, dev)
    ws = tsp.alloc_workspace(dims, D)
    K = torch.zeros(T, h7, dtype=torch.float16, device="cuda")
    V = torch.zeros_like(K)
    xs = [dev["x"].index_select(0, tsp.zigzag_index(T, D, r).long()).contiguous() for r in range(D)]
    for r in range(D):
        tsp.kv_project(dims, sw, r, xs[r], K, V, ws)
    got = {}
    for r in (0, 5):
        y = torch.empty(L, h7, dtype=torch.float32, device="cuda")
        tsp.layer_forward(dims, sw, r, xs[r], K, V, y, ws)
        rows = inputs.sample_rows(L, 12, seed + r, must=(0, c - 1, c, L - 1))
        got[r] = (rows, f64(y[rows]))
    assert tsp.get_device_status(ws) == tsp.TSP_OK
    del K, V, dev, ws, sw, xs
    torch.cuda.empty_cache()
    x = f64(raw["x"])
    for storage in ("fp16", None):
        w = O.stored_weights(weights_f64(raw), storage)
        Kr, Vr = O.kv_project(x, w, storage=storage)
        for r, (rows, y_s) in got.items():
            pos = O.zigzag_index(T, D, r)[rows]
            ref = O.rank_rows_forward(x[pos], pos, Kr, Vr, w, H7, storage=storage)
            assert_layer_close(y_s, ref["y"], f"128K rank {r}, K/V projected by every rank, oracle {storage}", x[pos])
        del Kr, Vr


@pytest.mark.parametrize("D", [1, 2, 4, 8, 16])
def test_7b_layer_T32768_shard_sweep_sampled(D):
    sampled_rank_check(32768, D, [0], 4, n_sample=30)


@pytest.mark.parametrize("T,h,H,F,D,ramp,n_sample", [
    (512, 256, 4, 1024, 2, 60.0, None),       # head_dim 64, every row of both ranks
    (8192, 4096, 32, 16384, 8, 3.0, 62),      # head_dim 128, sampled rows of ranks 0 and 5
])
def test_growing_logits_force_rescales(T, h, H, F, D, ramp, n_sample):
    """K rows scaled by 1 + ramp * position / T: the logits grow along the
    sequence, so a row's running maximum grows by 17-25 in log2 units after
    its first key tile (about 0 at these sizes without the ramp), and the
    attention kernel's move of its offset (a tile whose probabilities would
    pass 2^15 is redone against the tile's maximum, O rescaled), including a
    growth of more than 2^16 inside one tile, runs many times.  The oracle
    takes the same fp16 K."""
    L = T // D
    raw = inputs.rank_inputs(L, T, h, F, 7)
    g = 1.0 + ramp * torch.arange(T, dtype=torch.float32) / T
    k_ramp = (raw["k_full"].float() * g[:, None]).to(torch.float16)
    assert torch.isfinite(k_ramp).all()
    dev = to_cuda({n: raw[n] for n in inputs.WEIGHT_NAMES})
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, dev)
    ws = tsp.alloc_workspace(dims, D)
    Kd, Vd = k_ramp.cuda(), raw["v_full"].cuda()
    w = O.stored_weights(weights_f64(raw))
    w0 = O.stored_weights(weights_f64(raw), None)
    Kf = k_ramp.double().numpy()
    Vf = raw["v_full"].double().numpy()
    x_all = f64(raw["x_local"])
    for r in (0, D - 3 if D > 2 else 1):
        y = torch.empty(L, h, dtype=torch.float32, device="cuda")
        tsp.layer_forward(dims, sw, r, raw["x_local"].cuda(), Kd, Vd, y, ws)
        assert tsp.get_device_status(ws) == tsp.TSP_OK
        pos = O.zigzag_index(T, D, r)
        rows = np.arange(L) if n_sample is None else inputs.sample_rows(L, n_sample, 7 + r, must=(0, L // 2, L - 1))
        plain = O.rank_rows_forward(x_all[rows], pos[rows], Kf, Vf, w0, H, storage=None)
        assert_layer_close(f64(y)[rows], plain["y"], f"growing logits T={T} D={D} rank {r} vs plain layer",
                           x_all[rows])
        ref = O.rank_rows_forward(x_all[rows], pos[rows], Kf, Vf, w, H)
        assert_layer_close(f64(y)[rows], ref["y"], f"growing logits T={T} D={D} rank {r}", x_all[rows])


@pytest.mark.parametrize("T,h,H,F,D,spike", [
    (512, 256, 4, 1024, 2, 2000.0),     # head_dim 64, every row of both ranks
    (2048, 512, 4, 2048, 2, 1500.0),    # head_dim 128
])
def test_score_jumps_beyond_fp32_range(T, h, H, F, D, spike):
    """Every 97th K row from position 200 on scaled by `spike`: a query's
    score against such a key exceeds the maximum of the query's first key
    tile by hundreds of log2 units (2^x overflows fp32), or by 8 to 128 units
    (2^x overflows fp16), or falls far below it, at random
    (test_score_jump_inputs.py checks on the CPU that all three occur).  The
    offset the attention kernel subtracts must follow the row's maximum in
    all three cases.  The gate is the oracle that rounds Q, K, V and A to fp16 where
    the kernels store them: with scores hundreds of units apart, Q's fp16
    rounding alone (relative 2^-11) moves a score by a tenth of a unit, which
    the softmax turns into output changes above the plain layer's max-abs
    2e-2 in any fp16 implementation; the plain fp64 layer is checked at
    rel-L2 5e-3 only."""
    L = T // D
    raw = inputs.rank_inputs(L, T, h, F, 9)
    kf = raw["k_full"].float()
    spikes = torch.arange(200, T, 97)
    kf[spikes] *= spike
    k_spiked = kf.to(torch.float16)
    assert torch.isfinite(k_spiked).all()
    dev = to_cuda({n: raw[n] for n in inputs.WEIGHT_NAMES})
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, dev)
    ws = tsp.alloc_workspace(dims, D)
    Kd, Vd = k_spiked.cuda(), raw["v_full"].cuda()
    Kf = k_spiked.double().numpy()
    Vf = raw["v_full"].double().numpy()
    x_all = f64(raw["x_local"])
    for r in range(D):
        y = torch.empty(L, h, dtype=torch.float32, device="cuda")
        tsp.layer_forward(dims, sw, r, raw["x_local"].cuda(), Kd, Vd, y, ws)
        assert tsp.get_device_status(ws) == tsp.TSP_OK
        pos = O.zigzag_index(T, D, r)
        w = O.stored_weights(weights_f64(raw))
        ref = O.rank_rows_forward(x_all, pos, Kf, Vf, w, H)
        assert_layer_close(f64(y), ref["y"], f"score jumps T={T} rank {r}", x_all)
        plain = O.rank_rows_forward(x_all, pos, Kf, Vf, O.stored_weights(weights_f64(raw), None), H, storage=None)
        rl = np.linalg.norm(f64(y) - plain["y"]) / np.linalg.norm(plain["y"])
        assert rl <= 5e-3, f"score jumps T={T} rank {r} vs plain layer: rel-L2 {rl:.3e}"


# --------------------------------------------------------------------------
# fp16 range: saturations are reported, not silent
# --------------------------------------------------------------------------
def test_fp16_saturation_is_reported():
    """Values beyond fp16's range are clamped to +-65504 and recorded in the
    status section: a weight when the shards are packed, and a Q entry in the
    QKV GEMM's epilogue.  Wq scaled by 1e5 (entries ~2000, representable)
    gives Q entries of std 16 * 2000 = 32000, so some exceed 65504; the
    inputs as drawn give none."""
    T, h, H, F, D = 512, 256, 4, 1024, 2
    raw = to_cuda(inputs.layer_inputs(T, h, F, 30))
    dims = tsp.make_dims(T, h, H, F)
    ws = tsp.alloc_workspace(dims, D)
    xs = [raw["x"].index_select(0, tsp.zigzag_index(T, D, r).long()).contiguous() for r in range(D)]
    y = torch.empty(T // D, h, dtype=torch.float32, device="cuda")

    def run(w_full):
        sw = tsp.pack_shards(dims, D, w_full)
        K = torch.zeros(T, h, dtype=torch.float16, device="cuda")
        V = torch.zeros_like(K)
        tsp.reset_device_status(ws)
        for r in range(D):
            tsp.kv_project(dims, sw, r, xs[r], K, V, ws)
        tsp.layer_forward(dims, sw, 0, xs[0], K, V, y, ws)
        return sw
    sw = run(raw)
    assert tsp.get_device_status(sw.buf) == tsp.TSP_OK
    assert tsp.get_device_status(ws) == tsp.TSP_OK
    big = dict(raw)
    big["wq"] = (raw["wq"].float() * 1e5).to(torch.bfloat16)
    sw = run(big)
    assert tsp.get_device_status(sw.buf) == tsp.TSP_OK          # the weights fit fp16
    assert tsp.get_device_status(ws) == tsp.TSP_ERR_SATURATED   # some Q entries did not
    assert torch.isfinite(y).all()
    tsp.reset_device_status(ws)
    assert tsp.get_device_status(ws) == tsp.TSP_OK
    huge = dict(raw)
    huge["w1"] = raw["w1"].clone()
    huge["w1"][3, 5] = 1.0e6
    sw = tsp.pack_shards(dims, D, huge)
    assert tsp.get_device_status(sw.buf) == tsp.TSP_ERR_SATURATED
    Fs = F // D
    assert sw.shard("w1", 5 // Fs, (Fs, h))[5 % Fs, 3].item() == 65504.0


# --------------------------------------------------------------------------
# failure detection without a GPU fault
# --------------------------------------------------------------------------
def test_bounded_wait_times_out_and_context_survives():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    assert tsp.get_device_status(ws) == tsp.TSP_OK
    tsp.selftest_wait_timeout(ws, 20_000_000)  # 20 ms
    assert tsp.get_device_status(ws) == tsp.TSP_ERR_TIMEOUT
    tsp.reset_device_status(ws)
    assert tsp.get_device_status(ws) == tsp.TSP_OK
    # the context still runs real work
    got = tsp.zigzag_index(512, 2, 1).cpu().numpy()
    assert np.array_equal(got.astype(np.int64), O.zigzag_index(512, 2, 1))


def test_empty_sequence():
    dims = tsp.make_dims(0, 256, 4, 1024)
    raw = to_cuda(inputs.layer_inputs(4, 256, 1024, 0))
    sw = tsp.pack_shards(tsp.make_dims(4, 256, 4, 1024), 2, raw)
    ws = tsp.alloc_workspace(dims, 2)
    e = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    e16 = torch.empty(0, 256, dtype=torch.float16, device="cuda")
    tsp.layer_forward(dims, sw, 0, e, e16, e16, torch.empty(0, 256, device="cuda"), ws)
    torch.cuda.synchronize()
