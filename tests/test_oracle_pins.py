"""Pins for the CPU oracle: each check compares it with something other than itself.

Sources of truth used here (no value comes from the CUDA path):
* closed forms (equal causal work per rank, LayerNorm moments, GELU's odd
  part, running means of V under uniform attention),
* brute force in pure Python loops on tiny inputs,
* independent library routines: torch's fp32->bf16 cast, F.layer_norm,
  F.gelu(approximate='tanh'), F.scaled_dot_product_attention(is_causal=True),
  composed into the whole layer in torch fp64,
* the one printed example of the partition (tests/golden/zigzag_T512_D2.txt),
* planted mistakes: a plausible bug put into the oracle (on the CPU) must make
  at least one of these pins fail.
"""
import math
import os
import re

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

from folded_tensor_sequence_rank_b200 import inputs
from oracle import tsp_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# helpers written independently of the oracle
# --------------------------------------------------------------------------
def bf16_rne_bits(t: torch.Tensor) -> torch.Tensor:
    """fp64 -> nearest bf16 (ties to even) by integer rounding of the fp64 bit
    pattern: drop the low 45 of 52 fraction bits with round-half-even."""
    bits = t.contiguous().view(torch.int64)
    lsb = (bits >> 45) & 1
    bits = (bits + ((1 << 44) - 1) + lsb) & ~((1 << 45) - 1)
    return bits.view(torch.float64)


def fp16_rne_bits(t: torch.Tensor) -> torch.Tensor:
    """fp64 -> nearest IEEE half (ties to even): for |x| >= 2^-14 drop the low
    42 of 52 fraction bits with round-half-even on the bit pattern; below that
    the half grid is uniform with step 2^-24, rounded with torch.round (which
    rounds halves to even)."""
    t = t.contiguous()
    bits = t.view(torch.int64)
    lsb = (bits >> 42) & 1
    normal = ((bits + ((1 << 41) - 1) + lsb) & ~((1 << 42) - 1)).view(torch.float64)
    sub = torch.round(t * 2.0 ** 24) / 2.0 ** 24
    return torch.where(t.abs() >= 2.0 ** -14, normal, sub)


ROUNDERS = {None: (lambda t: t), "fp16": fp16_rne_bits, "bf16": bf16_rne_bits}


def torch_layer(x, w, n_heads, eps=1e-5, storage="fp16"):
    """The layer composed from torch library routines, in fp64."""
    rd = ROUNDERS[storage]
    X = torch.as_tensor(np.asarray(x, dtype=np.float64))
    W = {n: rd(torch.as_tensor(np.asarray(a, dtype=np.float64))) for n, a in w.items()}
    T, h = X.shape
    d = h // n_heads
    xn = rd(Fn.layer_norm(X, (h,), eps=eps))
    q, k, v = (rd(Fn.linear(xn, W[n].t())) for n in ("wq", "wk", "wv"))

    def heads(t):
        return t.view(T, n_heads, d).transpose(0, 1).unsqueeze(0)

    att = Fn.scaled_dot_product_attention(heads(q), heads(k), heads(v), is_causal=True)
    a = rd(att[0].transpose(0, 1).reshape(T, h))
    y1 = X + Fn.linear(a, W["wo"].t())
    xn2 = rd(Fn.layer_norm(y1, (h,), eps=eps))
    hh = rd(Fn.gelu(Fn.linear(xn2, W["w1"].t()), approximate="tanh"))
    y = y1 + Fn.linear(hh, W["w2"].t())
    return {"y": y.numpy(), "k": k.numpy(), "v": v.numpy(), "a": a.numpy(),
            "h": hh.numpy(), "y1": y1.numpy()}


def f64(t):
    return t.to(torch.float64).numpy()


TINY = dict(T=64, h=64, H=4, F=256)        # d = 16
SMALL = dict(T=512, h=256, H=4, F=1024)    # the tiny TSP workload's layer, d = 64


def tiny_inputs(cfg, seed):
    raw = inputs.layer_inputs(cfg["T"], cfg["h"], cfg["F"], seed)
    return f64(raw["x"]), {n: f64(raw[n]) for n in inputs.WEIGHT_NAMES}


# --------------------------------------------------------------------------
# bf16 rounding
# --------------------------------------------------------------------------
def test_round_bf16_matches_torch_cast_on_fp32_values():
    g = torch.Generator().manual_seed(11)
    vals = torch.cat([torch.randn(20000, generator=g) * s for s in (1e-3, 1.0, 37.0)])
    bits = torch.randint(0, 1 << 30, (4000,), generator=g, dtype=torch.int64)
    # exact halfway cases and their neighbours (low 16 bits 0x8000, 0x7fff, 0x8001)
    base = (bits << 16) & 0x3FFF0000 | 0x3C000000
    ties = torch.cat([base | 0x8000, base | 0x7FFF, base | 0x8001, base | 0x18000])
    ties = ties.to(torch.int32).view(torch.float32)
    vals = torch.cat([vals, ties, -ties])
    ref = vals.to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(vals.to(torch.float64).numpy())
    assert np.array_equal(got, ref)


def test_round_fp16_matches_torch_cast_on_fp32_values():
    g = torch.Generator().manual_seed(17)
    vals = torch.cat([torch.randn(20000, generator=g) * s for s in (1e-6, 1e-4, 1.0, 300.0)])
    bits = torch.randint(0, 1 << 20, (4000,), generator=g, dtype=torch.int64)
    # fp32 values exactly halfway between halves, and next to halfway
    base = ((bits << 13) & 0x0FFFE000) | 0x38000000
    ties = torch.cat([base | 0x1000, base | 0x0FFF, base | 0x1001]).to(torch.int32).view(torch.float32)
    vals = torch.cat([vals, ties, -ties])
    ref = vals.to(torch.float16).to(torch.float64).numpy()
    got = O.round_fp16(vals.to(torch.float64).numpy())
    assert np.array_equal(got, ref)


def test_round_fp16_direct_from_fp64():
    assert O.round_fp16(np.array([1 + 2 ** -11 + 2 ** -40]))[0] == 1 + 2 ** -10  # just above a tie
    assert O.round_fp16(np.array([1 + 2 ** -11]))[0] == 1.0                      # tie -> even
    assert O.round_fp16(np.array([2 ** -25]))[0] == 0.0                          # subnormal tie -> even
    assert O.round_fp16(np.array([3 * 2 ** -25]))[0] == 2 ** -23
    x = np.random.default_rng(4).standard_normal(50000) * np.repeat([1e-6, 1e-3, 1.0, 50.0], 12500)
    assert np.array_equal(O.round_fp16(x), fp16_rne_bits(torch.as_tensor(x)).numpy())


def test_round_bf16_direct_from_fp64():
    # 1 + 2^-8 + 2^-30 sits just above the midpoint between 1 and 1 + 2^-7
    assert O.round_bf16(np.array([1 + 2 ** -8 + 2 ** -30]))[0] == 1 + 2 ** -7
    assert O.round_bf16(np.array([1 + 2 ** -8]))[0] == 1.0            # tie -> even
    assert O.round_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6  # tie -> even
    x = np.random.default_rng(3).standard_normal(50000) * 5
    assert np.array_equal(O.round_bf16(x), bf16_rne_bits(torch.as_tensor(x)).numpy())


# --------------------------------------------------------------------------
# zigzag partition
# --------------------------------------------------------------------------
def test_zigzag_matches_printed_example():
    ranges = {}
    with open(os.path.join(GOLDEN, "zigzag_T512_D2.txt")) as f:
        for line in f:
            m = re.match(r"rank (\d+): (.*)", line.strip())
            if not m:
                continue
            idx = []
            for part in m.group(2).split(","):
                a, b = part.strip().split("..")
                idx.extend(range(int(a), int(b) + 1))
            ranges[int(m.group(1))] = idx
    for r, expect in ranges.items():
        assert O.zigzag_index(512, 2, r).tolist() == expect


@pytest.mark.parametrize("T,D", [(8, 1), (16, 2), (48, 3), (64, 4), (512, 2), (8192, 8), (4096, 16)])
def test_zigzag_is_a_permutation_with_equal_causal_work(T, D):
    c = T // (2 * D)
    seen = np.concatenate([O.zigzag_index(T, D, r) for r in range(D)])
    assert sorted(seen.tolist()) == list(range(T))
    closed = c * c * (2 * D - 1) + c * (c + 1)
    # brute force: count pairs (query p, key j) with j <= p over each rank's tokens
    for r in range(D):
        idx = O.zigzag_index(T, D, r)
        assert len(idx) == 2 * c
        assert O.causal_pairs(T, D, r) == closed
        if T <= 64:
            assert sum(1 for p in idx.tolist() for j in range(T) if j <= p) == closed


def test_zigzag_equal_work_values():
    assert O.causal_pairs(512, 2, 0) == 65664
    assert O.causal_pairs(8192, 8, 3) == 4194816
    assert O.causal_pairs(131072, 8, 7) == 1073750016


def test_zigzag_rejects_bad_arguments():
    with pytest.raises(ValueError):
        O.zigzag_index(10, 2, 0)
    with pytest.raises(ValueError):
        O.zigzag_index(16, 2, 2)


# --------------------------------------------------------------------------
# LayerNorm, GELU
# --------------------------------------------------------------------------
def test_layer_norm_closed_form_and_library():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 256)) * rng.uniform(0.01, 30, (64, 1)) + rng.uniform(-5, 5, (64, 1))
    y = O.layer_norm(x, 1e-5)
    var_in = x.var(axis=1)
    assert np.allclose(y.mean(axis=1), 0, atol=1e-12)
    assert np.allclose(y.var(axis=1), var_in / (var_in + 1e-5), rtol=1e-12)
    ref = Fn.layer_norm(torch.as_tensor(x), (256,), eps=1e-5).numpy()
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_gelu_tanh_identities_and_library():
    x = np.linspace(-12, 12, 4801)
    g = O.gelu_tanh(x)
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert np.allclose(g - O.gelu_tanh(-x), x, atol=1e-13)          # odd part is x/2
    assert np.allclose(g[x > 8], x[x > 8], rtol=1e-12)                # -> identity
    assert np.all(np.abs(g[x < -8]) < 1e-12)                          # -> 0
    ref = Fn.gelu(torch.as_tensor(x), approximate="tanh").numpy()
    assert np.allclose(g, ref, rtol=1e-13, atol=1e-15)


# --------------------------------------------------------------------------
# causal attention
# --------------------------------------------------------------------------
def brute_force_attention(q, k, v, q_pos, n_heads, scale):
    n, hd = len(q), len(q[0])
    d = hd // n_heads
    out = [[0.0] * hd for _ in range(n)]
    for i in range(n):
        for hh in range(n_heads):
            s = []
            for j in range(q_pos[i] + 1):
                s.append(scale * sum(q[i][hh * d + t] * k[j][hh * d + t] for t in range(d)))
            mx = max(s)
            e = [math.exp(z - mx) for z in s]
            tot = sum(e)
            for t in range(d):
                out[i][hh * d + t] = sum(e[j] * v[j][hh * d + t] for j in range(len(e))) / tot
    return out


def test_attention_brute_force_tiny():
    rng = np.random.default_rng(9)
    T, H, d = 12, 2, 3
    q, k, v = (rng.standard_normal((T, H * d)) for _ in range(3))
    pos = np.array([0, 5, 11, 3, 7])
    got = O.causal_attention(q[pos], k, v, pos, H, 0.7)
    ref = brute_force_attention(q[pos].tolist(), k.tolist(), v.tolist(), pos.tolist(), H, 0.7)
    assert np.allclose(got, np.array(ref), rtol=1e-12, atol=1e-12)


def test_attention_probabilities_rows_sum_to_one_and_are_causal():
    rng = np.random.default_rng(10)
    T, H, d = 40, 2, 8
    q, k, v = (rng.standard_normal((T, H * d)) * 2 for _ in range(3))
    pos = np.arange(T)
    out, probs = O.causal_attention(q, k, v, pos, H, 1 / math.sqrt(d), return_probs=True)
    for p in probs:
        assert np.allclose(p.sum(axis=1), 1.0, atol=1e-14)
        assert np.all(p[np.triu_indices(T, 1)] == 0.0)
    # the query at position 0 sees key 0 only: its output is V[0]
    assert np.allclose(out[0], v[0], rtol=0, atol=1e-15)


def test_attention_uniform_keys_give_running_mean_of_values():
    rng = np.random.default_rng(12)
    T, H, d = 30, 3, 4
    q = rng.standard_normal((T, H * d))
    k = np.tile(rng.standard_normal((1, H * d)), (T, 1))   # every key identical
    v = rng.standard_normal((T, H * d))
    out = O.causal_attention(q, k, v, np.arange(T), H, 0.5)
    running = np.cumsum(v, axis=0) / np.arange(1, T + 1)[:, None]
    assert np.allclose(out, running, rtol=1e-12, atol=1e-12)


def test_attention_matches_sdpa_and_zigzag_rows():
    rng = np.random.default_rng(13)
    T, H, d = 64, 4, 16
    q, k, v = (rng.standard_normal((T, H * d)) for _ in range(3))
    out = O.causal_attention(q, k, v, np.arange(T), H, 1 / math.sqrt(d))
    tq, tk, tv = (torch.as_tensor(a).view(T, H, d).transpose(0, 1)[None] for a in (q, k, v))
    ref = Fn.scaled_dot_product_attention(tq, tk, tv, is_causal=True)[0].transpose(0, 1).reshape(T, H * d)
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
    for r in range(4):
        idx = O.zigzag_index(T, 4, r)
        rows = O.causal_attention(q[idx], k, v, idx, H, 1 / math.sqrt(d))
        assert np.allclose(rows, out[idx], rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------
# whole layer against the independent torch composition
# --------------------------------------------------------------------------
@pytest.mark.parametrize("cfg,seed", [(TINY, 1), (SMALL, 0)])
@pytest.mark.parametrize("storage", [None, "fp16", "bf16"])
def test_layer_matches_torch_composition(cfg, seed, storage):
    x, w = tiny_inputs(cfg, seed)
    got = O.layer_forward(x, w, cfg["H"], storage=storage)
    ref = torch_layer(x, w, cfg["H"], storage=storage)
    for key in ("k", "v", "a", "y1", "h", "y"):
        assert np.allclose(got[key], ref[key], rtol=1e-10, atol=1e-10), key
    # the storage points really round: stored operands are 16-bit numbers
    if storage is not None:
        rnd = O.round_fp16 if storage == "fp16" else O.round_bf16
        for key in ("xn1", "q", "a", "xn2", "h", "k", "v"):
            assert np.array_equal(got[key], rnd(got[key])), key


# --------------------------------------------------------------------------
# the TSP schedule equals the plain layer  (sum over shards = full contraction)
# --------------------------------------------------------------------------
ODD = dict(T=120, h=120, H=15, F=480)      # d = 8; divisible by D = 3, 5, 15


@pytest.mark.parametrize("cfg,D", [(TINY, 1), (TINY, 2), (TINY, 4), (ODD, 3), (ODD, 5), (ODD, 15)])
def test_sharded_schedule_equals_unsharded_layer(cfg, D):
    x, w = tiny_inputs(cfg, 21 + D)
    full = O.layer_forward(x, w, cfg["H"])
    K, V = O.kv_all_gather_sharded(x, D, w)
    assert np.array_equal(K, full["k"]) and np.array_equal(V, full["v"])
    for r in range(D):
        idx = O.zigzag_index(cfg["T"], D, r)
        y = O.rank_forward_sharded(r, D, x[idx], K, V, w, cfg["H"])
        assert np.allclose(y, full["y"][idx], rtol=1e-11, atol=1e-11)
        rows = O.rank_rows_forward(x[idx], idx, K, V, w, cfg["H"])
        assert np.allclose(rows["y"], full["y"][idx], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("storage", [None, "fp16", "bf16"])
def test_stored_weights_give_identical_results(storage):
    """Weights rounded once (stored_weights) and handed to the layer functions
    give bit-identical outputs: rounding to nearest is idempotent, so the
    pre-rounding only saves the per-call rounding work."""
    cfg = TINY
    x, w = tiny_inputs(cfg, 33)
    sw = O.stored_weights(w, storage)
    a = O.layer_forward(x, w, cfg["H"], storage=storage)
    b = O.layer_forward(x, sw, cfg["H"], storage=storage)
    for key in ("k", "v", "q", "a", "y1", "h", "y"):
        assert np.array_equal(a[key], b[key]), key
    # weights stored for another format are rounded again to this one
    w_off = {n: a_ * (1.0 + 2.0 ** -20) for n, a_ in w.items()}   # not 16-bit numbers
    other = O.stored_weights(w_off, None)
    c = O.layer_forward(x, other, cfg["H"], storage=storage)
    d = O.layer_forward(x, w_off, cfg["H"], storage=storage)
    assert np.array_equal(c["y"], d["y"])


def test_d1_reduces_to_plain_layer():
    cfg = TINY
    x, w = tiny_inputs(cfg, 31)
    full = O.layer_forward(x, w, cfg["H"], storage=None)
    y = O.rank_forward_sharded(0, 1, x, full["k"], full["v"], w, cfg["H"], storage=None)
    assert np.allclose(y, full["y"], rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# planted mistakes: each must be caught by the pins above
# --------------------------------------------------------------------------
def _layer_error(monkeypatch_fn=None):
    cfg = TINY
    x, w = tiny_inputs(cfg, 41)
    got = O.layer_forward(x, w, cfg["H"], storage=None)
    ref = torch_layer(x, w, cfg["H"], storage=None)
    return float(np.max(np.abs(got["y"] - ref["y"])))


MISTAKES = {
    "gelu drops the cubic term": ("gelu_tanh", lambda x: 0.5 * np.asarray(x) * (1 + np.tanh(np.sqrt(2 / np.pi) * np.asarray(x)))),
    "layer norm uses unbiased variance": ("layer_norm", lambda x, eps=1e-5: (np.asarray(x) - np.asarray(x).mean(-1, keepdims=True)) / np.sqrt(np.asarray(x).var(-1, ddof=1, keepdims=True) + eps)),
    "layer norm drops eps": ("layer_norm", lambda x, eps=1e-5: (np.asarray(x) - np.asarray(x).mean(-1, keepdims=True)) / np.asarray(x).std(-1, keepdims=True)),
}


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_planted_elementwise_mistakes_are_caught(monkeypatch, name):
    attr, bad = MISTAKES[name]
    assert _layer_error() < 1e-10
    monkeypatch.setattr(O, attr, bad)
    assert _layer_error() > 1e-8, name  # the composition pin tolerates 1e-10


def test_planted_attention_mistakes_are_caught(monkeypatch):
    good = O.causal_attention

    def no_mask(q, k, v, q_pos, n_heads, scale, return_probs=False):
        T = np.asarray(k).shape[0]
        return good(q, k, v, np.full_like(np.asarray(q_pos), T - 1), n_heads, scale, return_probs)

    def off_by_one(q, k, v, q_pos, n_heads, scale, return_probs=False):
        return good(q, k, v, np.maximum(np.asarray(q_pos) - 1, 0), n_heads, scale, return_probs)

    def wrong_scale(q, k, v, q_pos, n_heads, scale, return_probs=False):
        return good(q, k, v, q_pos, n_heads, scale * 2, return_probs)

    for bad in (no_mask, off_by_one, wrong_scale):
        monkeypatch.setattr(O, "causal_attention", bad)
        assert _layer_error() > 1e-6, bad.__name__
    monkeypatch.setattr(O, "causal_attention", good)
    assert _layer_error() < 1e-10


def test_planted_shard_mistakes_are_caught(monkeypatch):
    cfg, D = TINY, 2
    x, w = tiny_inputs(cfg, 51)
    full = O.layer_forward(x, w, cfg["H"])
    K, V = O.kv_all_gather_sharded(x, D, w)
    idx = O.zigzag_index(cfg["T"], D, 1)
    good_zz = O.zigzag_index
    # a zigzag map that hands rank r chunks r and 2D-2-r (wrong mirror)
    def bad_zz(T, D_, rank):
        c = T // (2 * D_)
        return np.concatenate([np.arange(rank * c, (rank + 1) * c),
                               np.arange(((2 * D_ - 2 - rank) % (2 * D_)) * c, ((2 * D_ - 2 - rank) % (2 * D_) + 1) * c)])
    monkeypatch.setattr(O, "zigzag_index", bad_zz)
    y = O.rank_forward_sharded(1, D, x[idx], K, V, w, cfg["H"])
    assert not np.allclose(y, full["y"][idx], atol=1e-6)
    monkeypatch.setattr(O, "zigzag_index", good_zz)
    # Wo applied transposed
    w_bad = dict(w, wo=w["wo"].T.copy())
    y = O.rank_forward_sharded(1, D, x[idx], K, V, w_bad, cfg["H"])
    assert not np.allclose(y, full["y"][idx], atol=1e-6)


def test_gpu_parity_gates_reject_planted_attention_mistakes(monkeypatch):
    """The forward GPU tests gate the attention output A at rel-L2 <= 2e-3 and
    the layer's own contribution Y - X at 2e-2 (tests/test_gpu_parity.py).  On
    the tiny layer, where attention is close to uniform averaging, each
    plausible attention bug still moves A well beyond its gate (CPU only)."""
    raw = inputs.layer_inputs(512, 256, 1024, 0)
    x = raw["x"].double().numpy()
    w = {n: raw[n].double().numpy() for n in inputs.WEIGHT_NAMES}
    ref = O.layer_forward(x, w, 4)
    good = O.causal_attention

    def off_by_one(q, k, v, q_pos, n_heads, scale, return_probs=False):
        return good(q, k, v, np.maximum(np.asarray(q_pos) - 1, 0), n_heads, scale, return_probs)

    def wrong_scale(q, k, v, q_pos, n_heads, scale, return_probs=False):
        return good(q, k, v, q_pos, n_heads, scale * 2 ** 0.5, return_probs)

    def no_mask(q, k, v, q_pos, n_heads, scale, return_probs=False):
        return good(q, k, v, np.full_like(np.asarray(q_pos), np.asarray(k).shape[0] - 1), n_heads, scale,
                    return_probs)

    def rel(a, b):
        return float(np.linalg.norm(a - b) / np.linalg.norm(b))
    for bad in (off_by_one, wrong_scale, no_mask):
        monkeypatch.setattr(O, "causal_attention", bad)
        out = O.layer_forward(x, w, 4)
        assert rel(out["a"], ref["a"]) > 10 * 2e-3 or rel(out["y"] - x, ref["y"] - x) > 2e-2, bad.__name__
