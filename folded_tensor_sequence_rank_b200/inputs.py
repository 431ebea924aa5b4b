"""Seeded synthetic inputs shared by the CUDA path, the tests and the oracle.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic (no zigzag map, no shard split, no normalisation), so
both sides of a parity check can take their inputs from it without sharing
any of the computation under test.

Recipe (one ``torch.Generator('cpu')`` stream per call, fp32 normal draws,
each tensor rounded once to bf16 round-to-nearest-even):

* ``layer_inputs``: X [T, h] ~ N(0, 1), then Wq, Wk, Wv, Wo [h, h],
  W1 [h, F], W2 [F, h] ~ N(0, 0.02^2), all in the math orientation
  ``y = x @ W`` ([in, out]).
* ``rank_inputs``: the rank's own tokens x_local [L, h] ~ N(0, 1), the six
  weights as above, then a stand-in for the all-gathered key/value tensors
  K, V [T, h] ~ N(0, kv_std^2), rounded to fp16 (the format the layer keeps
  K and V in) instead of bf16.  ``kv_std`` defaults to 0.02*sqrt(h), the
  standard deviation of LayerNorm(x) @ W for such weights, so attention
  logits have the spread the real projection gives.
* ``mlp_backward_inputs``: the rank's residual rows Y1 [L, h] ~ N(0, 1) kept
  in fp32 (the residual stream is fp32), the six weights as above, then the
  loss gradient dY [L, h] ~ N(0, 1) rounded to bf16.
* ``attention_grad_inputs``: a gradient of the attention output dA [L, h] ~
  N(0, (0.02 sqrt(h))^2) rounded to fp16.
"""
from __future__ import annotations

import math

import torch

WEIGHT_STD = 0.02
WEIGHT_NAMES = ("wq", "wk", "wv", "wo", "w1", "w2")


def _draw(gen: torch.Generator, shape, std: float, dtype=torch.bfloat16) -> torch.Tensor:
    t = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def _weights(gen: torch.Generator, h: int, F: int) -> dict:
    shapes = {"wq": (h, h), "wk": (h, h), "wv": (h, h), "wo": (h, h),
              "w1": (h, F), "w2": (F, h)}
    return {n: _draw(gen, shapes[n], WEIGHT_STD) for n in WEIGHT_NAMES}


def layer_inputs(T: int, h: int, F: int, seed: int) -> dict:
    """Full-sequence activations X [T, h] and the six layer weights (bf16, CPU)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    out = {"x": _draw(gen, (T, h), 1.0)}
    out.update(_weights(gen, h, F))
    return out


def rank_inputs(L: int, T: int, h: int, F: int, seed: int,
                kv_std: float | None = None) -> dict:
    """One rank's tokens and the weights (bf16), stand-in full-sequence K/V (fp16); CPU."""
    if kv_std is None:
        kv_std = WEIGHT_STD * math.sqrt(h)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    out = {"x_local": _draw(gen, (L, h), 1.0)}
    out.update(_weights(gen, h, F))
    out["k_full"] = _draw(gen, (T, h), kv_std, torch.float16)
    out["v_full"] = _draw(gen, (T, h), kv_std, torch.float16)
    return out


def mlp_backward_inputs(L: int, h: int, F: int, seed: int) -> dict:
    """Residual rows Y1 (fp32), the weights (bf16) and a loss gradient dY (bf16); CPU."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    out = {"y1": _draw(gen, (L, h), 1.0, torch.float32)}
    out.update(_weights(gen, h, F))
    out["dy"] = _draw(gen, (L, h), 1.0)
    return out


def attention_grad_inputs(L: int, h: int, seed: int) -> torch.Tensor:
    """A gradient of the attention output dA [L, h] ~ N(0, (0.02 sqrt(h))^2),
    the spread dY1 Wo^T has for dY1 ~ N(0, 1) and weights ~ N(0, 0.02^2),
    rounded to fp16 (the format the attention backward takes it in); CPU."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return _draw(gen, (L, h), WEIGHT_STD * math.sqrt(h), torch.float16)


def sample_rows(n_rows: int, n_sample: int, seed: int, must: tuple = ()) -> list:
    """A deterministic sorted sample of row indices in [0, n_rows), including `must`."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed + 7919)
    picked = set(int(m) for m in must if 0 <= int(m) < n_rows)
    extra = torch.randperm(n_rows, generator=gen)[: max(0, n_sample)].tolist()
    for e in extra:
        if len(picked) >= len(set(must)) + n_sample:
            break
        picked.add(int(e))
    return sorted(picked)
