"""The attention kernel computes one in four softmax exponentials with a
polynomial (exp2_poly in csrc/ptx.cuh) instead of the MUFU unit.  This replays
its fp32 steps on the CPU, with the constants read from the kernel source,
and checks them against 2^x: relative error within the polynomial's fitted
bound plus fp32 rounding, over the whole input range the softmax produces."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "folded_tensor_sequence_rank_b200", "csrc", "ptx.cuh")


def kernel_constants():
    body = open(SRC).read().split("float exp2_poly(float x)")[1].split("}")[0]
    c = [float(v) for v in re.findall(r"(-?\d+\.\d+(?:e-?\d+)?)f", body)]
    # order in source: clamp (-125), magic, c4, c3, c2, c1, c0
    assert c[0] == -125.0 and c[1] == 12582912.0
    return c[2:]


def test_packed_variant_uses_the_same_constants():
    body = open(SRC).read().split("float2 exp2_poly2(float2 x)")[1].split("return")[0]
    c = [float(v) for v in re.findall(r"(-?\d+\.\d+(?:e-?\d+)?)f", body)]
    uniq = []
    for v in c:
        if v not in uniq:
            uniq.append(v)
    assert uniq == [-125.0, 12582912.0, -12582912.0] + kernel_constants()


def exp2_poly_fp32(x):
    c4, c3, c2, c1, c0 = (np.float32(v) for v in kernel_constants())
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = (c4 * f + c3).astype(np.float32)     # fmaf rounds once; the error bound below covers both
    p = (p * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_exp2_poly_relative_error():
    x = np.concatenate([np.linspace(-124.9, 8.0, 400001), np.arange(-124, 9).astype(np.float64),
                        np.arange(-124, 9) + 0.5]).astype(np.float32)
    got = exp2_poly_fp32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 4e-6, rel.max()


def test_exp2_poly_clamps_and_signs():
    x = np.array([-np.inf, -1000.0, -125.0, -126.5, 0.0, 8.0], dtype=np.float32)
    y = exp2_poly_fp32(x).astype(np.float64)
    assert np.all(y > 0) and np.all(np.isfinite(y))
    assert y[0] == y[1] == y[3] and abs(y[2] / 2.0 ** -125 - 1) < 4e-6   # clamp at 2^-125
    assert abs(y[4] - 1) < 4e-6 and abs(y[5] / 256 - 1) < 4e-6
    # below fp16's smallest subnormal: the probability rounds to zero
    assert np.float16(y[0]) == 0
