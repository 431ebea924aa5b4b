"""The inputs of the GPU test test_score_jumps_beyond_fp32_range reach the
regimes that test is about (CPU only; no value here comes from the CUDA path).

For rank 0 of each of the test's shapes, a row's score against a spiked key is
compared with the maximum of the row's first key tile (keys 0..127, which
holds no spike), in log2 units of the softmax, s * scale * log2(e): the rows
must include jumps past fp32's range (more than 128), jumps between 8 and 128
(probabilities past fp16 but inside fp32) and rows within 8.  Q here is LN1(x)
Wq in fp64 from the same seeded inputs; the kernels' fp16 rounding moves these
jumps by far less than the margins the checks leave.
"""
import math

import numpy as np
import pytest
import torch

from folded_tensor_sequence_rank_b200 import inputs

SHAPES = [(512, 256, 4, 1024, 2, 2000.0), (2048, 512, 4, 2048, 2, 1500.0)]  # those of the GPU test


def rank0_jumps(T, h, H, F, D, spike):
    L, hd = T // D, h // H
    raw = inputs.rank_inputs(L, T, h, F, 9)
    kf = raw["k_full"].float()
    spikes = torch.arange(200, T, 97)
    kf[spikes] *= spike
    K = kf.to(torch.float16).double().numpy()
    x = raw["x_local"].double().numpy()
    xn = (x - x.mean(1, keepdims=True)) / np.sqrt(x.var(1, keepdims=True) + 1e-5)
    q = xn @ raw["wq"].double().numpy()
    c = T // (2 * D)
    pos = np.r_[np.arange(c), np.arange((2 * D - 1) * c, 2 * D * c)]  # rank 0: chunks 0 and 2D-1
    scale_log2 = math.log2(math.e) / math.sqrt(hd)
    sp = spikes.numpy()
    jumps = []
    for hh in range(H):
        s = (q[:, hh * hd:(hh + 1) * hd] @ K[:, hh * hd:(hh + 1) * hd].T) * scale_log2
        for i, p in enumerate(pos):
            seen = sp[sp <= p]
            if len(seen):
                jumps.append((s[i, seen] - s[i, :min(128, p + 1)].max()).max())
    return np.array(jumps)


@pytest.mark.parametrize("T,h,H,F,D,spike", SHAPES)
def test_score_jump_inputs_reach_every_regime(T, h, H, F, D, spike):
    j = rank0_jumps(T, h, H, F, D, spike)
    assert (j > 160).mean() > 0.5       # 2^x overflows fp32 (with a margin of 32 log2 units)
    assert ((j > 16) & (j < 100)).sum() > 20  # past fp16, inside fp32
    assert (j < 4).sum() > 20           # no rescale needed
