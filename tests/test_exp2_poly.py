"""CPU checks of the arithmetic building blocks the attention softmax uses in
place of library calls: the FMA-pipe 2^x (Cody-Waite split + degree-3
minimax polynomial) and the integer bf16 packing.  The constants are read
from the CUDA source and the same fp32 operations are emulated with numpy."""
import os
import re

import numpy as np
import torch

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "medusa_head_speculative_02_b200", "csrc", "common.cuh")


def _coeffs():
    body = open(SRC).read()
    fn = body[body.index("float exp2_fma(float x)"):]
    fn = fn[:fn.index("}")]
    c = [np.float32(float(v)) for v in re.findall(r"(\d+\.\d+)f", fn)]
    # fmaf(fmaf(fmaf(c3, f, c2), f, c1), f, c0), with 12582912 the rounding constant
    c = [v for v in c if v != np.float32(12582912.0) and v != np.float32(126.0)]
    c3, c2, c1, c0 = c
    return c0, c1, c2, c3


def _exp2_fma(x):
    x = np.maximum(np.float32(x), np.float32(-126.0)).astype(np.float32)
    c0, c1, c2, c3 = _coeffs()
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = t.view(np.int32) - np.int32(0x4B400000)
    f = (x - (t - np.float32(12582912.0)).astype(np.float32)).astype(np.float32)
    p = np.float32(c3)
    for c in (c2, c1, c0):            # fp32 fused multiply-add per step
        p = (p.astype(np.float64) * f + c).astype(np.float32)
    return (p.view(np.int32) + (n << 23)).view(np.float32)


def test_exp2_fma_relative_error_bound():
    x = np.linspace(-125.9, 8.0, 400001).astype(np.float32)
    y = _exp2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 2.0e-4            # far below bf16's 2^-9 = 2e-3
    assert abs(_exp2_fma(np.float32(0.0)) - 1.0) < 2e-4
    # very negative arguments collapse to 2^-126 (callers zero masked entries)
    assert abs(_exp2_fma(np.float32(-1000.0)) / 2.0 ** -126 - 1.0) < 2e-4


def test_bf16_pack_rounds_like_round_to_nearest_away_from_ties():
    g = np.random.default_rng(0)
    v = np.concatenate([g.uniform(0, 256, 100000), [0.0, 1.0, 255.99, 1e-30]]).astype(np.float32)
    packed = ((v.view(np.uint32) + np.uint32(0x8000)) >> 16).astype(np.uint16)
    got = torch.from_numpy(packed.view(np.int16)).view(torch.bfloat16).float().numpy()
    ref = torch.from_numpy(v).bfloat16().float().numpy()   # round to nearest even
    diff = got != ref
    # only exact ties may differ (half up vs half to even)
    ties = (v.view(np.uint32) & np.uint32(0xFFFF)) == np.uint32(0x8000)
    assert not (diff & ~ties).any()
