"""CPU check of the FMA-pipe 2^x the attention softmax uses for one
exponential pair in four (Cody-Waite split + degree-3 minimax polynomial,
exp2_fma2): the constants are read from the CUDA source and the same
per-lane fp32 operations are emulated with numpy."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "medusa_head_speculative_02_b200", "csrc", "common.cuh")


def _coeffs():
    """kExp2C0..kExp2C3 as the CUDA source defines them."""
    body = open(SRC).read()
    c = {}
    for k in range(4):
        m = re.search(r"constexpr float kExp2C%d = ([0-9.]+)f;" % k, body)
        c[k] = np.float32(float(m.group(1)))
    return c[0], c[1], c[2], c[3]


def _poly_parts(x):
    x = np.maximum(np.float32(x), np.float32(-126.0)).astype(np.float32)
    c0, c1, c2, c3 = _coeffs()
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0)).astype(np.float32)).astype(np.float32)
    p = np.float32(c3)
    for c in (c2, c1, c0):            # fp32 fused multiply-add per step
        p = (p.astype(np.float64) * f + c).astype(np.float32)
    return np.atleast_1d(t), np.atleast_1d(p)


def _exp2_fma(x):
    """As the kernel forms it: one integer multiply-add per lane, the bits
    of t times 2^23 plus the bits of p, modulo 2^32."""
    t, p = _poly_parts(x)
    u = (p.view(np.uint32).astype(np.uint64) + t.view(np.uint32).astype(np.uint64) * (1 << 23))
    return (u & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_exponent_insertion_equals_adding_n_to_the_exponent_field():
    # n = bits(t) - bits(1.5 * 2^23) = round(x); p * 2^n by adding n << 23
    x = np.linspace(-126.0, 9.0, 200001).astype(np.float32)
    t, p = _poly_parts(x)
    n = t.view(np.int32) - np.int32(0x4B400000)
    assert np.array_equal(n, np.rint(np.maximum(x, -126.0)).astype(np.int32))
    direct = (p.view(np.int32) + (n << 23)).view(np.float32)
    assert np.array_equal(_exp2_fma(x).view(np.uint32), direct.view(np.uint32))


def test_exp2_fma_relative_error_bound():
    x = np.linspace(-125.9, 8.0, 400001).astype(np.float32)
    y = _exp2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 2.0e-4            # far below bf16's 2^-9 = 2e-3
    assert abs(_exp2_fma(np.float32(0.0)) - 1.0) < 2e-4
    # very negative arguments collapse to 2^-126 (callers zero masked entries)
    assert abs(_exp2_fma(np.float32(-1000.0)) / 2.0 ** -126 - 1.0) < 2e-4
