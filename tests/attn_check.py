"""Comparison of tree-attention outputs with the oracle, shared by the GPU
parity tests and the CPU test that shows the comparison can fail.

Two criteria, both required:
  - max-abs error <= atol (2e-2 for bf16 against the fp64 oracle, the
    workload tolerance);
  - per output row, relative L2 error ||o - o_ref||_2 / ||o_ref||_2 <= rel.
The second one scales with the output: at a 32K-key prefix each output
element is ~0.01, so a max-abs bound of 2e-2 alone would accept a result
that lost a tenth of the keys, while dropping a single 128-key tile moves a
row by several percent of its norm.  bf16 probabilities and the bf16
output rounding keep the kernel's rows within a few 1e-3.
"""
from __future__ import annotations

import numpy as np

ATOL_BF16 = 2e-2
REL_BF16 = 1e-2
ATOL_F32 = 1e-4
REL_F32 = 1e-4


def attention_errors(got, ref):
    """(max-abs error, max per-row relative L2 error) over rows of the last axis."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    d = got.reshape(-1, got.shape[-1]) - ref.reshape(-1, ref.shape[-1])
    num = np.linalg.norm(d, axis=1)
    den = np.linalg.norm(ref.reshape(-1, ref.shape[-1]), axis=1)
    rel = np.where(den > 0, num / np.where(den > 0, den, 1.0), num)
    return float(np.abs(d).max()) if d.size else 0.0, float(rel.max()) if rel.size else 0.0


def assert_attention_close(got, ref, bf16: bool = True, what: str = ""):
    atol, rel = (ATOL_BF16, REL_BF16) if bf16 else (ATOL_F32, REL_F32)
    err, rl2 = attention_errors(got, ref)
    assert err <= atol and rl2 <= rel, (
        f"{what}: max-abs {err:.3e} (limit {atol:g}), max rel-L2 {rl2:.3e} (limit {rel:g})")
    return err, rl2
