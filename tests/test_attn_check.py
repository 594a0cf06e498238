"""CPU: the attention comparison used by the GPU parity tests can fail.

A kernel that skipped one 128-key tile of the prefix would produce, for
every row, the exact attention over the prefix without those keys.  That is
computed here with the oracle on a perturbed input (the cache with the
tile's slots removed, the prefix 128 shorter) and compared, with the same
function the GPU tests use, against the oracle on the full input: the
comparison must reject it at the long-context and 8B-GQA shapes, where
max-abs 2e-2 alone accepts it.  The exact result rounded to bf16 must
pass.
"""
import math

import numpy as np
import pytest
import torch

from attn_check import REL_BF16, assert_attention_close, attention_errors
from oracle import medusa_oracle as O


def _slice(L, N, G, dh, seed):
    """One (sequence, kv-head) of a workload: prefix L, N tree nodes, GQA group G."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(1, N, G, dh, generator=g).bfloat16()
    kc = torch.randn(1, L + N, 1, dh, generator=g).bfloat16()
    vc = torch.randn(1, L + N, 1, dh, generator=g).bfloat16()
    return q, kc, vc


@pytest.mark.parametrize("L,tree,G", [(32768, (5, 3, 256), 1), (8192, (5, 8, 128), 4)])
def test_dropping_one_key_tile_fails_the_check(L, tree, G):
    K, s, N = tree
    dh = 128
    q, kc, vc = _slice(L, N, G, dh, seed=L + G)
    plan = O.tree_plan(K, s, N)
    scale = 1.0 / math.sqrt(dh)
    rows = [(0, i, g) for i in (0, N // 2, N - 1) for g in range(G)]
    ref = O.tree_attention(q, kc, vc, [L], plan, scale, rows=rows)

    # the exact result in the kernel's output precision passes
    assert_attention_close(torch.tensor(ref).bfloat16().double().numpy(), ref,
                           what="bf16-rounded exact result")

    n_tiles = L // 128
    for tile in (0, n_tiles // 2, n_tiles - 1):
        keep = torch.cat([torch.arange(0, tile * 128), torch.arange((tile + 1) * 128, L + N)])
        dropped = O.tree_attention(q, kc[:, keep], vc[:, keep], [L - 128], plan, scale,
                                   rows=rows)
        err, rl2 = attention_errors(dropped, ref)
        assert rl2 > 2 * REL_BF16, (tile, err, rl2)
        with pytest.raises(AssertionError):
            assert_attention_close(dropped, ref, what=f"tile {tile} dropped")
        if L >= 32768:
            # what the relative criterion adds: max-abs alone cannot see it
            assert err <= 2e-2, err


def test_errors_of_identical_and_empty_inputs():
    x = np.random.default_rng(0).standard_normal((5, 128))
    assert attention_errors(x, x) == (0.0, 0.0)
    err, rl2 = attention_errors(np.zeros((2, 4)), np.zeros((2, 4)))
    assert err == 0.0 and rl2 == 0.0
